"""Benchmark of the DSA hot path: query tokens/s through indexer + top-k + sparse MLA.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path (dsa_forward: Lightning-Indexer
scores, per-query top-k, sparse MLA) over one batch of synthetic inputs that
already sit in HBM.  The default workload is the 32K-context chunked prefill
(4096 new queries after a 28672-token prefix, top-2048, 128 MLA heads).
Rank 0 prints one JSON line.

With N > 1 (torchrun, one process per GPU) every rank runs its own replica of
the workload (weak scaling, no data-path collective); value = all ranks'
tokens / the slowest rank's time.

The e2e object is the same metric through the same C-ABI call with every
step copying all of its inputs from pinned host memory and its results (out,
idx, lse) back; consecutive steps overlap on three streams (copy in, compute,
copy out) over double-buffered device buffers, as a serving loop runs them, and
the timed region spans the first copy in to the last copy out.

The prep object times the upstream preparation of the same batch outside the
step (the per-128 FP8 quantiser over its q, the cache write of its new
tokens) against the HBM roofline; it is not part of `value`.

On one GPU the line also carries `workloads`: the forward step and its three
stages, each against its roofline, for the other four configurations (decode
at 16K-32K context, speculative decode at 128K, the 8K prefill and the tiny
prefill), so one run reports all five.  `--no-extra-workloads` skips them.

Roofline denominators: MEASURED_PEAKS.json's HBM copy bandwidth and burst
bf16 GEMM rate (each stage is timed on its own, not inside a seconds-long
loop), and an FP8 e4m3 GEMM rate measured at the start of the run
(torch._scaled_mm), 2 x bf16 if that probe fails.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import threading
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "query tokens/s through indexer+top-k+sparse MLA @32K ctx; % of roofline"
UNIT = "query tokens/s"
DEFAULT_WORKLOAD = "chunked_prefill_28k_4k"
L2_FLUSH_BYTES = 256 << 20


def peaks():
    """Roofline denominators: MEASURED_PEAKS.json (HBM copy bandwidth and the
    burst cuBLAS bf16 GEMM rate) when present, else the profiling fallback.
    Each stage is timed on its own (per-launch CUDA events over a short loop),
    so the burst GEMM figure is the matching denominator, not the sustained one.
    The FP8 peak is filled in by fp8_peak_probe() at run time."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        pk = {"hbm_gbs": m["hbm_gbs"], "bf16_tflops": m["bf16_tflops"], "source": "measured"}
    else:
        pk = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
    pk["fp8_tflops"] = 2.0 * pk["bf16_tflops"]
    pk["fp8_source"] = "2 x bf16 burst (nominal dense FP8/bf16 ratio)"
    return pk


def fp8_peak_probe(dev, n=8192, reps=10):
    """Burst FP8 e4m3 dense GEMM rate (torch._scaled_mm, n^3, best of `reps`,
    CUDA events): the denominator of the FP8 indexer's tensor roofline.
    Returns (TFLOP/s, description) or (None, reason)."""
    import torch
    try:
        g = torch.Generator(device=dev).manual_seed(99)
        a = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn).t()   # column-major operand
        one = torch.ones((), dtype=torch.float32, device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1) / 1e3)
        del a, b
        return 2.0 * n ** 3 / best / 1e12, f"measured: torch._scaled_mm e4m3 {n}^3, best of {reps} (burst)"
    except Exception as exc:   # the nominal ratio stands in
        return None, f"probe failed ({type(exc).__name__}); 2 x bf16 burst"


# ----------------------------------------------------------------- work model
def work_model(x):
    """Algorithmic FLOPs and bytes of each stage for a DSAInputs batch."""
    b = x.batch
    t = b.q_pos.astype(np.int64)
    n_valid = t + 1
    pairs = int(n_valid.sum())
    k = x.k_sel
    n_sel = np.minimum(n_valid, k)
    H = x.n_heads
    # keys each sequence's queries can reach (max t + 1 per sequence)
    reach = np.zeros(b.num_seqs, np.int64)
    np.maximum.at(reach, b.q_seq, n_valid)
    idx_flops = pairs * 2 * 64 * 128
    idx_bytes = int(reach.sum()) * (128 + 4) + b.total_q * (64 * 128 + 64 * 4 * 2) + pairs * 4
    topk_bytes = pairs * 4 + b.total_q * k * 4
    mla_flops = int((n_sel * H).sum()) * 2 * (576 + 512)
    # every latent row a sequence's selections may touch is read once (upper bound: the reachable prefix)
    mla_bytes = int(np.minimum(reach, n_sel.max() * np.bincount(b.q_seq, minlength=b.num_seqs)).sum()) * 1152 \
        + b.total_q * (H * 576 * 2 + H * 512 * 2 + k * 4 + H * 4)
    return {"indexer": {"flops": idx_flops, "bytes": idx_bytes, "peak": "fp8"},
            "topk": {"flops": 0, "bytes": topk_bytes, "peak": None},
            "sparse_mla": {"flops": mla_flops, "bytes": mla_bytes, "peak": "bf16"}}


def prep_work(total_q):
    """Bytes of the upstream preparation of one batch: the FP8 quantiser over q
    (total_q x 64 vectors: 256 B read, 128 + 4 B written each) and the cache
    write of the new tokens (key 256 B read, 132 B written; latent 1152 B read
    and written)."""
    return {"quantize_q": {"flops": 0, "bytes": total_q * 64 * (256 + 128 + 4), "peak": None},
            "cache_write": {"flops": 0, "bytes": total_q * (256 + 132 + 2 * 1152), "peak": None}}


def prep_line(prep_sec, total_q, pk):
    """The preparation kernels' times against their HBM roofline (not part of `value`)."""
    if prep_sec is None or "error" in prep_sec:
        return prep_sec
    w = prep_work(total_q)
    return {n: roofline_entry(n, w[n], prep_sec[n], pk) for n in w}


def roofline_entry(stage, work, sec, pk):
    """One stage against its roofline: the slower of its FLOPs at the tensor
    peak of its type (burst) and its algorithmic bytes at the HBM peak decides
    the bound; achieved = that work / the measured time."""
    tensor_peak = {"fp8": pk["fp8_tflops"], "bf16": pk["bf16_tflops"], None: None}[work["peak"]]
    t_flops = work["flops"] / (tensor_peak * 1e12) if tensor_peak else 0.0
    t_bytes = work["bytes"] / (pk["hbm_gbs"] * 1e9)
    if t_flops >= t_bytes:
        achieved = work["flops"] / sec / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": achieved / tensor_peak, "ideal_us": t_flops * 1e6, "us": sec * 1e6,
                "work": work["flops"]}
    achieved = work["bytes"] / sec / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / pk["hbm_gbs"], "ideal_us": t_bytes * 1e6, "us": sec * 1e6, "work": work["bytes"]}


def ncu_traffic(kernel_file, kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source
    is unchanged since the capture; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel_key)
    if not d:
        return None
    src = os.path.join(ROOT, "long_context_sparse_lightning_b200", "csrc", kernel_file)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return d.get("bytes_per_launch") if d.get("source_sha") == sha else None


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region.

    Polls NVML every few milliseconds from a thread (the timed region can be
    tens of milliseconds, shorter than one nvidia-smi period); falls back to
    an `nvidia-smi -lms` subprocess when NVML is unavailable."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.sm, self.mask, self.mx, self.lines = [], 0, None, []
        self.proc = self.thread = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        prop = torch.cuda.get_device_properties(self.cuda_index)
        bus = f"{prop.pci_domain_id:08X}:{prop.pci_bus_id:02X}:{prop.pci_device_id:02X}.0"
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId_v2(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.stop = threading.Event()

            def poll():
                while True:
                    self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                    self.mask |= int(get_reasons(h))
                    if self.stop.wait(0.005):
                        break

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
        except Exception:
            q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            try:
                self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={q}",
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for l in out.splitlines():
                f = [v.strip() for v in l.split(",")]
                if len(f) < 9:
                    continue
                try:
                    self.sm.append(float(f[1]))
                    self.mx = float(f[2])
                except ValueError:
                    continue
                for n, v in zip(names, f[5:9]):
                    if v.lower() == "active":
                        self.mask |= self.REASONS[n]

    def summary(self):
        reasons = sorted(n for n, bit in self.REASONS.items() if self.mask & bit)
        return {"sm_mhz": statistics.median(self.sm) if self.sm else None, "sm_max_mhz": self.mx,
                "reasons": reasons, "samples": len(self.sm)}


# --------------------------------------------------------------- CPU oracle
def oracle_rows_per_sec(x, budget_s=15.0, min_rows=4, max_rows=4096, seed=7):
    """Time the fp64 oracle (scores -> top-k -> sparse MLA) on query rows of x
    until ~budget_s of CPU time; returns (rows/s, rows done, seconds)."""
    from oracle import indexer, mla, topk
    rng = np.random.default_rng(seed)
    order = rng.permutation(x.batch.total_q)
    done = 0
    t0 = time.perf_counter()
    while done < min(max_rows, x.batch.total_q):
        r = int(order[done])
        (_, t, I, B), = indexer.scores(x, [r])
        sel, _ = topk.select(I, x.k_sel)
        mla.sparse(x, topk.padded(sel, x.k_sel)[None, :], [r])
        done += 1
        el = time.perf_counter() - t0
        if done >= min_rows and el >= budget_s:
            break
    el = time.perf_counter() - t0
    return done / el, done, el


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


# --------------------------------------------------------------------- main
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def slowest_rank(sec, pg, device):
    """The largest of the ranks' elapsed times (every rank gets it); `sec` as is
    without a process group.  Multi-GPU numbers are timed as the max over ranks."""
    if pg is None:
        return sec
    import torch
    t = torch.tensor([float(sec)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, rows_per_rank, steps, slowest_sec):
    """Query tokens/s of all ranks together: every rank runs its own replica of
    the workload (weak scaling), so the job ends with the slowest rank."""
    return world * rows_per_rank * steps / slowest_sec


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    from dsa_inputs import make_inputs
    x = make_inputs(args.workload, seed=0)
    per_step = max(1, args.ref_rows)
    times = []
    done_rows = 0
    for s in range(args.warmup + args.steps):
        rps, n, el = oracle_rows_per_sec(x, budget_s=0.0, min_rows=per_step, max_rows=per_step, seed=100 + s)
        if s >= args.warmup:
            times.append(el)
            done_rows += n
    total = sum(times)
    value = done_rows / total
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(x, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{per_step} query rows of {args.workload} per step (scores over the "
                                       f"full causal prefix, exact top-k, sparse MLA), fp64 numpy"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(x, args):
    b = x.batch
    return {"workload": x.workload.name, "description": x.workload.description, "n_q": b.total_q,
            "num_seqs": b.num_seqs, "max_kv_len": b.max_kv_len, "k_sel": x.k_sel, "n_heads": x.n_heads,
            "index_heads": 64, "index_dim": 128, "latent_dim": 576, "value_dim": 512,
            "l2": "flushed between timed steps (256 MiB write, outside the events)", "seed": 0}


EXTRA_WORKLOADS = ["decode_64x16k_32k", "spec_decode_8x2_128k", "prefill_8k", "tiny_prefill_512"]


def measure(x, args, dev, pg, world, full, min_region_s=0.0):
    """Time the forward step of one workload on resident inputs (L2 flushed
    between steps), then each stage on its own; with `full`, also end to end
    from pinned host buffers and the upstream preparation kernels."""
    import torch
    import long_context_sparse_lightning_b200 as dsa
    from dsa_inputs.torch_io import host_tensors

    b = x.batch
    host = host_tensors(x, pin=full)
    t = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    batch = dsa.Batch(t["cu_q"], t["kv_len"], t["kv_start"], b.total_q, b.max_q_per_seq, b.max_kv_len, b.total_keys)
    k, H = x.k_sel, x.n_heads
    idx = torch.empty((b.total_q, k), dtype=torch.int32, device=dev)
    out = torch.empty((b.total_q, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((b.total_q, H), dtype=torch.float32, device=dev)
    ws = dsa.workspace(dsa.OP_FORWARD, batch, k, H, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    def step():
        dsa.forward(batch, t["q8"], t["q_scale"], t["w"], t["k8"], t["k_scale"], k, t["q_mla"], t["latent"],
                    x.sm_scale, idx, out, lse, ws)

    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for _ in range(args.warmup):
        step()
    w1.record(stream)
    torch.cuda.synchronize()
    dsa.check_device_error(ws)
    steps = args.steps
    if min_region_s > 0:        # short steps: enough of them for the clock samples to mean something
        per = w0.elapsed_time(w1) / 1e3 / args.warmup
        steps = int(min(500, max(steps, math.ceil(min_region_s / max(per, 1e-6)))))

    # ---- K steps on resident inputs, L2 flushed between steps ----
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for i in range(steps):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    dsa.check_device_error(ws)
    sec = slowest_rank(sum(a.elapsed_time(c) for a, c in ev) / 1e3, pg, dev)
    res = {"steps": steps, "sec": sec, "value": whole_job_rate(world, b.total_q, steps, sec),
           "launches_per_step": dsa.forward_launches(batch, k, H), "clocks": clk.summary()}
    if getattr(args, "forward_only", False):      # profiling runs: the forward launches and nothing else
        return res

    # ---- per-stage device time (same stream, CUDA events between the launches) ----
    ld = ((b.max_kv_len + 3) // 4) * 4
    scores = torch.empty((b.total_q, ld), dtype=torch.float32, device=dev)
    # one workspace for the three standalone stages: the largest of their sizes
    ws_op = max((dsa.OP_TOPK, dsa.OP_SPARSE_MLA), key=lambda op: dsa.workspace_size(op, batch, k, H))
    ws_s = dsa.workspace(ws_op, batch, k, H, device=dev)
    st_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(args.warmup + steps):
        flush.fill_(float(i))
        e = st_ev[i - args.warmup] if i >= args.warmup else None
        if e: e[0].record(stream)
        dsa.indexer_scores(batch, t["q8"], t["q_scale"], t["w"], t["k8"], t["k_scale"], scores, ws_s)
        if e: e[1].record(stream)
        dsa.topk(batch, scores, k, idx, ws_s)
        if e: e[2].record(stream)
        dsa.sparse_mla(batch, t["q_mla"], t["latent"], idx, k, x.sm_scale, out, lse, ws_s)
        if e: e[3].record(stream)
    torch.cuda.synchronize()
    dsa.check_device_error(ws_s)
    res["stage_sec"] = {name: sum(e[j].elapsed_time(e[j + 1]) for e in st_ev) / 1e3 / steps
                        for j, name in enumerate(["indexer", "topk", "sparse_mla"])}
    del scores, ws_s
    if not full:
        return res

    # ---- end to end through the C ABI from pinned host buffers ----
    # Every step copies all of its inputs in and its results (out, idx, lse)
    # out; consecutive steps overlap on three streams (copy in / compute /
    # copy out) over double-buffered device inputs and outputs, the way a
    # serving loop runs them.  The timed region spans the first step's copy in
    # to the last step's copy out.
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    idx_h = torch.empty(idx.shape, dtype=idx.dtype, pin_memory=True)
    lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in (out_h, idx_h, lse_h))
    sets = [(t, batch, (out, idx, lse), ws)]
    t2 = {name: torch.empty_like(v) for name, v in t.items()}
    b2 = dsa.Batch(t2["cu_q"], t2["kv_len"], t2["kv_start"], b.total_q, b.max_q_per_seq, b.max_kv_len, b.total_keys)
    sets.append((t2, b2, (torch.empty_like(out), torch.empty_like(idx), torch.empty_like(lse)),
                 dsa.workspace(dsa.OP_FORWARD, b2, k, H, device=dev)))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        j = i % 2
        tj, bj, (oj, ij, lj), wsj = sets[j]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[j])        # step i-2 no longer reads these inputs
            for name, v in host.items():
                tj[name].copy_(v, non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if i >= 2:
            stream.wait_event(ev_out[j])           # step i-2's results have left these buffers
        dsa.forward(bj, tj["q8"], tj["q_scale"], tj["w"], tj["k8"], tj["k_scale"], k, tj["q_mla"], tj["latent"],
                    x.sm_scale, ij, oj, lj, wsj)
        ev_done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[j])
            out_h.copy_(oj, non_blocking=True)
            idx_h.copy_(ij, non_blocking=True)
            lse_h.copy_(lj, non_blocking=True)
            ev_out[j].record(s_out)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(s_in)
    for i in range(args.warmup, args.warmup + steps):
        e2e_step(i)
    e_end.record(s_out)
    torch.cuda.synchronize()
    for _, _, _, wsj in sets:
        dsa.check_device_error(wsj)
    e2e_sec = slowest_rank(e_start.elapsed_time(e_end) / 1e3, pg, dev)
    res["e2e"] = {"value": whole_job_rate(world, b.total_q, steps, e2e_sec), "unit": UNIT,
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del sets, t2

    # ---- upstream preparation, outside the step: the per-128 FP8 quantiser
    # over this batch's q (bf16 -> codes + scales) and the write of its new
    # tokens' keys and latent rows into caches of the workload's size ----
    prep_sec = None
    try:
        gen = torch.Generator(device=dev).manual_seed(1234 + dev.index)
        q_bf = torch.randn((b.total_q, 64, 128), generator=gen, device=dev).to(torch.bfloat16)
        k_bf = torch.randn((b.total_q, 128), generator=gen, device=dev).to(torch.bfloat16)
        lat_bf = torch.randn((b.total_q, 576), generator=gen, device=dev).to(torch.bfloat16)
        q8p = torch.empty((b.total_q, 64, 128), dtype=torch.uint8, device=dev)
        qsp = torch.empty((b.total_q, 64), dtype=torch.float32, device=dev)
        k8c, ksc, latc = torch.empty_like(t["k8"]), torch.empty_like(t["k_scale"]), torch.empty_like(t["latent"])
        ws_p = dsa.workspace(dsa.OP_CACHE_WRITE, batch, 0, 0, device=dev)
        pe = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(args.warmup + steps):
            flush.fill_(float(i))
            e = pe[i - args.warmup] if i >= args.warmup else None
            if e: e[0].record(stream)
            dsa.quantize_fp8(q_bf, q8p, qsp)
            if e: e[1].record(stream)
            dsa.cache_write(batch, k_bf, lat_bf, k8c, ksc, latc, ws_p)
            if e: e[2].record(stream)
        torch.cuda.synchronize()
        dsa.check_device_error(ws_p)
        prep_sec = {"quantize_q": sum(e[0].elapsed_time(e[1]) for e in pe) / 1e3 / steps,
                    "cache_write": sum(e[1].elapsed_time(e[2]) for e in pe) / 1e3 / steps}
        del q_bf, k_bf, lat_bf, q8p, qsp, k8c, ksc, latc
    except Exception as exc:     # reported in the line; the step's numbers above stand
        prep_sec = {"error": f"{type(exc).__name__}: {exc}"[:200]}
    res["prep_sec"] = prep_sec
    return res


def stage_lines(x, stage_sec, pk):
    wm = work_model(x)
    return {n: roofline_entry(n, wm[n], stage_sec[n], pk) for n in stage_sec}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=8, help="query rows per reference step")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="measure only --workload (by default a 1-GPU run also measures the other four configs)")
    ap.add_argument("--forward-only", action="store_true",
                    help="for profiler command lines: only the warm-up and timed forward steps of --workload "
                         "(no stage timing, end-to-end run, preparation kernels, other configs or CPU baseline)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)

    import torch
    from dsa_inputs import make_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as td
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = td

    x = make_inputs(args.workload, seed=rank)
    r = measure(x, args, dev, pg, world, full=not args.forward_only)
    if args.forward_only:
        if pg:
            pg.barrier()
            pg.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world,
                              "steps": r["steps"], "warmup": args.warmup, "ms_per_step": 1e3 * r["sec"] / r["steps"],
                              "forward_only": True, "config": config_of(x, args),
                              "gpu_launches": r["launches_per_step"] * r["steps"], "clocks": r["clocks"]}), flush=True)
        return 0
    extra = {}
    if world == 1 and not args.no_extra_workloads:
        for name in EXTRA_WORKLOADS:
            if name == args.workload:
                continue
            xe = make_inputs(name, seed=rank)
            re_ = measure(xe, args, dev, None, world, full=False, min_region_s=0.05)
            extra[name] = (xe, re_)
            torch.cuda.empty_cache()
    pk = peaks()
    fp8, fp8_src = fp8_peak_probe(dev)
    if fp8 is not None:
        pk["fp8_tflops"], pk["fp8_source"] = fp8, fp8_src
    else:
        pk["fp8_source"] = fp8_src

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0

    stages = stage_lines(x, r["stage_sec"], pk)
    dom = max(r["stage_sec"], key=r["stage_sec"].get)
    kfile = {"indexer": "indexer_sm100.cu", "topk": "topk.cu", "sparse_mla": "sparse_mla_sm100.cu"}[dom]
    roof = {k2: v for k2, v in stages[dom].items() if k2 != "work"}
    roof["kernel"] = dom
    roof["traffic"] = ncu_traffic(kfile, dom)
    roof["peak_source"] = pk["source"] + (" burst bf16 GEMM" if stages[dom]["peak"] == pk["bf16_tflops"] and
                                          roof["unit"] == "TFLOP/s" else "")
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        rps, n_rows, el = oracle_rows_per_sec(x, budget_s=args.cpu_budget)
        cpu = {"value": rps, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n_rows} query rows of {args.workload} ({el:.1f} s): fp64 scores over each row's "
                         f"causal prefix, exact top-k, sparse MLA"}
    line = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * r["sec"] / r["steps"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3+bf16/f16", "data": "synthetic",
            "config": config_of(x, args), "roofline": roof,
            "stages": stages, "peaks": {k2: pk[k2] for k2 in ("hbm_gbs", "bf16_tflops", "fp8_tflops", "fp8_source",
                                                              "source")},
            "cpu_baseline": cpu, "e2e": r["e2e"],
            "gpu_launches": r["launches_per_step"] * r["steps"], "clocks": r["clocks"],
            "prep": prep_line(r["prep_sec"], x.batch.total_q, pk)}
    if extra:
        line["workloads"] = {
            name: {"value": re_["value"], "unit": UNIT, "steps": re_["steps"],
                   "ms_per_step": 1e3 * re_["sec"] / re_["steps"], "stages": stage_lines(xe, re_["stage_sec"], pk),
                   "gpu_launches": re_["launches_per_step"] * re_["steps"], "clocks": re_["clocks"],
                   "config": config_of(xe, args)}
            for name, (xe, re_) in extra.items()}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
