"""Sparse MLA parity under magnitude stress (GPU through the C ABI vs the fp64 oracle).

The configs draw q and the latent entries from N(0,1), where raw partial
logits stay around +-20 and a reduced-precision score path would go unseen.
Here the MLA inputs are rescaled (exactly, by powers of two where possible):

* q and latent x8 and x64: raw logits in the thousands to hundreds of
  thousands, a peaky softmax (close to an argmax);
* q alone x8 / x64: a peaky softmax over unit-scale values;
* latent values up to ~60000 (the largest bf16 magnitudes fp16 still holds
  exactly reach 65280);
* tiny latent (x2^-14, most values below fp16's normal range) and tiny q.

Each case runs on the three kernel paths: the bf16-cache kernel with the
selection split over several CTA pairs and merged by log-sum-exp, the same
kernel unsplit, and the fp16-copy kernel a prefill-shaped batch takes.  The
whole forward (indexer -> top-k -> sparse MLA) runs on the split decode batch.
Bounds: the configs' max |d| <= 2e-2 on the output divided by the latent scale
(attention output is linear in the values) or one bf16 step of the reference
element, whichever is larger (a peaky softmax gives outputs as large as the
values, where an fp32 result and the fp64 one can round to neighbouring bf16
numbers, one step apart), and the configs' mean relative error <= 1e-3.
"""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import bf16_bits_to_f32, custom_workload, f32_to_bf16_bits, make_inputs
from oracle import topk as o_topk
from oracle import indexer as o_indexer
from tests.parity import GpuRun, check_mla, check_topk

pytestmark = pytest.mark.gpu

# (name, kv_lens, q_lens, k_sel, n_heads)
SHAPES = {
    "decode_split": ([4000, 3100, 5000, 2600], [1, 1, 1, 1], 2048, 128),
    "decode_unsplit": ([2100 + 37 * i for i in range(40)], [1] * 40, 2048, 128),
    "prefill_fp16_copy": ([2048], [192], 512, 128),
}

# (name, q factor, latent factor): latent factor None = scale to max |c| ~ 60000
SCALES = [
    ("qc_x8", 8.0, 8.0),
    ("qc_x64", 64.0, 64.0),
    ("q_x8", 8.0, 1.0),
    ("q_x64", 64.0, 1.0),
    ("latent_60000", 1.0, None),
    ("latent_tiny", 1.0, 2.0 ** -14),
    ("qc_tiny", 2.0 ** -14, 2.0 ** -14),
]


def _scaled(bits, factor):
    f = bf16_bits_to_f32(bits).astype(np.float64) * factor
    return f32_to_bf16_bits(f.astype(np.float32))


def _inputs(shape, scale):
    kv, q, k_sel, H = SHAPES[shape]
    x = make_inputs(custom_workload(f"stress_{shape}", kv, q, k_sel=k_sel, n_heads=H), seed=17)
    _, qf, cf = scale
    if cf is None:
        cf = 60000.0 / float(np.abs(bf16_bits_to_f32(x.latent)).max())
    x.q_mla = _scaled(x.q_mla, qf)
    x.latent = _scaled(x.latent, cf)
    # every latent value stays a bf16 number fp16 holds exactly or a tiny one
    assert float(np.abs(bf16_bits_to_f32(x.latent)).max()) <= 65280.0
    return x, cf


def _host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _oracle_idx(x):
    rows = list(range(x.batch.total_q))
    idx = np.full((len(rows), x.k_sel), -1, np.int32)
    for i, (_, t, I, _) in enumerate(o_indexer.scores(x, rows)):
        sel, _ = o_topk.select(I, x.k_sel)
        idx[i, : sel.size] = sel
    return idx


@pytest.mark.parametrize("scale", SCALES, ids=[s[0] for s in SCALES])
@pytest.mark.parametrize("shape", list(SHAPES))
def test_sparse_mla_magnitude_stress(shape, scale):
    x, cf = _inputs(shape, scale)
    g = GpuRun(x)
    b = x.batch
    H, k = x.n_heads, x.k_sel
    ws_bytes = dsa.workspace_size(dsa.OP_SPARSE_MLA, g.batch, k, H)
    if shape == "prefill_fp16_copy":
        assert ws_bytes >= 256 + b.total_keys * 576 * 2          # the fp16 copy of the cache is made
    if shape == "decode_split":
        assert ws_bytes > 256                                    # split partials in the workspace
    idx = _oracle_idx(x)
    out, lse = g.mla(torch.from_numpy(idx).cuda(), k)
    rows = list(range(b.total_q))
    check_mla(x, _host(out), _host(lse), idx, rows, value_scale=cf, ulp_floor=True)


@pytest.mark.parametrize("scale", SCALES[:4] + SCALES[5:6], ids=[s[0] for s in SCALES[:4] + SCALES[5:6]])
def test_forward_magnitude_stress_split_decode(scale):
    x, cf = _inputs("decode_split", scale)
    g = GpuRun(x)
    idx, out, lse = g.forward(x.k_sel)
    ih = _host(idx)
    rows = list(range(x.batch.total_q))
    check_topk(x, ih, rows, x.k_sel)
    check_mla(x, _host(out), _host(lse), ih, rows, value_scale=cf, ulp_floor=True)
