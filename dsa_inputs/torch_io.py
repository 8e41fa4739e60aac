"""Move generated inputs into torch tensors (host or device) without touching values."""

from __future__ import annotations

import numpy as np
import torch


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def host_tensors(x, pin: bool = False) -> dict:
    """CPU tensors of every hot-path input of a DSAInputs (bf16 as torch.bfloat16,
    FP8 codes as uint8), optionally in pinned memory."""
    b = x.batch
    t = {
        "q8": torch.from_numpy(np.ascontiguousarray(x.q8)),
        "q_scale": torch.from_numpy(np.ascontiguousarray(x.q_scale)),
        "w": torch.from_numpy(np.ascontiguousarray(x.w)),
        "k8": torch.from_numpy(np.ascontiguousarray(x.k8)),
        "k_scale": torch.from_numpy(np.ascontiguousarray(x.k_scale)),
        "q_mla": _bf16(x.q_mla),
        "latent": _bf16(x.latent),
        "cu_q": torch.from_numpy(b.cu_q.astype(np.int32)),
        "kv_len": torch.from_numpy(b.kv_len.astype(np.int32)),
        "kv_start": torch.from_numpy(b.kv_start.astype(np.int64)),
    }
    if pin:
        t = {k: v.pin_memory() for k, v in t.items()}
    return t


def device_tensors(x, device="cuda") -> dict:
    return {k: v.to(device) for k, v in host_tensors(x).items()}


def batch_sizes(x) -> dict:
    b = x.batch
    return dict(total_q=b.total_q, max_q_per_seq=b.max_q_per_seq, max_kv_len=b.max_kv_len,
                total_keys=b.total_keys)
