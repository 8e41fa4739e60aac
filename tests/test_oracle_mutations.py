"""Planted mistakes in the oracle arithmetic must be caught by its pins.

Each mutant is a plausible slip (a dropped ReLU, a dropped weight, a wrong sign,
a transposed operand, a missing max-subtraction guard replaced by a wrong
scale, a value slice taken from the wrong end).  The same reference routes the
real pins use (brute-force loops, torch SDPA) must reject every one of them.
"""

import numpy as np
import torch

from oracle import brute, fp8

SM = 1.0 / np.sqrt(192.0)


def _fp8(rng, shape):
    return fp8.act_quant(rng.standard_normal(shape).astype(np.float32))


def _scores_variants(q8, qs, w, k8, ks):
    q = fp8.dequant(q8, qs)
    k = fp8.dequant(k8, ks)
    d = q @ k.T
    wc = w.astype(np.float64)[:, None]
    return {
        "ok": (wc * np.maximum(d, 0)).sum(0),
        "no_relu": (wc * d).sum(0),
        "no_weight": np.maximum(d, 0).sum(0),
        "relu_after_sum": np.maximum((wc * d).sum(0), 0),
        "abs_instead_of_relu": (wc * np.abs(d)).sum(0),
        "scale_dropped": (wc * np.maximum(fp8.decode_e4m3(q8) @ k.T, 0)).sum(0),
    }


def test_indexer_mutants_fail_brute_force():
    rng = np.random.default_rng(30)
    q8, qs = _fp8(rng, (64, 128))
    k8, ks = _fp8(rng, (6, 128))
    w = (rng.standard_normal(64) * 0.125).astype(np.float32)
    ref = np.array([brute.index_score(fp8.dequant(q8, qs).tolist(), w.tolist(),
                                      fp8.dequant(k8, ks)[s].tolist()) for s in range(6)])
    variants = _scores_variants(q8, qs, w, k8, ks)
    assert np.allclose(variants.pop("ok"), ref, rtol=1e-12, atol=1e-12)
    for name, v in variants.items():
        assert not np.allclose(v, ref, rtol=1e-6, atol=1e-9), name


def _attn_variants(q, lat, sel):
    c = lat[sel]
    logits = SM * q @ c.T
    p = np.exp(logits - logits.max(1, keepdims=True))
    out = {
        "ok": (p / p.sum(1, keepdims=True)) @ c[:, :512],
        "value_from_tail": (p / p.sum(1, keepdims=True)) @ c[:, 64:],
        "no_scale": None,
        "unnormalised": p @ c[:, :512],
        "rope_dropped": None,
    }
    l2 = q @ c.T
    p2 = np.exp(l2 - l2.max(1, keepdims=True))
    out["no_scale"] = (p2 / p2.sum(1, keepdims=True)) @ c[:, :512]
    l3 = SM * q[:, :512] @ c[:, :512].T
    p3 = np.exp(l3 - l3.max(1, keepdims=True))
    out["rope_dropped"] = (p3 / p3.sum(1, keepdims=True)) @ c[:, :512]
    return out


def test_attention_mutants_fail_sdpa():
    rng = np.random.default_rng(31)
    lat = rng.standard_normal((20, 576))
    q = rng.standard_normal((4, 576))
    sel = np.arange(20)
    Q = torch.from_numpy(q)[None, :, None, :]
    K = torch.from_numpy(lat)[None, None].expand(1, 4, 20, 576)
    V = torch.from_numpy(lat[:, :512])[None, None].expand(1, 4, 20, 512)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=SM)[0, :, 0].numpy()
    variants = _attn_variants(q, lat, sel)
    assert np.allclose(variants.pop("ok"), ref, rtol=1e-12, atol=1e-13)
    for name, v in variants.items():
        assert not np.allclose(v, ref, rtol=1e-4, atol=1e-6), name
