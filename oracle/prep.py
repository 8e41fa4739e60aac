"""The indexer's input chain before the FP8 quantiser (oracle side; test
infrastructure only).

"详解DSA", indexer code: each 128-dim q head vector and each key is split into
its first rope_head_dim = 64 dims (q_pe / k_pe) and the rest; the 64 pe dims
get rotary position embedding; the vector is then passed through
rotate_activation and act_quant.  "DeepSeek V3.2 稀疏注意力" (position-encoding
correctness boundary) adds that the indexer expects the non-interleaved RoPE
layout.  Readings taken (the pages print neither function):

* non-interleaved RoPE on the 64 pe dims: dims i and i + 32 (i < 32) rotate
  together by the angle of frequency i, whose cosine and sine come from the
  caller's table row of the token's position (the pages fix no base);
      out[i]      = x[i] * cos_i - x[i + 32] * sin_i
      out[i + 32] = x[i + 32] * cos_i + x[i] * sin_i
  each product rounded to fp32, then the sum / difference (no fused
  multiply-add), the result stored as bf16 (the activation type);
* rotate_activation = the normalised Walsh-Hadamard transform over the 128
  dims, y = H_128 x / sqrt(128) with H_128 the Sylvester-ordered Hadamard
  matrix ([[H, H], [H, -H]]), computed in fp32 by the butterfly stages
  h = 1, 2, 4, ..., 64 (pair (d, d + h): sum to d, difference to d + h), then
  scaled by fp32(128 ** -0.5) and stored as bf16;
* act_quant as in ``oracle.fp8``.

Every step is the arithmetic named above in float32, in the order named, so
the FP8 codes it gives are the ones a kernel with the same steps must give.
"""

from __future__ import annotations

import numpy as np

from . import fp8

HEAD_DIM = 128
ROPE_DIM = 64
HALF = ROPE_DIM // 2


def to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest-even bf16 value, returned as fp32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32)


def rope_non_interleaved(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """x [n, 128] fp32 (bf16 values), cos / sin [n, 32] fp32 rows of each
    vector's position -> [n, 128] with the 64 pe dims rotated, as bf16 values."""
    x = np.asarray(x, dtype=np.float32)
    out = x.copy()
    a = x[:, :HALF]
    b = x[:, HALF:ROPE_DIM]
    c = np.asarray(cos, dtype=np.float32)
    s = np.asarray(sin, dtype=np.float32)
    out[:, :HALF] = (a * c).astype(np.float32) - (b * s).astype(np.float32)
    out[:, HALF:ROPE_DIM] = (b * c).astype(np.float32) + (a * s).astype(np.float32)
    return to_bf16(out)


def hadamard_f32(x: np.ndarray) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform of the last axis (length 128) by
    butterfly stages h = 1, 2, ..., 64 in fp32."""
    y = np.array(x, dtype=np.float32, copy=True)
    n = y.shape[-1]
    h = 1
    while h < n:
        v = y.reshape(y.shape[:-1] + (n // (2 * h), 2, h))
        lo = v[..., 0, :].copy()
        hi = v[..., 1, :].copy()
        v[..., 0, :] = lo + hi
        v[..., 1, :] = lo - hi
        y = v.reshape(y.shape)
        h *= 2
    return y


def rotate_activation(x: np.ndarray) -> np.ndarray:
    """Normalised Walsh-Hadamard transform of bf16-valued [n, 128] data, as bf16 values."""
    return to_bf16(hadamard_f32(x) * np.float32(HEAD_DIM ** -0.5))


def indexer_inputs(x: np.ndarray, cos: np.ndarray, sin: np.ndarray):
    """The whole chain: RoPE on the pe dims -> rotate_activation -> act_quant.
    x [n, 128] bf16 values (fp32), cos / sin [n, 32] -> (codes [n, 128] uint8, scales [n])."""
    return fp8.act_quant(rotate_activation(rope_non_interleaved(x, cos, sin)))
