"""FP8 e4m3 decoding and the per-block activation quantiser (oracle side).

The indexer code on the "详解DSA" page quantises q and k with
``act_quant(x, block_size)`` into float8_e4m3fn values plus one fp32 scale per
128-element block (block_size equals the indexer head dim, so one scale per q
head vector and one per key row), stores them in ``k_cache``/``k_scale_cache``
and passes them to the FP8 index kernel.  The page leaves the scale rule open
(``scale_fmt``); the reading taken here is the plain one: scale = amax / 448 in
fp32, value = round-to-nearest-even(x / scale) in e4m3, saturating at 448.

This module is written from the e4m3 format definition (1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits, exponent field 0 = subnormal, code 0x7F /
0xFF = NaN, no infinities) with integer bit manipulation on fp32 words, and is
independent of the generator's table-based encoder.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """e4m3 codes (uint8) -> float64 values."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = m.astype(np.float64) * 2.0 ** -9
    v = sign * np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def _round_shift_rne(x: np.ndarray, shift: np.ndarray) -> np.ndarray:
    """Integer x >> shift with round-to-nearest-even (x >= 0, 1 <= shift <= 62)."""
    shift = shift.astype(np.int64)
    q = x >> shift
    rem = x - (q << shift)
    half = np.int64(1) << (shift - 1)
    up = (rem > half) | ((rem == half) & ((q & 1) == 1))
    return q + up.astype(np.int64)


def encode_e4m3_from_f32(y: np.ndarray) -> np.ndarray:
    """fp32 values -> e4m3 codes, RNE, saturating to +-448, sign of zero kept."""
    bits = np.ascontiguousarray(y, dtype=np.float32).view(np.uint32).astype(np.int64)
    sign = (bits >> 31) & 1
    E = (bits >> 23) & 0xFF
    M = bits & 0x7FFFFF
    e = E - 127                                   # unbiased fp32 exponent
    # normal e4m3 range: e >= -6; keep 3 mantissa bits of 23, RNE on the 20 dropped
    sig = M | (1 << 23)                           # 1.M as a 24-bit integer
    q_norm = _round_shift_rne(sig, np.full(sig.shape, 20))   # 8..16 (16 = carried into exponent)
    e_n = e + (q_norm >> 4)                       # a carry makes q_norm 16 -> exponent + 1
    m_n = np.where(q_norm >= 16, 0, q_norm - 8)
    biased = e_n + 7
    sat = (biased > 15) | ((biased == 15) & (m_n == 7))
    code_norm = np.where(sat, (15 << 3) | 6, (biased << 3) | m_n)
    # subnormal e4m3 range (|y| < 2^-6): value / 2^-9 rounded to an integer 0..8
    # |y| * 2^9 = sig * 2^(E - 150 + 9) for E > 0, or M * 2^(-149 + 9) for E == 0
    sub_sig = np.where(E > 0, sig, M)
    sub_shift = np.where(E > 0, 141 - E, 140)
    sub_shift = np.clip(sub_shift, 1, 62)
    q_sub = np.where(sub_shift >= 62, 0, _round_shift_rne(sub_sig, sub_shift))
    code_sub = np.where(q_sub >= 8, 1 << 3, q_sub)          # 8 * 2^-9 = 2^-6, the smallest normal
    code = np.where(e >= -6, code_norm, code_sub)
    return (code | (sign << 7)).astype(np.uint8)


def act_quant(x: np.ndarray, block: int = 128):
    """Per-``block`` quantisation along the last axis of fp32 (bf16-valued) data.

    Returns (codes uint8, scales float32 with one entry per block, the block
    axis dropped when the last axis holds a single block).
    """
    x = np.asarray(x, dtype=np.float32)
    shp = x.shape
    xb = x.reshape(shp[:-1] + (shp[-1] // block, block))
    amax = np.abs(xb).max(axis=-1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), scale).astype(np.float32)
    y = (xb / scale[..., None]).astype(np.float32)
    codes = encode_e4m3_from_f32(y).reshape(shp)
    if scale.shape[-1] == 1:
        scale = scale[..., 0]
    return codes, scale


def dequant(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """codes * scale in float64 (one scale per last-axis vector)."""
    return decode_e4m3(codes) * np.asarray(scale, dtype=np.float64)[..., None]
