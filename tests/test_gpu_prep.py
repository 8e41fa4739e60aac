"""The upstream preparation kernels against the oracle's per-128 FP8 quantiser.

dsa_quantize_fp8 and dsa_cache_write are called through the C ABI; codes and
scales must equal oracle.fp8.act_quant bit for bit (both sides divide in fp32
with round-to-nearest and round the quotient to e4m3 with ties to even,
saturating at 448), latent rows must arrive unchanged, and no other cache row
may change.
"""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from oracle.fp8 import act_quant

pytestmark = pytest.mark.gpu


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _edge_vectors() -> np.ndarray:
    v = []
    v.append(np.zeros(128))                              # all zero: scale 1, codes 0
    z = np.zeros(128)
    z[::2] = -0.0
    v.append(z)                                          # signed zeros keep their sign
    one = np.zeros(128)
    one[5] = 3.0
    v.append(one)                                        # a single value: x / scale at the 448 edge
    neg = np.zeros(128)
    neg[127] = -1.0e-3
    v.append(neg)
    ties = np.zeros(128)
    ties[0] = 448.0                                      # scale exactly 1
    ties[1:9] = [1.0625, 1.1875, -1.0625, 3 * 2.0 ** -10, 2.0 ** -10, 5 * 2.0 ** -10, 2.0 ** -12, 15 * 2.0 ** -10]
    v.append(ties)                                       # ties to even, normal and subnormal codes
    big = np.full(128, 1.0)
    big[3] = 3.0e38                                      # large finite bf16 magnitudes
    v.append(big)
    small = np.random.default_rng(3).standard_normal(128) * 1.0e-30
    v.append(small)
    return np.stack(v)


def _random_vectors(n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 128))
    x *= np.exp2(rng.integers(-12, 13, size=(n, 1)))     # per-vector magnitudes over many binades
    return x


def _check_quant(x_np: np.ndarray):
    xb = _bf16(x_np)                                     # the bytes both sides see
    codes_ref, scale_ref = act_quant(xb.float().numpy())
    x = xb.cuda()
    n = x.shape[0]
    codes = torch.full((n, 128), 0x5A, dtype=torch.uint8, device="cuda")
    scales = torch.full((n,), -1.0, dtype=torch.float32, device="cuda")
    dsa.quantize_fp8(x, codes, scales)
    torch.cuda.synchronize()
    got_c = codes.cpu().numpy()
    got_s = scales.cpu().numpy()
    assert np.array_equal(got_c, codes_ref), np.argwhere(got_c != codes_ref)[:5]
    assert np.array_equal(got_s.view(np.uint32), np.asarray(scale_ref, np.float32).view(np.uint32))


def test_quantize_edge_vectors():
    _check_quant(_edge_vectors())


@pytest.mark.parametrize("n", [1, 3, 37, 4096 + 5, 148 * 8 * 8 * 4 + 13])
def test_quantize_random_vectors(n):
    # counts that leave a partial unroll group and, for the largest, more than
    # one pass of the grid-stride loop
    _check_quant(_random_vectors(n, seed=n))


def _batch(q_lens, kv_lens, kv_starts, total_keys):
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    cu_q = torch.from_numpy(cu).cuda()
    kv_len = torch.tensor(kv_lens, dtype=torch.int32, device="cuda")
    kv_start = torch.tensor(kv_starts, dtype=torch.int64, device="cuda")
    return dsa.Batch(cu_q, kv_len, kv_start, int(cu[-1]), max(q_lens), max(kv_lens), total_keys)


def test_cache_write_places_new_tokens():
    q_lens, kv_lens, kv_starts, total_keys = [2, 7, 1, 9], [5, 300, 1, 9], [0, 40, 1000, 1100], 1200
    batch = _batch(q_lens, kv_lens, kv_starts, total_keys)
    total_q = sum(q_lens)
    rng = np.random.default_rng(11)
    k_new = _bf16(rng.standard_normal((total_q, 128)) * 0.5)
    lat_new = _bf16(rng.standard_normal((total_q, 576)))
    k_cache = torch.full((total_keys, 128), 0xAB, dtype=torch.uint8, device="cuda")
    k_scale = torch.full((total_keys,), -7.0, dtype=torch.float32, device="cuda")
    lat0 = _bf16(rng.standard_normal((total_keys, 576)))
    lat_cache = lat0.cuda()
    ws = dsa.workspace(dsa.OP_CACHE_WRITE, batch, 0, 0)
    dsa.cache_write(batch, k_new.cuda(), lat_new.cuda(), k_cache, k_scale, lat_cache, ws)
    dsa.check_device_error(ws)

    codes_ref, scale_ref = act_quant(k_new.float().numpy())
    exp_codes = np.full((total_keys, 128), 0xAB, np.uint8)
    exp_scale = np.full(total_keys, -7.0, np.float32)
    exp_lat = lat0.view(torch.int16).numpy().copy()
    r = 0
    for b, (ql, kv, ks) in enumerate(zip(q_lens, kv_lens, kv_starts)):
        for i in range(ql):
            row = ks + kv - ql + i                       # the token's position t = kv - q_len + i
            exp_codes[row] = codes_ref[r]
            exp_scale[row] = scale_ref[r]
            exp_lat[row] = lat_new[r].view(torch.int16).numpy()
            r += 1
    assert np.array_equal(k_cache.cpu().numpy(), exp_codes)
    assert np.array_equal(k_scale.cpu().numpy().view(np.uint32), exp_scale.view(np.uint32))
    assert np.array_equal(lat_cache.cpu().view(torch.int16).numpy(), exp_lat)


def test_cache_write_out_of_range_sequence_is_reported_and_skipped():
    # sequence 1 claims more new tokens than positions (q_len > kv_len): it is
    # skipped with a bounds error; sequence 0 is still written
    q_lens, kv_lens, kv_starts, total_keys = [1, 4], [3, 2], [0, 10], 64
    batch = _batch(q_lens, [3, 4], kv_starts, total_keys)         # host view consistent
    batch.kv_len.copy_(torch.tensor(kv_lens, dtype=torch.int32))  # device kv_len: 2 < q_len 4
    k_new = _bf16(np.ones((5, 128))).cuda()
    lat_new = _bf16(np.ones((5, 576))).cuda()
    k_cache = torch.zeros((total_keys, 128), dtype=torch.uint8, device="cuda")
    k_scale = torch.zeros((total_keys,), dtype=torch.float32, device="cuda")
    lat_cache = torch.zeros((total_keys, 576), dtype=torch.bfloat16, device="cuda")
    ws = dsa.workspace(dsa.OP_CACHE_WRITE, batch, 0, 0)
    dsa.cache_write(batch, k_new, lat_new, k_cache, k_scale, lat_cache, ws)
    with pytest.raises(dsa.DSAError) as e:
        dsa.check_device_error(ws)
    assert e.value.status == 6 and e.value.site == 401 and e.value.info == 1
    # sequence 0 (one token at position 2) is written, sequence 1 is not
    assert k_scale[2].item() == float(np.float32(1.0) / np.float32(448.0))
    assert torch.count_nonzero(k_scale).item() == 1
    assert torch.all(lat_cache[2] == 1.0)
    assert torch.count_nonzero(lat_cache[10:]).item() == 0
