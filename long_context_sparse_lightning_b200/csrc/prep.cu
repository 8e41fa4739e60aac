// Upstream preparation of the indexer inputs on sm_100a: the per-128 FP8
// quantiser of q / k vectors, and the write of new tokens' keys (FP8 codes +
// scale) and latent rows into the flat caches.  Both are HBM-bound streams:
// one warp per 128-element vector, lane l holding elements 4l..4l+3, so a
// warp reads 256 contiguous bytes and writes 128.
//
// "详解DSA" (the indexer code): q and k reach the FP8 index kernel through a
// per-block activation quantiser whose block is the indexer head dim (128),
// giving one fp32 scale per head vector of q and per key row; the new tokens'
// quantised keys and their scales are stored in the key cache, the latent rows
// in the MLA cache ("DeepSeek V3.2 稀疏注意力", data-flow section).  The page
// leaves the scale rule open; the reading taken: scale = amax / 448 in fp32
// (an all-zero vector gets scale 1), code = e4m3(x / scale) rounded to
// nearest even and saturated at +-448.  Inputs are finite bf16 values.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kWarps = 8;          // warps per CTA
constexpr int kUnroll = 4;         // vectors in flight per warp

// The lane's four bf16 values (one 8-byte load) -> four e4m3 codes (element
// 4l at the lowest byte) and the vector's scale (identical in every lane).
__device__ __forceinline__ uint32_t quant_lane(uint2 raw, float& scale) {
  const float x0 = __uint_as_float(raw.x << 16), x1 = __uint_as_float(raw.x & 0xFFFF0000u);
  const float x2 = __uint_as_float(raw.y << 16), x3 = __uint_as_float(raw.y & 0xFFFF0000u);
  float amax = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  scale = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);     // IEEE division, round to nearest
  const float y0 = __fdiv_rn(x0, scale), y1 = __fdiv_rn(x1, scale);
  const float y2 = __fdiv_rn(x2, scale), y3 = __fdiv_rn(x3, scale);
  uint16_t lo, hi;
  // e4m3x2: the first source lands in the upper byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(y1), "f"(y0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(y3), "f"(y2));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__global__ void __launch_bounds__(kWarps * 32)
    quantize_fp8_kernel(const uint2* __restrict__ x, int64_t n_vec, uint32_t* __restrict__ codes,
                        float* __restrict__ scales) {
  const int lane = static_cast<int>(threadIdx.x & 31u);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t v0 = warp * kUnroll; v0 < n_vec; v0 += n_warps * kUnroll) {
    uint2 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t v = v0 + u;
      raw[u] = v < n_vec ? __ldcs(x + v * 32 + lane) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t v = v0 + u;
      if (v < n_vec) {                     // warp-uniform
        float s;
        const uint32_t c = quant_lane(raw[u], s);
        __stcs(codes + v * 32 + lane, c);
        if (lane == 0) scales[v] = s;
      }
    }
  }
}

struct CacheWriteParams {
  const int32_t* cu_q;
  const int32_t* kv_len;
  const int64_t* kv_start;
  PageTable pt;
  const uint2* k;          // bf16 [total_q, 128]
  const uint4* latent;     // bf16 [total_q, 576]
  uint32_t* k_cache;       // e4m3 [total_keys, 128]
  float* k_scale;          // [total_keys]
  uint4* latent_cache;     // bf16 [total_keys, 576]
  int64_t total_keys;
  int32_t total_q;
  uint32_t* err;
};

// grid (ceil(max_q_per_seq / kWarps), num_seqs): one warp per new token
__global__ void __launch_bounds__(kWarps * 32) cache_write_kernel(const CacheWriteParams p) {
  const int lane = static_cast<int>(threadIdx.x & 31u);
  const int b = blockIdx.y;
  const int tok = static_cast<int>(blockIdx.x) * kWarps + static_cast<int>(threadIdx.x >> 5);
  const int q0 = __ldg(&p.cu_q[b]);
  const int q_len = __ldg(&p.cu_q[b + 1]) - q0;
  if (tok >= q_len) return;
  const int kv = __ldg(&p.kv_len[b]);
  const int64_t ks = seq_start(p.pt, p.kv_start, b);
  if (q0 < 0 || q0 + q_len > p.total_q || q_len > kv || !seq_rows_ok(p.pt, ks, kv, p.total_keys)) {
    if (lane == 0) report_error(p.err, kDevErrBounds, 401, b);
    return;
  }
  const int64_t src = q0 + tok;
  const int64_t dst = cache_row(p.pt, b, ks, kv - q_len + tok);   // the token's position t = kv - q_len + tok
  if (dst < 0) {                                                  // a page id outside the pool
    if (lane == 0) report_error(p.err, kDevErrBounds, 402, b);
    return;
  }
  float s;
  const uint32_t c = quant_lane(__ldg(p.k + src * 32 + lane), s);
  p.k_cache[dst * 32 + lane] = c;
  if (lane == 0) p.k_scale[dst] = s;
  // 1152-byte latent row: 72 16-byte units
  for (int u = lane; u < 72; u += 32) p.latent_cache[dst * 72 + u] = __ldg(p.latent + src * 72 + u);
}

}  // namespace

cudaError_t launch_quantize_fp8(const void* x, int64_t n_vec, void* codes, float* scales, cudaStream_t stream) {
  const int64_t need = (n_vec + kWarps * kUnroll - 1) / (kWarps * kUnroll);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;     // 8 CTAs (64 warps) per SM, then grid-stride
  const int grid = static_cast<int>(need < cap ? need : cap);
  quantize_fp8_kernel<<<grid, kWarps * 32, 0, stream>>>(static_cast<const uint2*>(x), n_vec,
                                                        static_cast<uint32_t*>(codes), scales);
  return cudaGetLastError();
}

cudaError_t launch_cache_write(int num_seqs, int max_q_per_seq, int total_q, int64_t total_keys,
                               const int32_t* cu_q, const int32_t* kv_len, const int64_t* kv_start,
                               const PageTable& pt, const void* k, const void* latent, void* k_cache, float* k_scale,
                               void* latent_cache, uint32_t* err, cudaStream_t stream) {
  CacheWriteParams p;
  p.cu_q = cu_q;
  p.kv_len = kv_len;
  p.kv_start = kv_start;
  p.pt = pt;
  p.k = static_cast<const uint2*>(k);
  p.latent = static_cast<const uint4*>(latent);
  p.k_cache = static_cast<uint32_t*>(k_cache);
  p.k_scale = k_scale;
  p.latent_cache = static_cast<uint4*>(latent_cache);
  p.total_keys = total_keys;
  p.total_q = total_q;
  p.err = err;
  const dim3 grid((max_q_per_seq + kWarps - 1) / kWarps, num_seqs);
  cache_write_kernel<<<grid, kWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dsa
