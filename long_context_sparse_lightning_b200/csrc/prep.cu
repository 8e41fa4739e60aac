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

// The indexer's input chain ("详解DSA", indexer code: the first 64 dims of each
// q head vector / key get rotary position embedding, then rotate_activation,
// then act_quant; "DeepSeek V3.2 稀疏注意力": the indexer wants the
// non-interleaved RoPE layout), fused per 128-element vector, one warp each:
//   RoPE   dims i and i + 32 (i < 32) rotate by the position's (cos_i, sin_i):
//          out_i = x_i c - x_{i+32} s, out_{i+32} = x_{i+32} c + x_i s (fp32
//          products and sums, no fused multiply-add), stored as bf16;
//   rotate the normalised Walsh-Hadamard transform over the 128 dims
//          (Sylvester order, butterfly stages h = 1 .. 64 in fp32, then
//          x fp32(128^-0.5)), stored as bf16;
//   act_quant as quant_lane.
// Lane l holds dims 4l .. 4l+3: the RoPE partner of lane l < 8 is lane l + 8,
// the Hadamard partner at stride h >= 4 is lane l ^ (h / 4).
__device__ __forceinline__ uint32_t bf16_bits(float x) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h));
}

__global__ void __launch_bounds__(kWarps * 32)
    indexer_prep_kernel(const uint2* __restrict__ x, int64_t n_vec, int vecs_per_pos, const int32_t* __restrict__ pos,
                        const float* __restrict__ rope_cos, const float* __restrict__ rope_sin, int n_pos,
                        uint32_t* __restrict__ codes, float* __restrict__ scales, uint32_t* err) {
  const uint32_t FULL = 0xffffffffu;
  const int lane = static_cast<int>(threadIdx.x & 31u);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t v = warp; v < n_vec; v += n_warps) {
    const int p = __ldg(&pos[v / vecs_per_pos]);
    if (p < 0 || p >= n_pos) {               // warp-uniform: no table row to read
      if (lane == 0) {
        report_error(err, kDevErrBounds, 501, static_cast<uint32_t>(v));
        scales[v] = 1.f;
      }
      codes[v * 32 + lane] = 0u;
      continue;
    }
    const uint2 raw = __ldcs(x + v * 32 + lane);
    float f[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                  __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
    // ---- RoPE on dims 0..63 (lanes 0..15) ----
    float g[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) g[j] = __shfl_xor_sync(FULL, f[j], 8);
    if (lane < 16) {
      const int i0 = 4 * (lane & 7);
      const float4 c = __ldg(reinterpret_cast<const float4*>(rope_cos + static_cast<int64_t>(p) * 32 + i0));
      const float4 sn = __ldg(reinterpret_cast<const float4*>(rope_sin + static_cast<int64_t>(p) * 32 + i0));
      const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // lane < 8: (x_i, x_{i+32}) = (f, g); lane >= 8: (x_{i+32}, x_i) = (f, g)
        const float r = lane < 8 ? __fsub_rn(__fmul_rn(f[j], cc[j]), __fmul_rn(g[j], ss[j]))
                                 : __fadd_rn(__fmul_rn(f[j], cc[j]), __fmul_rn(g[j], ss[j]));
        f[j] = __uint_as_float(bf16_bits(r) << 16);
      }
    }
    // ---- Walsh-Hadamard: stages 1, 2 inside the lane, 4 .. 64 across lanes ----
    float a0 = __fadd_rn(f[0], f[1]), a1 = __fsub_rn(f[0], f[1]);
    float a2 = __fadd_rn(f[2], f[3]), a3 = __fsub_rn(f[2], f[3]);
    float b[4] = {__fadd_rn(a0, a2), __fadd_rn(a1, a3), __fsub_rn(a0, a2), __fsub_rn(a1, a3)};
#pragma unroll
    for (int m = 1; m <= 16; m <<= 1) {
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float o = __shfl_xor_sync(FULL, b[j], m);
        b[j] = upper ? __fsub_rn(o, b[j]) : __fadd_rn(b[j], o);
      }
    }
    uint2 rot;
    rot.x = bf16_bits(__fmul_rn(b[0], 0.08838834764831845f)) | (bf16_bits(__fmul_rn(b[1], 0.08838834764831845f)) << 16);
    rot.y = bf16_bits(__fmul_rn(b[2], 0.08838834764831845f)) | (bf16_bits(__fmul_rn(b[3], 0.08838834764831845f)) << 16);
    float sc;
    const uint32_t cd = quant_lane(rot, sc);
    codes[v * 32 + lane] = cd;
    if (lane == 0) scales[v] = sc;
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

cudaError_t launch_indexer_prep(const void* x, int64_t n_vec, int vecs_per_pos, const int32_t* pos,
                                const float* rope_cos, const float* rope_sin, int n_pos, void* codes, float* scales,
                                uint32_t* err, cudaStream_t stream) {
  const int64_t need = (n_vec + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int grid = static_cast<int>(need < cap ? need : cap);
  indexer_prep_kernel<<<grid, kWarps * 32, 0, stream>>>(static_cast<const uint2*>(x), n_vec, vecs_per_pos, pos,
                                                        rope_cos, rope_sin, n_pos, static_cast<uint32_t*>(codes),
                                                        scales, err);
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
