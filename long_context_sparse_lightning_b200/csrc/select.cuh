// Device helpers of the top-k selections (the standalone top-k kernels and
// the fused decode indexer + top-k): the order-preserving key of a score,
// lane masks and a block-wide exclusive scan.
#pragma once

#include <stdint.h>

namespace dsa {

// Order-preserving unsigned key of an fp32 score: a > b as floats <=> key(a) >
// key(b); -0 and +0 get the same key, as they compare equal.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Exclusive prefix sum over the block (BLOCK threads, a multiple of 32, at
// most 1024), in thread order; also returns the total.  Every thread calls it.
template <int BLOCK>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp, uint32_t& total) {
  constexpr int NW = BLOCK / 32;
  static_assert(BLOCK % 32 == 0 && NW <= 32, "whole warps, at most 32");
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < NW ? s_warp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NW) s_warp[lane] = w;
  }
  __syncthreads();
  const uint32_t before = wid > 0 ? s_warp[wid - 1] : 0u;
  total = s_warp[NW - 1];
  __syncthreads();
  return before + x - v;
}

}  // namespace dsa
