// Per-query top-k over the causal prefix of each score row: radix select on
// order-preserving uint32 keys of the fp32 scores, then an ordered compaction.
//
// Eq. (2) of "详解DSA": S_t = { s : I[t, s] in Top-k(I[t, :]) } over s <= t; a
// row with at most k positions keeps them all ("详解DSA", prefill analysis).
// "DeepSeek V3.2 稀疏注意力" (top-k as the algorithm/kernel interface) asks for
// a selection kernel rather than a generic sort, with the tie and padding rules
// defined; here: higher score first, ties broken by the lower position, output
// = the selected set in ascending position order within each of the two
// groups (strictly above the threshold, then threshold ties), -1 padding.
//
// One CTA per query row.  Rows up to BLOCK*32 positions keep their keys in
// registers (32 per thread, loaded once with 16-byte loads); longer rows are
// re-streamed from global memory (L2) on every pass.  Three histogram passes
// over 11/11/10-bit digits (2048 shared-memory bins, warp-aggregated atomics)
// locate the exact 32-bit threshold key T and how many of the T-valued
// positions are needed; a final pass writes the positions in index order using
// block-wide prefix sums.
#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kEPT = 32;             // keys per thread in the register path
constexpr int kBins = 2048;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the block, in thread order; also returns the total.
template <int BLOCK>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp, uint32_t& total) {
  constexpr int NW = BLOCK / 32;
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

template <int BLOCK, bool IN_REGS>
__global__ void __launch_bounds__(BLOCK) topk_kernel(const TopkParams p) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_digit, s_above;
  const int k_out = p.k_sel;

  if (error_pending(p.err)) return;
  const int b = blockIdx.y;
  const int i = blockIdx.x;
  const int q0 = __ldg(&p.cu_q[b]);
  const int q_len = __ldg(&p.cu_q[b + 1]) - q0;
  if (i >= q_len) return;
  const int kv = __ldg(&p.kv_len[b]);
  const int r = q0 + i;
  const int t = kv - q_len + i;
  const int k = p.k_sel;
  int32_t* out = p.idx + static_cast<int64_t>(r) * k;
  if (t < 0 || kv > p.ld) {
    if (threadIdx.x == 0) report_error(p.err, kDevErrBounds, 201, r);
    return;
  }
  const int n = t + 1;
  if (n <= k) {
    for (int j = threadIdx.x; j < k; j += BLOCK) out[j] = j < n ? j : -1;
    return;
  }
  const float* row = p.scores + static_cast<int64_t>(r) * p.ld;
  const int tid = threadIdx.x;
  const int n_vec = (n + 3) >> 2;                         // float4 vectors covering the row
  const int n_chunks = (n_vec + BLOCK - 1) / BLOCK;       // vectors per thread (register path: <= kEPT/4)

  uint32_t keys[IN_REGS ? kEPT : 1];
  if constexpr (IN_REGS) {
#pragma unroll
    for (int v = 0; v < kEPT / 4; ++v) {
      const int vec = v * BLOCK + tid;
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (vec < n_vec) f = __ldg(reinterpret_cast<const float4*>(row) + vec);
      keys[4 * v + 0] = order_key(f.x);
      keys[4 * v + 1] = order_key(f.y);
      keys[4 * v + 2] = order_key(f.z);
      keys[4 * v + 3] = order_key(f.w);
    }
  }
  // key of component c of this thread's vector in chunk v (position (v*BLOCK+tid)*4+c)
  auto load4 = [&](int v, uint32_t (&k4)[4]) {
    if constexpr (IN_REGS) {
#pragma unroll
      for (int c = 0; c < 4; ++c) k4[c] = keys[4 * v + c];
    } else {
      const int vec = v * BLOCK + tid;
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (vec < n_vec) f = __ldg(reinterpret_cast<const float4*>(row) + vec);
      k4[0] = order_key(f.x);
      k4[1] = order_key(f.y);
      k4[2] = order_key(f.z);
      k4[3] = order_key(f.w);
    }
  };

  // visit this thread's vectors in position order (unrolled when keys live in registers)
  auto for_chunks = [&](auto&& fn) {
    if constexpr (IN_REGS) {
#pragma unroll
      for (int v = 0; v < kEPT / 4; ++v)
        if (v < n_chunks) fn(v);
    } else {
#pragma unroll 1
      for (int v = 0; v < n_chunks; ++v) fn(v);
    }
  };

  // ---- radix select: 11 + 11 + 10 bits from the top ----
  uint32_t prefix = 0;
  uint32_t remaining = static_cast<uint32_t>(k);
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int width = pass == 2 ? 10 : 11;
    const uint32_t mask = (1u << width) - 1u;
    for (int j = tid; j < kBins; j += BLOCK) hist[j] = 0u;
    __syncthreads();
    const int upper = shift + width;   // bits above the current digit must equal prefix
    for_chunks([&](int v) {
      uint32_t k4[4];
      load4(v, k4);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int pos = (v * BLOCK + tid) * 4 + c;
        const bool match = pos < n && (upper >= 32 || (k4[c] >> upper) == prefix);
        const uint32_t digit = (k4[c] >> shift) & mask;
        const uint32_t active = __ballot_sync(0xffffffffu, match);
        if (match) {
          const uint32_t peers = __match_any_sync(active, digit);
          if ((__ffs(peers) - 1) == static_cast<int>(threadIdx.x & 31)) atomicAdd(&hist[digit], __popc(peers));
        }
      }
    });
    __syncthreads();
    // find the digit d with count(> d) < remaining <= count(>= d), scanning from the top bin
    constexpr int BPT = kBins / BLOCK;        // bins per thread (>= 2)
    uint32_t local[BPT];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      local[j] = hist[kBins - 1 - (tid * BPT + j)];
      sum += local[j];
    }
    if (tid == 0) {
      s_digit = 0u;
      s_above = 0u;
    }
    uint32_t total;
    uint32_t above = block_excl_scan<BLOCK>(sum, s_warp, total);
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      if (above < remaining && above + local[j] >= remaining) {
        s_digit = static_cast<uint32_t>(kBins - 1 - (tid * BPT + j));
        s_above = above;
      }
      above += local[j];
    }
    __syncthreads();
    prefix = (prefix << width) | s_digit;
    remaining -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;                 // exact threshold key
  const uint32_t n_gt = static_cast<uint32_t>(k) - remaining;   // positions strictly above T

  // ---- ordered compaction ----
  uint32_t base_gt = 0, base_eq = 0;
  for_chunks([&](int v) {
    uint32_t k4[4];
    load4(v, k4);
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int pos = (v * BLOCK + tid) * 4 + c;
      if (pos < n) {
        gt += k4[c] > T;
        eq += k4[c] == T;
      }
    }
    uint32_t total;
    const uint32_t off = block_excl_scan<BLOCK>((gt << 16) | eq, s_warp, total);
    uint32_t o_gt = base_gt + (off >> 16);
    uint32_t o_eq = base_eq + (off & 0xFFFFu);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int pos = (v * BLOCK + tid) * 4 + c;
      if (pos < n) {
        if (k4[c] > T) {
          if (o_gt < static_cast<uint32_t>(k_out)) out[o_gt] = pos;
          ++o_gt;
        } else if (k4[c] == T) {
          if (o_eq < remaining && n_gt + o_eq < static_cast<uint32_t>(k_out)) out[n_gt + o_eq] = pos;
          ++o_eq;
        }
      }
    }
    base_gt += total >> 16;
    base_eq += total & 0xFFFFu;
  });
}

template <int BLOCK, bool IN_REGS>
cudaError_t launch_cfg(dim3 grid, const TopkParams& p, cudaStream_t stream) {
  topk_kernel<BLOCK, IN_REGS><<<grid, BLOCK, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk(int max_kv_len, dim3 grid, const TopkParams& p, cudaStream_t stream) {
  if (max_kv_len <= 256 * kEPT) return launch_cfg<256, true>(grid, p, stream);
  if (max_kv_len <= 1024 * kEPT) return launch_cfg<1024, true>(grid, p, stream);
  return launch_cfg<1024, false>(grid, p, stream);
}

}  // namespace dsa
