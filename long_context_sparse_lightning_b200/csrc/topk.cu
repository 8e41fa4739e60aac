// Per-query top-k over the causal prefix of each score row.
//
// Eq. (2) of "详解DSA": S_t = { s : I[t, s] in Top-k(I[t, :]) } over s <= t; a
// row with at most k positions keeps them all ("详解DSA", prefill analysis).
// "DeepSeek V3.2 稀疏注意力" (top-k as the algorithm/kernel interface) asks for
// a selection kernel rather than a generic sort, with the tie and padding rules
// defined; here: higher score first, ties broken by the lower position (scores
// compare as floats, so -0 and +0 tie), output = the selected positions in
// ascending order, -1 padding.
//
// Selection is one histogram pass in value space, not a digit-by-digit radix
// select: the row's finite range [min, max] is cut into 2048 equal-width bins
// (a monotone map of the value, so bins are ordered like the scores), a
// shared-memory histogram locates the bin b* that holds the k-th largest score,
// every position above b* is selected, and the few positions inside b* (tens
// on indexer score rows) are ranked against each other exactly.  Equal-width
// value bins spread the bulk of a score row over hundreds of bins, where the
// top bits of the float encoding would pile it into a handful and serialise
// the shared-memory atomics.  Rows whose boundary bin holds more than
// kCandCap positions, or that contain a non-finite score, take an exact
// 32-bit radix select instead (11/11/10-bit digits on order-preserving keys).
//
// Rows of up to 32768 positions run in a persistent kernel: each CTA keeps the
// current row in registers (up to 64 scores per thread) while the bulk-copy
// engine streams its next row into shared memory.  Longer rows run one CTA
// per row and re-read the row from global memory (L2) on every pass.
#include <algorithm>
#include <atomic>
#include <cfloat>

#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace dsa {
namespace {

constexpr int kBins = 2048;
constexpr int kCandCap = 512;     // boundary-bin positions ranked pairwise
constexpr int kSegChunks = 16;    // chunks per compaction segment: 16 x 4 flags per thread
constexpr int kMaxK = 2048;       // largest k_sel

template <int BLOCK, int CAPW>
struct TopkShared {
  static constexpr int NW = BLOCK / 32;
  uint32_t hist[kBins];
  float cand_v[kCandCap];
  int32_t cand_p[kCandCap];
  uint8_t cand_sel[kCandCap];
  uint32_t selbits[CAPW > 0 ? CAPW : 1];   // the row's selection bitmap, one word per 32 positions
  int32_t out_s[kMaxK];                     // the row's output, compacted before one coalesced store
  uint32_t tab[kSegChunks * NW];
  float s_red[4][32];
  uint32_t s_warp[32];
  uint32_t s_bstar, s_above, s_cnt, s_ncand, s_total, s_digit;
  alignas(8) uint64_t bar;
};

// Sequence of query row r (binary search over cu_q) and its causal length n.
__device__ __forceinline__ bool row_info(const TopkParams& p, int r, int& n) {
  int lo = 0, hi = p.num_seqs;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(&p.cu_q[mid]) <= r) lo = mid;
    else hi = mid;
  }
  const int q0 = __ldg(&p.cu_q[lo]);
  const int q_len = __ldg(&p.cu_q[lo + 1]) - q0;
  const int kv = __ldg(&p.kv_len[lo]);
  const int i = r - q0;
  const int t = kv - q_len + i;
  if (i < 0 || i >= q_len || t < 0 || kv > p.ld) return false;
  n = t + 1;
  return true;
}

// Selects the top k of one row with n > k positions and writes them to `out`.
// get4(v) returns the float4 of vector v*BLOCK + tid (positions 4 * that ..+3).
// EPT > 0: the row is held in registers, EPT positions per thread, and every
// chunk loop is unrolled; EPT == 0: get4 reads memory, loops stay rolled.
// Calls fn(v) for v in [v0, v1): unrolled over the EPT/4 register chunks when
// EPT > 0, a rolled loop otherwise.
template <int EPT, typename Fn>
__device__ __forceinline__ void for_range(int v0, int v1, Fn&& fn) {
  if constexpr (EPT > 0) {
#pragma unroll
    for (int v = 0; v < EPT / 4; ++v)
      if (v >= v0 && v < v1) fn(v);
  } else {
#pragma unroll 1
    for (int v = v0; v < v1; ++v) fn(v);
  }
}

// Register rows (EPT > 0) hold -inf at positions >= n: no score reaches the
// finite histogram bound there, so only the range pass needs the row length.
__device__ __forceinline__ float4 load_padded(const float4* src, int vec, int n_vec, int n, bool cg) {
  const float NI = __int_as_float(0xff800000);
  if (vec >= n_vec) return make_float4(NI, NI, NI, NI);
  float4 f = cg ? __ldcg(&src[vec]) : src[vec];
  const int p0 = vec * 4;
  if (p0 + 4 > n) {
    if (p0 + 1 > n) f.x = NI;
    if (p0 + 2 > n) f.y = NI;
    if (p0 + 3 > n) f.z = NI;
    f.w = NI;
  }
  return f;
}

// max / min that return NaN when either input is NaN
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float min_nan(float a, float b) {
  float r;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Value-bin selection.  Returns false, having written nothing, when the row
// holds a non-finite score or its boundary bin holds more than kCandCap
// positions; the caller then runs select_radix.
//
// The histogram covers [lo, max] rather than the whole row: lo is the value a
// normal fit of the row (mean and spread) expects about 4k positions to reach
// (upper-tail normal quantile by the rational approximation 26.2.23 of
// Abramowitz & Stegun).  Positions below lo cost no atomic and no ranking.  The
// fit only has to be roughly right: when fewer than k positions reach lo, the
// histogram is rebuilt over the full range.
// Range statistics of chunk v (4 positions from pos0): NaN-propagating max
// and min (so any NaN or inf shows) and, for the sample chunks, the sum and
// sum of squares about x0.  One order of operations for every caller.
__device__ __forceinline__ void range_chunk(const float4 f, int pos0, int n, bool sample, float x0, float& mx,
                                            float& mn, float& s1, float& s2) {
  const float e[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (pos0 + c < n) {
      mx = max_nan(mx, e[c]);
      mn = min_nan(mn, e[c]);
      if (sample) {
        const float d = e[c] - x0;
        s1 += d;
        s2 = fmaf(d, d, s2);
      }
    }
  }
}

// butterfly reductions leave the same value in every lane (fp add commutes)
__device__ __forceinline__ void range_warp_all(float& a, float& b, float& c, float& d) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a = max_nan(a, __shfl_xor_sync(0xffffffffu, a, o));
    b = min_nan(b, __shfl_xor_sync(0xffffffffu, b, o));
    c += __shfl_xor_sync(0xffffffffu, c, o);
    d += __shfl_xor_sync(0xffffffffu, d, o);
  }
}

// The warp's range partials to shared memory, the histogram cleared: what
// the range pass leaves for the block-wide reduction after a barrier.
template <int BLOCK, int CAPW>
__device__ __forceinline__ void range_publish(TopkShared<BLOCK, CAPW>& sh, float mx, float mn, float s1, float s2) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  range_warp_all(mx, mn, s1, s2);
  if (lane == 0) {
    sh.s_red[0][warp] = mx;
    sh.s_red[1][warp] = mn;
    sh.s_red[2][warp] = s1;
    sh.s_red[3][warp] = s2;
  }
  for (int j = tid; j < kBins; j += BLOCK) sh.hist[j] = 0u;
  if (tid == 0) sh.s_ncand = 0u;
}

// published: the caller already ran the range pass over the row (range_chunk
// per chunk in ascending order, then range_publish) and a block barrier.
template <int BLOCK, int EPT, int CAPW, typename Get4>
__device__ __forceinline__ bool select_fast(TopkShared<BLOCK, CAPW>& sh, Get4&& get4, int n, int n_chunks, int k,
                                            float x0, int32_t* __restrict__ out, bool published = false) {
  constexpr int NW = BLOCK / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t FULL = 0xffffffffu;
  auto pos_of = [&](int v, int c) { return (v * BLOCK + tid) * 4 + c; };

  // ---- range; mean and spread about x0 from a sample: the first chunk and
  // the middle one ----
  const int v_mid = n_chunks / 2;
  float mx = -FLT_MAX, mn = FLT_MAX, s1 = 0.f, s2 = 0.f;
  if (!published) {
    for_range<EPT>(0, n_chunks,
                   [&](int v) { range_chunk(get4(v), pos_of(v, 0), n, v == 0 || v == v_mid, x0, mx, mn, s1, s2); });
    range_publish(sh, mx, mn, s1, s2);
    __syncthreads();
  }
  auto warp_all = [&](float& a, float& b, float& c, float& d) { range_warp_all(a, b, c, d); };
  mx = lane < NW ? sh.s_red[0][lane] : -FLT_MAX;
  mn = lane < NW ? sh.s_red[1][lane] : FLT_MAX;
  s1 = lane < NW ? sh.s_red[2][lane] : 0.f;
  s2 = lane < NW ? sh.s_red[3][lane] : 0.f;
  warp_all(mx, mn, s1, s2);   // every warp reduces the same partials in the same order
  if (!(fabsf(mx) <= FLT_MAX && fabsf(mn) <= FLT_MAX)) return false;   // uniform

  float lo = mn;
  {
    const float f = 4.f * static_cast<float>(k) / static_cast<float>(n);
    if (f < 0.5f) {
      auto in_chunk = [&](int v) { return min(max(n - 4 * BLOCK * v, 0), 4 * BLOCK); };
      const int n_sample = in_chunk(0) + (v_mid != 0 ? in_chunk(v_mid) : 0);
      const float inv_n = 1.f / static_cast<float>(n_sample);
      const float mean = s1 * inv_n;
      const float var = fmaxf(s2 * inv_n - mean * mean, 0.f);
      const float t = sqrtf(-2.f * logf(f));
      const float z = t - (2.515517f + t * (0.802853f + t * 0.010328f)) /
                              (1.f + t * (1.432788f + t * (0.189269f + t * 0.001308f)));
      lo = fminf(fmaxf(mn, x0 + mean + z * sqrtf(var)), mx);
    }
  }

  // Bin of a score x >= lo: the integer part of 2^23 + (x - lo) * 2048 / (mx - lo),
  // read from the float's bits and clamped to [0, 2047].  One rounding (fma)
  // of a function increasing in x, so the map is monotone: bins are ordered
  // like the scores.  (The positions inside b* are then ranked exactly, so
  // rounding only moves positions between neighbouring bins.)
  float scale = 0.f, off = 0.f;
  auto bin_of = [&](float x) -> int {
    const int b = static_cast<int>(__float_as_uint(__fmaf_rn(x, scale, off))) - 0x4B000000;
    return min(max(b, 0), kBins - 1);
  };
#pragma unroll 1
  for (int attempt = 0;; ++attempt) {
    scale = static_cast<float>(kBins) / (mx - lo);
    off = 8388608.0f - lo * scale;
    // ---- histogram of the positions at or above lo ----
    for_range<EPT>(0, n_chunks, [&](int v) {
      const float4 f = get4(v);
      const float e[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if ((EPT > 0 || pos_of(v, c) < n) && e[c] >= lo) atomicAdd(&sh.hist[bin_of(e[c])], 1u);
    });
    __syncthreads();
    // ---- bin b* with count(bins above) < k <= count(bins at or above) ----
    constexpr int BPT = kBins / BLOCK;
    uint32_t local[BPT];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      local[j] = sh.hist[kBins - 1 - (tid * BPT + j)];
      sum += local[j];
    }
    uint32_t total;
    uint32_t above = block_excl_scan<BLOCK>(sum, sh.s_warp, total);
    if (total >= static_cast<uint32_t>(k) || attempt > 0) {
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        if (above < static_cast<uint32_t>(k) && above + local[j] >= static_cast<uint32_t>(k)) {
          sh.s_bstar = static_cast<uint32_t>(kBins - 1 - (tid * BPT + j));
          sh.s_above = above;
          sh.s_cnt = local[j];
        }
        above += local[j];
      }
      break;
    }
    // fewer than k positions reach lo: histogram the whole row
    lo = mn;
    for (int j = tid; j < kBins; j += BLOCK) sh.hist[j] = 0u;
    __syncthreads();
  }
  __syncthreads();
  const int bstar = static_cast<int>(sh.s_bstar);
  const uint32_t rem = static_cast<uint32_t>(k) - sh.s_above;
  if (sh.s_cnt > static_cast<uint32_t>(kCandCap)) return false;             // uniform

  // ---- classify: above b* (selected) / inside b* (ranked); collect b* ----
  // masks hold one bit per position of a segment of kSegChunks chunks
  auto classify = [&](int seg0, int seg1, bool collect, uint64_t& sel, uint64_t& inb) {
    sel = 0;
    inb = 0;
    for_range<EPT>(seg0, seg1, [&](int v) {
      const float4 f = get4(v);
      const float e[4] = {f.x, f.y, f.z, f.w};
      uint32_t cs = 0, cb = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int b = ((EPT > 0 || pos_of(v, c) < n) && e[c] >= lo) ? bin_of(e[c]) : -1;
        cs |= static_cast<uint32_t>(b > bstar) << c;
        cb |= static_cast<uint32_t>(b == bstar) << c;
      }
      sel |= static_cast<uint64_t>(cs) << (4 * (v - seg0));
      inb |= static_cast<uint64_t>(cb) << (4 * (v - seg0));
      if (collect && __any_sync(FULL, cb != 0u)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const bool is = (cb >> c) & 1u;
          const uint32_t m = __ballot_sync(FULL, is);
          if (m != 0u) {
            const int leader = __ffs(m) - 1;
            uint32_t base = 0;
            if (lane == leader) base = atomicAdd(&sh.s_ncand, static_cast<uint32_t>(__popc(m)));
            base = __shfl_sync(FULL, base, leader);
            const uint32_t slot = base + __popc(m & lanemask_lt());
            if (is && slot < static_cast<uint32_t>(kCandCap)) {
              sh.cand_v[slot] = e[c];
              sh.cand_p[slot] = pos_of(v, c);
            }
          }
        }
      }
    });
  };
  // Register rows of BLOCK x 32 positions: one 32-bit word of the selection
  // bitmap per thread.  Classify writes the bits of the positions above b*
  // (8 lanes' 4-bit nibbles form one word: no atomics), the ranking adds the
  // chosen b* positions, and thread t then writes the set bits of word t --
  // positions 32t .. 32t+31, already ascending -- at its offset from one
  // block-wide scan.
  if constexpr (EPT > 0 && CAPW == BLOCK) {
    for_range<EPT>(0, n_chunks, [&](int v) {
      const float4 f = get4(v);
      const float e[4] = {f.x, f.y, f.z, f.w};
      uint32_t cs = 0, cb = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int b = e[c] >= lo ? bin_of(e[c]) : -1;
        cs |= static_cast<uint32_t>(b > bstar) << c;
        cb |= static_cast<uint32_t>(b == bstar) << c;
      }
      uint32_t wv = cs << (4 * (lane & 7));
      wv |= __shfl_xor_sync(FULL, wv, 1);
      wv |= __shfl_xor_sync(FULL, wv, 2);
      wv |= __shfl_xor_sync(FULL, wv, 4);
      if ((lane & 7) == 0) sh.selbits[(v * BLOCK + tid) >> 3] = wv;
      if (__any_sync(FULL, cb != 0u)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const bool is = (cb >> c) & 1u;
          const uint32_t m = __ballot_sync(FULL, is);
          if (m != 0u) {
            const int leader = __ffs(m) - 1;
            uint32_t base = 0;
            if (lane == leader) base = atomicAdd(&sh.s_ncand, static_cast<uint32_t>(__popc(m)));
            base = __shfl_sync(FULL, base, leader);
            const uint32_t slot = base + __popc(m & lanemask_lt());
            if (is && slot < static_cast<uint32_t>(kCandCap)) {
              sh.cand_v[slot] = e[c];
              sh.cand_p[slot] = pos_of(v, c);
            }
          }
        }
      }
    });
    __syncthreads();
    const uint32_t ncand = min(sh.s_ncand, static_cast<uint32_t>(kCandCap));
    for (uint32_t i = warp; i < ncand; i += NW) {
      const float x = sh.cand_v[i];
      const int pos = sh.cand_p[i];
      uint32_t rank = 0;
      for (uint32_t j = lane; j < ncand; j += 32) {
        const float y = sh.cand_v[j];
        rank += (y > x) || (y == x && sh.cand_p[j] < pos);
      }
      rank = __reduce_add_sync(FULL, rank);
      if (lane == 0 && rank < rem) atomicOr(&sh.selbits[pos >> 5], 1u << (pos & 31));
    }
    __syncthreads();
    // words of chunks past the row were not written for this row
    uint32_t w = tid < n_chunks * (BLOCK / 8) ? sh.selbits[tid] : 0u;
    uint32_t total;
    uint32_t o = block_excl_scan<BLOCK>(static_cast<uint32_t>(__popc(w)), sh.s_warp, total);
    while (w != 0u) {
      const int bit = __ffs(w) - 1;
      w &= w - 1;
      if (o < static_cast<uint32_t>(k)) out[o] = 32 * tid + bit;
      ++o;
    }
    return true;
  }
  // Rows streamed from memory (register rows returned above): classify and
  // compact segment by segment, the positions' verdicts kept in registers as
  // 4-bit flags.
  const bool one_seg = n_chunks <= kSegChunks;
  uint64_t sel = 0, inb = 0;
  if (one_seg) {
    classify(0, n_chunks, true, sel, inb);
  } else {
    for (int seg0 = 0; seg0 < n_chunks; seg0 += kSegChunks)
      classify(seg0, min(seg0 + kSegChunks, n_chunks), true, sel, inb);
  }
  __syncthreads();
  // ---- rank each b* position (higher score first, then lower position), one
  // warp per position; the first `rem` are selected ----
  const uint32_t ncand = min(sh.s_ncand, static_cast<uint32_t>(kCandCap));
  for (uint32_t i = warp; i < ncand; i += NW) {
    const float x = sh.cand_v[i];
    const int pos = sh.cand_p[i];
    uint32_t rank = 0;
    for (uint32_t j = lane; j < ncand; j += 32) {
      const float y = sh.cand_v[j];
      rank += (y > x) || (y == x && sh.cand_p[j] < pos);
    }
    rank = __reduce_add_sync(FULL, rank);
    if (lane == 0) sh.cand_sel[i] = rank < rem;
  }
  __syncthreads();

  // ---- ordered compaction into shared memory, segment by segment ----
  uint32_t base = 0;
#pragma unroll 1
  for (int seg0 = 0; seg0 < n_chunks; seg0 += kSegChunks) {
    const int seg1 = min(seg0 + kSegChunks, n_chunks);
    if (!one_seg) classify(seg0, seg1, false, sel, inb);
#pragma unroll 1
    while (inb != 0) {               // this thread's b* positions: look up their verdict
      const int bit = __ffsll(static_cast<long long>(inb)) - 1;
      inb &= inb - 1;
      const int pos = ((seg0 + (bit >> 2)) * BLOCK + tid) * 4 + (bit & 3);
      bool chosen = false;
      for (uint32_t j = 0; j < ncand; ++j)
        if (sh.cand_p[j] == pos) chosen = sh.cand_sel[j];
      if (chosen) sel |= uint64_t(1) << bit;
    }
    for_range<EPT>(seg0, seg1, [&](int v) {
      const uint32_t fl = static_cast<uint32_t>(sel >> (4 * (v - seg0))) & 15u;
      const uint32_t tot = __reduce_add_sync(FULL, static_cast<uint32_t>(__popc(fl)));
      if (lane == 0) sh.tab[(v - seg0) * NW + warp] = tot;
    });
    __syncthreads();
    if (warp == 0) {
      constexpr int PER = kSegChunks * NW / 32;
      const int n_ent = (seg1 - seg0) * NW;
      uint32_t loc[PER];
      uint32_t s = 0;
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int e = lane * PER + j;
        loc[j] = e < n_ent ? sh.tab[e] : 0u;
        s += loc[j];
      }
      uint32_t x = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
      }
      uint32_t run = base + x - s;
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int e = lane * PER + j;
        if (e < n_ent) sh.tab[e] = run;
        run += loc[j];
      }
      if (lane == 31) sh.s_total = base + x;
    }
    __syncthreads();
    const uint32_t lt = lanemask_lt();
    for_range<EPT>(seg0, seg1, [&](int v) {
      const uint32_t fl = static_cast<uint32_t>(sel >> (4 * (v - seg0))) & 15u;
      // selected positions of lower lanes in this chunk, then lower components
      uint32_t o = sh.tab[(v - seg0) * NW + warp];
      o += __popc(__ballot_sync(FULL, fl & 1u) & lt) + __popc(__ballot_sync(FULL, fl & 2u) & lt) +
           __popc(__ballot_sync(FULL, fl & 4u) & lt) + __popc(__ballot_sync(FULL, fl & 8u) & lt);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if ((fl >> c) & 1u) {
          if (o < static_cast<uint32_t>(k)) sh.out_s[o] = pos_of(v, c);
          ++o;
        }
      }
    });
    base = sh.s_total;
    __syncthreads();
  }
  for (int j = tid; j < k; j += BLOCK) out[j] = sh.out_s[j];
  return true;
}

// Exact radix select on order-preserving keys (11/11/10-bit digits,
// warp-aggregated histogram updates), for rows select_fast declines: finds the
// threshold key T and how many T-valued positions are needed, then writes the
// selected positions in ascending order.
template <int BLOCK, int CAPW, typename Get4>
__device__ __noinline__ void select_radix(TopkShared<BLOCK, CAPW>& sh, Get4 get4, int n, int n_chunks, int k,
                                          int32_t* __restrict__ out) {
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t FULL = 0xffffffffu;
  auto for_chunks = [&](auto&& fn) { for_range<0>(0, n_chunks, fn); };
  auto pos_of = [&](int v, int c) { return (v * BLOCK + tid) * 4 + c; };
  uint32_t prefix = 0;
  uint32_t remaining = static_cast<uint32_t>(k);
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int width = pass == 2 ? 10 : 11;
    const uint32_t mask = (1u << width) - 1u;
    for (int j = tid; j < kBins; j += BLOCK) sh.hist[j] = 0u;
    __syncthreads();
    const int upper = shift + width;
    for_chunks([&](int v) {
      const float4 f = get4(v);
      const float e[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t key = order_key(e[c]);
        const bool match = pos_of(v, c) < n && (upper >= 32 || (key >> upper) == prefix);
        const uint32_t digit = (key >> shift) & mask;
        const uint32_t active = __ballot_sync(FULL, match);
        if (match) {
          const uint32_t peers = __match_any_sync(active, digit);
          if ((__ffs(peers) - 1) == lane) atomicAdd(&sh.hist[digit], static_cast<uint32_t>(__popc(peers)));
        }
      }
    });
    __syncthreads();
    constexpr int BPT = kBins / BLOCK;
    uint32_t local[BPT];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      local[j] = sh.hist[kBins - 1 - (tid * BPT + j)];
      sum += local[j];
    }
    if (tid == 0) {
      sh.s_digit = 0u;
      sh.s_above = 0u;
    }
    uint32_t total;
    uint32_t above = block_excl_scan<BLOCK>(sum, sh.s_warp, total);
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      if (above < remaining && above + local[j] >= remaining) {
        sh.s_digit = static_cast<uint32_t>(kBins - 1 - (tid * BPT + j));
        sh.s_above = above;
      }
      above += local[j];
    }
    __syncthreads();
    prefix = (prefix << width) | sh.s_digit;
    remaining -= sh.s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;
  // a position's output slot = positions selected before it: (#above T before)
  // + min(#ties before, remaining); the first `remaining` ties are selected
  uint32_t base_gt = 0, base_eq = 0;
  for_chunks([&](int v) {
    const float4 f = get4(v);
    const float e[4] = {f.x, f.y, f.z, f.w};
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (pos_of(v, c) < n) {
        const uint32_t key = order_key(e[c]);
        gt += key > T;
        eq += key == T;
      }
    }
    uint32_t total;
    const uint32_t off = block_excl_scan<BLOCK>((gt << 16) | eq, sh.s_warp, total);
    uint32_t o_gt = base_gt + (off >> 16);
    uint32_t o_eq = base_eq + (off & 0xFFFFu);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int pos = pos_of(v, c);
      if (pos < n) {
        const uint32_t key = order_key(e[c]);
        if (key > T) {
          const uint32_t o = o_gt + min(o_eq, remaining);
          if (o < static_cast<uint32_t>(k)) out[o] = pos;
          ++o_gt;
        } else if (key == T) {
          if (o_eq < remaining && o_gt + o_eq < static_cast<uint32_t>(k)) out[o_gt + o_eq] = pos;
          ++o_eq;
        }
      }
    }
    base_gt += total >> 16;
    base_eq += total & 0xFFFFu;
  });
}

// get4 over a row in global memory (read through L1 / L2).
template <int BLOCK>
struct GlobalRow {
  const float4* row4;
  int n_vec;
  __device__ __forceinline__ float4 operator()(int v) const {
    const int vec = v * BLOCK + static_cast<int>(threadIdx.x);
    return vec < n_vec ? __ldg(row4 + vec) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
};

__device__ __forceinline__ void fill_short_row(int32_t* out, int n, int k, int block) {
  for (int j = threadIdx.x; j < k; j += block) out[j] = j < n ? j : -1;
}

// Global -> shared bulk copy of one row (positions 0 .. n-1, rounded up to a
// whole float4; the row stride is a multiple of 4 floats and >= that).
__device__ __forceinline__ void issue_row_copy(float* buf, const float* row, int n, uint64_t* bar) {
  const uint32_t bytes = static_cast<uint32_t>((n + 3) & ~3) * 4u;
  fence_proxy_async_smem();   // earlier generic reads of the buffer precede the async writes
  mbar_arrive_expect_tx(bar, bytes);
  constexpr uint32_t kPiece = 32768;
  for (uint32_t off = 0; off < bytes; off += kPiece) {
    const uint32_t sz = min(kPiece, bytes - off);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(reinterpret_cast<const uint8_t*>(buf) + off)),
        "l"(reinterpret_cast<const uint8_t*>(row) + off), "r"(sz), "r"(smem_u32(bar))
        : "memory");
  }
}

template <int BLOCK, int EPT>
constexpr size_t reg_smem_bytes() {
  return ((sizeof(TopkShared<BLOCK, BLOCK * EPT / 32>) + 127) / 128) * 128 + static_cast<size_t>(BLOCK) * EPT * sizeof(float);
}

// Persistent kernel for rows of up to BLOCK*EPT positions: the row being
// selected lives in registers, the CTA's next row is bulk-copied into shared
// memory meanwhile.
template <int BLOCK, int EPT, int MIN_CTAS>
__global__ void __launch_bounds__(BLOCK, MIN_CTAS) topk_reg_kernel(const TopkParams p) {
  extern __shared__ __align__(128) uint8_t dyn[];
  constexpr int CAP = BLOCK * EPT;
  using Shared = TopkShared<BLOCK, CAP / 32>;
  auto& sh = *reinterpret_cast<Shared*>(dyn);
  float* buf = reinterpret_cast<float*>(dyn + ((sizeof(Shared) + 127) / 128) * 128);
  const int k = p.k_sel;
  const int tid = threadIdx.x;
  const int G = gridDim.x;

  if (error_pending(p.err)) return;
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto needs_copy = [&](int r, int& n) { return r < p.total_q && row_info(p, r, n) && n > k && n <= CAP; };
  const float* scores = p.scores;
  uint32_t phase = 0;
  bool pending = false;
  {
    int n0;
    if (needs_copy(blockIdx.x, n0)) {
      if (tid == 0) issue_row_copy(buf, scores + static_cast<int64_t>(blockIdx.x) * p.ld, n0, &sh.bar);
      pending = true;
    }
  }
#pragma unroll 1
  for (int r = blockIdx.x; r < p.total_q; r += G) {
    int n = 0;
    int32_t* out = p.idx + static_cast<int64_t>(r) * k;
    if (!row_info(p, r, n) || n > CAP) {
      if (tid == 0) report_error(p.err, kDevErrBounds, 201, r);
      continue;
    }
    if (n <= k) {
      fill_short_row(out, n, k, BLOCK);
      continue;
    }
    if (!pending && tid == 0) issue_row_copy(buf, scores + static_cast<int64_t>(r) * p.ld, n, &sh.bar);
    pending = false;
    const bool ok = mbar_wait(&sh.bar, phase, p.budget);
    phase ^= 1u;
    if (!__syncthreads_and(ok)) {
      if (tid == 0) report_error(p.err, kDevErrTimeout, 202, r);
      break;
    }
    const int n_vec = (n + 3) >> 2;
    const int n_chunks = (n_vec + BLOCK - 1) / BLOCK;
    float x[EPT];
    const float4* b4 = reinterpret_cast<const float4*>(buf);
    const float x0 = buf[0];
    // the row into registers, its range pass on the way (one barrier fewer
    // than a separate pass: the partials go out before the buffer barrier)
    const int v_mid = n_chunks / 2;
    float mx = -FLT_MAX, mn = FLT_MAX, s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int v = 0; v < EPT / 4; ++v) {
      const float4 f = load_padded(b4, v * BLOCK + tid, n_vec, n, false);
      x[4 * v + 0] = f.x;
      x[4 * v + 1] = f.y;
      x[4 * v + 2] = f.z;
      x[4 * v + 3] = f.w;
      if (v < n_chunks) range_chunk(f, (v * BLOCK + tid) * 4, n, v == 0 || v == v_mid, x0, mx, mn, s1, s2);
    }
    range_publish(sh, mx, mn, s1, s2);
    __syncthreads();   // the buffer is free: start the next row's copy
    {
      int nn;
      if (needs_copy(r + G, nn)) {
        if (tid == 0) issue_row_copy(buf, scores + static_cast<int64_t>(r + G) * p.ld, nn, &sh.bar);
        pending = true;
      }
    }
    auto get4 = [&](int v) { return make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]); };
    if (!select_fast<BLOCK, EPT>(sh, get4, n, n_chunks, k, x0, out, true)) {
      const GlobalRow<BLOCK> g{reinterpret_cast<const float4*>(scores + static_cast<int64_t>(r) * p.ld), n_vec};
      select_radix<BLOCK>(sh, g, n, n_chunks, k, out);
    }
  }
}

// One CTA per row for rows longer than the register path holds.
template <int BLOCK>
__global__ void __launch_bounds__(BLOCK) topk_stream_kernel(const TopkParams p) {
  __shared__ TopkShared<BLOCK, 0> sh;
  const int k = p.k_sel;
  const int r = blockIdx.x;
  if (error_pending(p.err)) return;
  int n = 0;
  if (!row_info(p, r, n)) {
    if (threadIdx.x == 0) report_error(p.err, kDevErrBounds, 201, r);
    return;
  }
  int32_t* out = p.idx + static_cast<int64_t>(r) * k;
  if (n <= k) {
    fill_short_row(out, n, k, BLOCK);
    return;
  }
  const float4* row4 = reinterpret_cast<const float4*>(p.scores + static_cast<int64_t>(r) * p.ld);
  const int n_vec = (n + 3) >> 2;
  const int n_chunks = (n_vec + BLOCK - 1) / BLOCK;
  const GlobalRow<BLOCK> g{row4, n_vec};
  if (!select_fast<BLOCK, 0>(sh, g, n, n_chunks, k, __ldg(p.scores + static_cast<int64_t>(r) * p.ld), out))
    select_radix<BLOCK>(sh, g, n, n_chunks, k, out);
}

// Rows longer than the register path holds, in two phases.  Phase 1 selects
// the top k of every seg_len-position segment of a row (one CTA per row and
// segment, the segment in registers) and writes the chosen positions
// (ascending, absolute) and their scores.  A row's candidates are then the
// concatenation of its segments' choices: all segments but the last
// non-empty one are longer than k and give k each, so the valid candidates
// form one prefix, ascending in position.  Phase 2 selects the top k of that
// prefix per row; a lower candidate index is a lower position, so the tie
// rule (equal scores: the lower position wins) carries over, and the chosen
// indices map back to positions.  Each of the row's top k is in the top k of
// its own segment, so the result equals a selection over the whole row.
constexpr int kSegLen = 1024 * 32;        // longest segment: one register row

template <int BLOCK, int EPT>
__global__ void __launch_bounds__(BLOCK, 1) topk_segment_kernel(const TopkParams p) {
  __shared__ TopkShared<BLOCK, BLOCK * EPT / 32> sh;
  static_assert(BLOCK * EPT == kSegLen, "one segment in registers");
  const int seg_len = p.seg_len;           // <= kSegLen, a multiple of 4
  const int k = p.k_sel;
  const int tid = threadIdx.x;
  const int r = blockIdx.x, seg = blockIdx.y;
  if (error_pending(p.err)) return;
  int n = 0;
  if (!row_info(p, r, n)) {
    if (tid == 0 && seg == 0) report_error(p.err, kDevErrBounds, 203, r);
    return;
  }
  const int seg0 = seg * seg_len;
  const int m = min(max(n - seg0, 0), seg_len);
  const int64_t blk = (static_cast<int64_t>(r) * p.n_seg + seg) * k;
  int32_t* out_pos = p.seg_pos + blk;
  float* out_val = p.seg_val + blk;
  const float* row = p.scores + static_cast<int64_t>(r) * p.ld + seg0;
  if (m <= k) {                            // the whole segment (or nothing)
    for (int j = tid; j < k; j += BLOCK) {
      out_pos[j] = j < m ? seg0 + j : -1;
      out_val[j] = j < m ? __ldg(&row[j]) : 0.f;
    }
    return;
  }
  __syncthreads();
  const int n_vec = (m + 3) >> 2;          // the row stride is a multiple of 4 and >= n
  const int n_chunks = (n_vec + BLOCK - 1) / BLOCK;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  float x[EPT];
#pragma unroll
  for (int v = 0; v < EPT / 4; ++v) {
    const float4 f = load_padded(r4, v * BLOCK + tid, n_vec, m, false);
    x[4 * v + 0] = f.x;
    x[4 * v + 1] = f.y;
    x[4 * v + 2] = f.z;
    x[4 * v + 3] = f.w;
  }
  auto get4 = [&](int v) { return make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]); };
  if (!select_fast<BLOCK, EPT>(sh, get4, m, n_chunks, k, __ldg(row), out_pos)) {
    const GlobalRow<BLOCK> g{r4, n_vec};
    select_radix<BLOCK>(sh, g, m, n_chunks, k, out_pos);
  }
  __syncthreads();                         // this CTA's position stores are visible to it
  for (int j = tid; j < k; j += BLOCK) {
    const int q = __ldcg(&out_pos[j]);     // a segment position; m > k, so never -1
    out_val[j] = __ldg(&row[q]);
    out_pos[j] = seg0 + q;
  }
}

template <int BLOCK, int EPT>
__global__ void __launch_bounds__(BLOCK, 1) topk_merge_kernel(const TopkParams p) {
  __shared__ TopkShared<BLOCK, BLOCK * EPT / 32> sh;
  const int k = p.k_sel;
  const int tid = threadIdx.x;
  const int r = blockIdx.x;
  if (error_pending(p.err)) return;
  int n = 0;
  if (!row_info(p, r, n)) return;          // phase 1 reported it
  int32_t* out = p.idx + static_cast<int64_t>(r) * k;
  if (n <= k) {
    fill_short_row(out, n, k, BLOCK);
    return;
  }
  // valid candidates: k per full segment, then the last segment's share
  int m = 0;
  for (int seg = 0; seg < p.n_seg; ++seg) m += min(max(n - seg * p.seg_len, 0), k);
  const int64_t blk = static_cast<int64_t>(r) * p.n_seg * k;
  const int32_t* cpos = p.seg_pos + blk;
  if (m <= k) {                            // one segment's choice is the answer
    for (int j = tid; j < k; j += BLOCK) out[j] = j < m ? __ldcg(&cpos[j]) : -1;
    return;
  }
  __syncthreads();
  const int n_vec = (m + 3) >> 2;          // k is a multiple of 4 or the tail lies inside the block
  const int n_chunks = (n_vec + BLOCK - 1) / BLOCK;
  const float4* c4 = reinterpret_cast<const float4*>(p.seg_val + blk);
  float x[EPT];
#pragma unroll
  for (int v = 0; v < EPT / 4; ++v) {
    const float4 f = load_padded(c4, v * BLOCK + tid, n_vec, m, true);
    x[4 * v + 0] = f.x;
    x[4 * v + 1] = f.y;
    x[4 * v + 2] = f.z;
    x[4 * v + 3] = f.w;
  }
  auto get4 = [&](int v) { return make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]); };
  if (!select_fast<BLOCK, EPT>(sh, get4, m, n_chunks, k, __ldcg(p.seg_val + blk), out)) {
    const GlobalRow<BLOCK> g{c4, n_vec};
    select_radix<BLOCK>(sh, g, m, n_chunks, k, out);
  }
  __syncthreads();
  for (int j = tid; j < k; j += BLOCK) out[j] = __ldcg(&cpos[__ldcg(&out[j])]);   // candidate -> position
}

// ---- key-sharded selection: a shard's candidates, and their merge ----
// "DeepSeek V3.2 稀疏注意力", top-k section: with the keys split across
// devices, each shard selects its local top k and the shards' candidates are
// merged into the global top k.  Each of a row's top k is in the top k of its
// own shard, so the merge equals a selection over the whole row.

// In place: idx (a shard's selected local positions, ascending, -1 padded)
// becomes global positions (+ the sequence's offset) and val their scores
// (-NaN for padding: its order key is below every score, -inf included).
__global__ void __launch_bounds__(256) topk_values_kernel(const TopkParams p, const int32_t* __restrict__ pos_offset,
                                                          float* __restrict__ vals) {
  const int r = blockIdx.x;
  int n = 0;
  if (!row_info(p, r, n)) return;                     // the selection reported it
  int lo = 0, hi = p.num_seqs;                        // the row's sequence
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(&p.cu_q[mid]) <= r) lo = mid;
    else hi = mid;
  }
  const int off = pos_offset != nullptr ? __ldg(&pos_offset[lo]) : 0;
  int32_t* row = p.idx + static_cast<int64_t>(r) * p.k_sel;
  float* v = vals + static_cast<int64_t>(r) * p.k_sel;
  const float* sc = p.scores + static_cast<int64_t>(r) * p.ld;
  for (int j = threadIdx.x; j < p.k_sel; j += blockDim.x) {
    const int q = row[j];
    v[j] = q >= 0 ? __ldg(&sc[q]) : __int_as_float(0xFFFFFFFF);
    row[j] = q >= 0 ? q + off : -1;
  }
}

// One CTA per row: the top k of n_src candidate lists of k entries (global
// positions ascending across the lists, -1 = none).  Candidate index order is
// position order, so the lower-position tie rule carries over.
template <int BLOCK, int EPT>
__global__ void __launch_bounds__(BLOCK, 1) topk_merge_sources_kernel(const int32_t* __restrict__ cand_pos,
                                                                      const float* __restrict__ cand_val, int m,
                                                                      int k, int32_t* __restrict__ idx) {
  __shared__ TopkShared<BLOCK, BLOCK * EPT / 32> sh;
  const int tid = threadIdx.x, r = blockIdx.x;
  const int32_t* cp = cand_pos + static_cast<int64_t>(r) * m;
  const float* cv = cand_val + static_cast<int64_t>(r) * m;
  int32_t* out = idx + static_cast<int64_t>(r) * k;
  // valid candidates, in order (each thread a contiguous odd-length run)
  const int seg = ((m + BLOCK - 1) / BLOCK) | 1;
  const int e0 = min(tid * seg, m), e1 = min(e0 + seg, m);
  uint32_t nv = 0;
  for (int e = e0; e < e1; ++e) nv += __ldg(&cp[e]) >= 0;
  uint32_t total;
  uint32_t o = block_excl_scan<BLOCK>(nv, sh.s_warp, total);
  if (total <= static_cast<uint32_t>(k)) {           // every valid candidate, then -1
    for (int e = e0; e < e1; ++e) {
      const int q = __ldg(&cp[e]);
      if (q >= 0) out[o++] = q;
    }
    for (int j = static_cast<int>(total) + tid; j < k; j += BLOCK) out[j] = -1;
    return;
  }
  __syncthreads();
  const int n_vec = m >> 2;                           // m is a multiple of 4
  const int n_chunks = (n_vec + BLOCK - 1) / BLOCK;
  const float4* v4 = reinterpret_cast<const float4*>(cv);
  const int4* p4 = reinterpret_cast<const int4*>(cp);
  const float NN = __int_as_float(0xFFFFFFFF);        // padding: below every score
  float x[EPT];
#pragma unroll
  for (int v = 0; v < EPT / 4; ++v) {
    const int vec = v * BLOCK + tid;
    float4 f = load_padded(v4, vec, n_vec, m, true);
    if (vec < n_vec) {
      const int4 q = __ldcg(&p4[vec]);
      if (q.x < 0) f.x = NN;
      if (q.y < 0) f.y = NN;
      if (q.z < 0) f.z = NN;
      if (q.w < 0) f.w = NN;
    }
    x[4 * v + 0] = f.x;
    x[4 * v + 1] = f.y;
    x[4 * v + 2] = f.z;
    x[4 * v + 3] = f.w;
  }
  auto get4 = [&](int v) { return make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]); };
  if (!select_fast<BLOCK, EPT>(sh, get4, m, n_chunks, k, x[0], out)) {
    // the register row, read back through a functor that keeps the padding rule
    struct Masked {
      const float4* v4;
      const int4* p4;
      int n_vec;
      __device__ float4 operator()(int v) const {
        const int vec = v * BLOCK + static_cast<int>(threadIdx.x);
        if (vec >= n_vec) return make_float4(0.f, 0.f, 0.f, 0.f);
        float4 f = __ldcg(v4 + vec);
        const int4 q = __ldcg(p4 + vec);
        const float NN2 = __int_as_float(0xFFFFFFFF);
        if (q.x < 0) f.x = NN2;
        if (q.y < 0) f.y = NN2;
        if (q.z < 0) f.z = NN2;
        if (q.w < 0) f.w = NN2;
        return f;
      }
    };
    select_radix<BLOCK>(sh, Masked{v4, p4, n_vec}, m, n_chunks, k, out);
  }
  __syncthreads();
  for (int j = tid; j < k; j += BLOCK) out[j] = __ldcg(&cp[__ldcg(&out[j])]);   // candidate -> position
}

template <int BLOCK, int EPT, int MIN_CTAS>
cudaError_t launch_reg(const TopkParams& p, cudaStream_t stream) {
  constexpr size_t smem = reg_smem_bytes<BLOCK, EPT>();
  cudaError_t e = cudaFuncSetAttribute(topk_reg_kernel<BLOCK, EPT, MIN_CTAS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.total_q, sm_count() * MIN_CTAS);
  topk_reg_kernel<BLOCK, EPT, MIN_CTAS><<<grid, BLOCK, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk_values(const TopkParams& p, const int32_t* pos_offset, float* vals, cudaStream_t stream) {
  if (p.total_q <= 0) return cudaSuccess;
  topk_values_kernel<<<p.total_q, 256, 0, stream>>>(p, pos_offset, vals);
  return cudaGetLastError();
}

cudaError_t launch_topk_merge_sources(int n_rows, int n_src, int k, const int32_t* cand_pos, const float* cand_val,
                                      int32_t* idx, cudaStream_t stream) {
  if (n_rows <= 0) return cudaSuccess;
  const int m = n_src * k;
  if (m > 1024 * 32 || (m & 3) != 0) return cudaErrorInvalidValue;
  topk_merge_sources_kernel<1024, 32><<<n_rows, 1024, 0, stream>>>(cand_pos, cand_val, m, k, idx);
  return cudaGetLastError();
}

int sm_count() {
  // per-device cache; concurrent first calls store the same value
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int v = cached[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cached[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

TopkSegments topk_segments(int max_kv_len, int k_sel, int total_q) {
  TopkSegments t{0, 0};
  // candidate blocks of k floats must keep float4 alignment
  if (k_sel < 1 || (k_sel & 3) != 0 || total_q < 1 || max_kv_len <= kSegLen) return t;
  // as few segments as register rows allow, of equal length.  (Splitting rows
  // that fit one register row, to put more CTAs on few rows, was slower:
  // 64 rows of 16K-32K positions 24 us in one CTA per row, 34 us in halves;
  // nor did 9 segments beat 4 on 16 rows of 128K: 38 us each.)
  const int segs = (max_kv_len + kSegLen - 1) / kSegLen;
  if (static_cast<int64_t>(segs) * k_sel > kSegLen) return t;        // phase 2 holds the candidates
  t.segs = segs;
  t.len = (((max_kv_len + segs - 1) / segs) + 3) & ~3;
  return t;
}

cudaError_t launch_topk(int max_kv_len, const TopkParams& p, cudaStream_t stream) {
  if (p.total_q <= 0) return cudaSuccess;
  if (p.n_seg == 0 && max_kv_len <= 256 * 32) return launch_reg<256, 32, 2>(p, stream);
  if (p.n_seg == 0 && max_kv_len <= 1024 * 32) return launch_reg<1024, 32, 1>(p, stream);
  const int segs = p.n_seg;
  if (segs > 0 && p.seg_pos != nullptr && p.seg_val != nullptr && p.seg_len > 0) {
    topk_segment_kernel<1024, 32><<<dim3(p.total_q, segs), 1024, 0, stream>>>(p);
    topk_merge_kernel<1024, 32><<<p.total_q, 1024, 0, stream>>>(p);
    return cudaGetLastError();
  }
  topk_stream_kernel<1024><<<p.total_q, 1024, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dsa
