// Lightning-Indexer scores on sm_100a: a tcgen05 FP8 contraction fed by TMA,
// with ReLU, the w-weighted head sum and both FP8 scales fused into the
// epilogue, so no [t, s, head] tensor ever exists.
//
//   I[t, s] = k_scale[s] * sum_j (w[t, j] * q_scale[t, j]) * ReLU(q8[t, j] . k8[s])
//
// which equals Eq. (1) of "详解DSA" on the dequantised q and k because the
// scales are positive and ReLU is positively homogeneous ("详解DSA", prefill
// analysis: the q scale multiplies w before the head sum, the k scale
// multiplies the summed result).
//
// Tile mapping (one CTA = TOK query tokens of one sequence x a range of
// 128-key tiles):
//   MMA  M = 128 keys (TMEM lanes), N = tokens x 64 heads (TMEM columns),
//        K = 128 FP8 dims = 4 x kind::f8f6f4 K32 instructions;
//        A = k tile [128 x 128 B] and B = q tile [N x 128 B], both K-major,
//        128-byte swizzled exactly as TMA writes them.
//   Each epilogue thread owns one key (one TMEM lane) and reads that key's 64
//   head values of a token from its own TMEM columns, so the head sum needs no
//   cross-thread traffic; a warp stores 32 consecutive scores (128 B).
//   Four accumulators in TMEM (2 tokens x 64 heads each) rotate between the
//   MMA warp and four epilogue warpgroups (group g drains buffer g): four
//   epilogue warps per SM sub-partition keep the issue slots busy while each
//   waits on its TMEM loads and FMA chains.
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (+ TMEM owner),
// warps 2..17 = epilogue (four warpgroups).
#include <atomic>

#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace dsa {
namespace {

constexpr int kEpiWarps = 16;
constexpr int kAccBufs = 4;                  // TMEM accumulators, one per epilogue warpgroup
constexpr int kThreads = 32 * (2 + kEpiWarps);

template <int TOK>
struct IdxCfg {
  static constexpr int GTOK = TOK >= 2 ? 2 : 1;      // tokens per accumulator group
  static constexpr int NG = TOK / GTOK;               // accumulator groups per key tile
  static constexpr int N = GTOK * 64;                 // MMA N
  static constexpr int STAGES = TOK >= 4 ? 6 : 8;
  static constexpr int TMEM_COLS = kAccBufs * N;      // 256 or 512 (powers of two)
  static constexpr int BOXQ = TOK * 64 < 256 ? TOK * 64 : 256;   // q rows per TMA box
  static constexpr int Q_BYTES = TOK * 64 * 128;
  static constexpr int K_BYTES = 128 * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_W = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_BAR = OFF_W + TOK * 64 * 4;
  static constexpr int NUM_BARS = 2 * STAGES + 1 + 2 * kAccBufs + 1;   // + the MMA warp's drain barrier
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_PAGE = OFF_MISC + 16;      // paged caches: pool row of each 64-key half tile
  static constexpr int SMEM = OFF_PAGE + 1024;        // + slack for 1024-byte alignment (+ 8 B per tile when paged)
  static_assert(OFF_K % 1024 == 0 && K_BYTES % 1024 == 0, "swizzle-128 tiles need 1024-byte alignment");
};

// Two fp32 values as one 64-bit register pair (low half first) and a packed
// fma: each lane computes fma.rn.f32 of its pair of elements.
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack2(unsigned long long v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return make_float2(lo, hi);
}
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Paged caches: the pool row of every 64-key half of this CTA's key tiles
// (positions past the sequence, or a page id outside the pool, get
// total_keys: a TMA box there reads zeros and no key scale is loaded).
__device__ __forceinline__ void stage_half_tile_rows(const PageTable& pt, int b, int kv, int tile_begin, int n_tiles,
                                                     int64_t total_keys, int32_t* sPage, uint32_t* err) {
  for (int i = threadIdx.x; i < 2 * n_tiles; i += blockDim.x) {
    const int s = tile_begin * 128 + i * 64;
    int64_t row = total_keys;
    if (s < kv) {
      row = cache_row(pt, b, 0, s);
      if (row < 0) {
        report_error(err, kDevErrBounds, 103, b);
        row = total_keys;
      }
    }
    sPage[i] = static_cast<int32_t>(row);
  }
}

// One 128-key tile of the key cache into a stage: one 128-row box (flat), or
// two 64-row boxes from their pages -- stacked, they form the same 128-byte
// swizzled layout (the swizzle repeats every 8 rows).
__device__ __forceinline__ void load_k_tile(uint8_t* dst, const CUtensorMap* tmap, uint64_t* bar, bool paged,
                                            const int32_t* sPage, int it, int64_t flat_row) {
  if (paged) {
    tma_load_2d(dst, tmap, bar, 0, sPage[2 * it]);
    tma_load_2d(dst + 8192, tmap, bar, 0, sPage[2 * it + 1]);
  } else {
    tma_load_2d(dst, tmap, bar, 0, static_cast<int32_t>(flat_row));
  }
}

// Scale of the key at position `flat_row - kstart` (flat) or at offset
// key_in_tile of local tile `it` (paged).
__device__ __forceinline__ float scale_of_key(const float* k_scale, bool paged, const int32_t* sPage, int it,
                                              int key_in_tile, int64_t flat_row, int64_t total_keys) {
  if (!paged) return __ldg(&k_scale[flat_row]);
  const int64_t base = sPage[2 * it + (key_in_tile >> 6)];
  return base < total_keys ? __ldg(&k_scale[base + (key_in_tile & 63)]) : 0.f;
}

template <int TOK>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const IndexerParams p) {
  using C = IdxCfg<TOK>;
  extern __shared__ uint8_t smem_raw[];

  // ---- work unit: sequence b, query block, key-tile chunk ----
  if (error_pending(p.err)) return;
  const int b = blockIdx.z;
  const int qblock = p.num_qblocks - 1 - static_cast<int>(blockIdx.y);   // long causal rows first
  const int q0 = __ldg(&p.cu_q[b]);
  const int q_len = __ldg(&p.cu_q[b + 1]) - q0;
  const int kv = __ldg(&p.kv_len[b]);
  const int first = qblock * TOK;
  if (first >= q_len) return;
  const int64_t kstart = seq_start(p.pt, p.kv_start, b);
  if (q_len > kv || kv > p.ld || !seq_rows_ok(p.pt, kstart, kv, p.total_keys)) {
    if (threadIdx.x == 0) report_error(p.err, kDevErrBounds, 101, b);
    return;
  }
  const int ntok = min(TOK, q_len - first);
  const int t_first = kv - q_len + first;
  const int t_last = t_first + ntok - 1;
  const int tiles_total = (t_last + 1 + 127) / 128;
  const int tile_begin = static_cast<int>(blockIdx.x) * p.tiles_per_chunk;
  if (tile_begin >= tiles_total) return;
  const bool paged = p.pt.table != nullptr;
  const int n_tiles = min(tile_begin + p.tiles_per_chunk, tiles_total) - tile_begin;
  const int row0 = q0 + first;

  // ---- shared memory carve-up (1024-byte aligned base) ----
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = sm + C::OFF_Q;
  uint8_t* sK = sm + C::OFF_K;
  float* sW = reinterpret_cast<float*>(sm + C::OFF_W);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* q_full = bars + 2 * C::STAGES;
  uint64_t* acc_full = q_full + 1;               // [kAccBufs]
  uint64_t* acc_empty = q_full + 1 + kAccBufs;    // [kAccBufs]
  uint64_t* mma_done = acc_empty + kAccBufs;       // every MMA of this CTA has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  int32_t* sPage = reinterpret_cast<int32_t*>(sm + C::OFF_PAGE);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (paged) stage_half_tile_rows(p.pt, b, kv, tile_begin, n_tiles, p.total_keys, sPage, p.err);
  // w' = w * q_scale for this CTA's tokens (0 for rows past the sequence)
  for (int i = threadIdx.x; i < TOK * 64; i += kThreads) {
    const int tk = i >> 6;
    float v = 0.f;
    if (tk < ntok) {
      const int64_t o = static_cast<int64_t>(row0 + tk) * 64 + (i & 63);
      v = __ldg(&p.w[o]) * __ldg(&p.q_scale[o]);
    }
    sW[i] = v;
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);   // one arrival per epilogue warp of the group
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // failure-path tests: this CTA withholds one accumulator release
  const int skip_item =
      (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) ? p.skip_arrival : -1;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer --
    if (elect_one()) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
      for (int piece = 0; piece < (TOK * 64) / C::BOXQ; ++piece) {
        tma_load_2d(sQ + piece * C::BOXQ * 128, &tmap_q, q_full, 0, row0 * 64 + piece * C::BOXQ);
      }
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.budget)) {
          report_error(p.err, kDevErrTimeout, 110, it);
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::K_BYTES);
        load_k_tile(sK + s * C::K_BYTES, &tmap_k, &full[s], paged, sPage, it,
                    kstart + static_cast<int64_t>(tile_begin + it) * 128);
        issued = it + 1;
      }
      // No copy may still be writing shared memory when the CTA leaves: wait
      // for the last load of every stage (already complete on the normal
      // path, where the MMA warp consumed them) and for the q tile.
      for (int it = max(0, issued - C::STAGES); it < issued; ++it) {
        if (!mbar_wait(&full[it % C::STAGES], (it / C::STAGES) & 1, p.budget))
          report_error(p.err, kDevErrTimeout, 111, it);
      }
      if (!mbar_wait(q_full, 0, p.budget)) report_error(p.err, kDevErrTimeout, 112, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer --
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, C::N, 0, 0);
      bool ok = mbar_wait(q_full, 0, p.budget);
      if (!ok) report_error(p.err, kDevErrTimeout, 120, 0);
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int s = it % C::STAGES;
        if (!mbar_wait(&full[s], (it / C::STAGES) & 1, p.budget)) {
          report_error(p.err, kDevErrTimeout, 121, it);
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sK + s * C::K_BYTES);
#pragma unroll
        for (int g = 0; g < C::NG; ++g) {
          const int item = it * C::NG + g;
          const int buf = item % kAccBufs;
          if (!mbar_wait(&acc_empty[buf], ((item / kAccBufs) & 1) ^ 1, p.budget)) {
            report_error(p.err, kDevErrTimeout, 122, it);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_base = smem_u32(sQ + g * C::N * 128);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            umma_e4m3(tmem + buf * C::N, smem_desc(a_base + k * 32, 16, 1024, kSwizzle128B),
                      smem_desc(b_base + k * 32, 16, 1024, kSwizzle128B), idesc, k > 0 ? 1u : 0u);
          }
          umma_commit(&acc_full[buf]);
        }
        umma_commit(&empty[s]);
      }
      // every MMA (and commit) of this CTA has completed before anyone frees
      // TMEM or leaves, whether the loop ran to the end or stopped on a timeout
      umma_commit(mma_done);
      if (!mbar_wait(mma_done, 0, p.budget)) report_error(p.err, kDevErrTimeout, 123, 0);
    }
  } else {
    // --------------------------------------------------- epilogue --
    const int ew = static_cast<int>(warp) - 2;   // 0..15
    const int g = ew >> 2;                       // accumulator buffer this warpgroup drains
    const uint32_t quarter = warp & 3u;          // TMEM lanes this warp may access
    const int key_in_tile = static_cast<int>(quarter * 32 + lane);
    const uint32_t lane_addr = (quarter * 32u) << 16;
    const int n_items = n_tiles * C::NG;
    // k_scale of this thread's key in the group's next item, fetched one item ahead
    auto key_scale = [&](int item) {
      const int it = item / C::NG;
      const int s = (tile_begin + it) * 128 + key_in_tile;
      return (item < n_items && s < kv) ? scale_of_key(p.k_scale, paged, sPage, it, key_in_tile, kstart + s,
                                                       p.total_keys)
                                        : 0.f;
    };
    float ks_next = key_scale(g);
    for (int item = g; item < n_items; item += kAccBufs) {
      const int it = item / C::NG;
      const int grp = item % C::NG;
      const float ks = ks_next;
      ks_next = key_scale(item + kAccBufs);
      if (!mbar_wait(&acc_full[g], (item / kAccBufs) & 1, p.budget)) {
        report_error(p.err, kDevErrTimeout, 130, item);
        break;
      }
      tc_fence_after();
      const int s = (tile_begin + it) * 128 + key_in_tile;
      // four running sums (heads j mod 4) kept as two f32x2 pairs: each lane
      // of fma.rn.f32x2 is the fp32 fma of the scalar form, so the sums are
      // bit-identical to it, in half the FMA instructions.  Heads 0-31 then
      // 32-63 of a token, in that order.
      auto half_sum = [&](const uint32_t (&r)[32], const ulonglong2* w, unsigned long long& a01,
                          unsigned long long& a23) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const ulonglong2 wv = w[j];
          a01 = ffma2(wv.x, pack2(fmaxf(__uint_as_float(r[4 * j + 0]), 0.f),
                                  fmaxf(__uint_as_float(r[4 * j + 1]), 0.f)), a01);
          a23 = ffma2(wv.y, pack2(fmaxf(__uint_as_float(r[4 * j + 2]), 0.f),
                                  fmaxf(__uint_as_float(r[4 * j + 3]), 0.f)), a23);
        }
      };
      auto store = [&](int tk, unsigned long long a01, unsigned long long a23) {
        const int tok = grp * C::GTOK + tk;
        const float2 s01 = unpack2(a01), s23 = unpack2(a23);
        const float acc = (s01.x + s01.y) + (s23.x + s23.y);
        if (tok < ntok && s <= t_first + tok) p.scores[static_cast<int64_t>(row0 + tok) * p.ld + s] = acc * ks;
      };
      const ulonglong2* w2 = reinterpret_cast<const ulonglong2*>(sW + grp * C::GTOK * 64);
      const uint32_t taddr = tmem + lane_addr + static_cast<uint32_t>(g * C::N);
      uint32_t ra[32], rb[32];
      tmem_ld32(taddr, ra);
      tmem_ld32(taddr + 32, rb);
      tmem_ld_wait();
      unsigned long long a01 = 0ull, a23 = 0ull;
      half_sum(ra, w2, a01, a23);
      // a second token: its first half is loaded while the first token's
      // second half is summed
      if constexpr (C::GTOK == 2) tmem_ld32(taddr + 64, ra);
      half_sum(rb, w2 + 8, a01, a23);
      store(0, a01, a23);
      if constexpr (C::GTOK == 2) {
        tmem_ld32(taddr + 96, rb);
        tmem_ld_wait();
        a01 = 0ull;
        a23 = 0ull;
        half_sum(ra, w2 + 16, a01, a23);
        half_sum(rb, w2 + 24, a01, a23);
        store(1, a01, a23);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && item != skip_item) mbar_arrive(&acc_empty[g]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ===========================================================================
// Fused decode indexer + top-k
//
// "DeepSeek V3.2 稀疏注意力" (what happens in prefill and decode): score the
// keys tile by tile, keep local candidates, merge them, and hand the selection
// straight to sparse MLA without writing the score matrix to HBM.  Here a
// cluster of C CTAs takes one (sequence, token group) of a decode batch: CTA r
// scores a contiguous chunk of the row's key tiles exactly as the indexer
// kernel above does, but keeps the scores in its shared memory; the cluster
// then selects the row's top k with an exact radix select over
// order-preserving keys (11/11/10-bit digits), the per-digit histograms
// all-reduced across the cluster through distributed shared memory.  Equal
// scores are taken in ascending position (lower position wins), so each CTA
// gets a quota of the threshold-valued positions in rank order, and writes its
// selected positions, ascending, at its offset in the output row -- the same
// set and order as dsa_topk on the same scores.
//
// Every CTA of a cluster executes the same sequence of cluster barriers: the
// only early exits depend on the cluster's (sequence, token group) alone, and
// a timed-out wait inside the tile loop only records the error and leaves the
// scores undefined, never the selection.
// ===========================================================================
constexpr int kRadixBins = 2048;

template <int TOK>
struct FusedCfg {
  static_assert(TOK == 1 || TOK == 2, "decode token groups");
  static constexpr int N = TOK * 64;                  // MMA N: the group's tokens x 64 heads
  static constexpr int STAGES = TOK == 1 ? 8 : 4;
  static constexpr int TMEM_COLS = kAccBufs * N;      // 256 or 512
  static constexpr int CAPT = 16384;                  // keys one CTA holds the scores of (per token)
  static constexpr int Q_BYTES = TOK * 64 * 128;
  static constexpr int K_BYTES = 128 * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_S = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_HIST = OFF_S + TOK * CAPT * 4;
  static constexpr int OFF_W = OFF_HIST + 2 * kRadixBins * 4;
  static constexpr int OFF_BAR = OFF_W + TOK * 64 * 4;
  static constexpr int NUM_BARS = 2 * STAGES + 1 + 2 * kAccBufs;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // tmem slot (4) + pad (12) | exchange slots [8] + per-rank counts [16] (96) | scan scratch [32] (128)
  // | broadcast [4] (16) | paged caches: pool rows of the chunk's 64-key halves [2 * CAPT / 128]
  static constexpr int OFF_CNT = (OFF_MISC + 16 + 15) / 16 * 16;   // 16-byte aligned: read as v4 by peers
  static constexpr int OFF_WARP = OFF_CNT + 96;
  static constexpr int OFF_BC = OFF_WARP + 128;
  static constexpr int OFF_PAGE = OFF_BC + 16;
  static constexpr int SMEM = OFF_PAGE + 4 * (2 * CAPT / 128) + 1024;
  static_assert(OFF_K % 1024 == 0 && OFF_S % 16 == 0 && OFF_HIST % 16 == 0 && OFF_CNT % 16 == 0, "alignment");
  static_assert(SMEM <= 232448, "shared memory");
};

// The row's top k, selected by the C CTAs of the cluster together.  CTA
// `crank` holds the scores of positions [p0, p0 + len) in sc[0 .. len); the
// CTAs' ranges follow each other in rank order and cover the n > k positions
// of the row.  Writes k positions into out (ascending).  Every thread of every
// CTA of the cluster calls it.
__device__ void cluster_radix_topk(const float* __restrict__ sc, int len, int p0, int k, int32_t* __restrict__ out,
                                   uint32_t* hist, uint32_t* cnt, uint32_t* s_warp, uint32_t* s_bc, int C,
                                   uint32_t crank) {
  constexpr int NT = kThreads;
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t FULL = 0xffffffffu;
  uint32_t prefix = 0, remaining = static_cast<uint32_t>(k);
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int width = pass == 2 ? 10 : 11;
    const uint32_t mask = (1u << width) - 1u;
    const int upper = shift + width;
    // two histogram buffers: a CTA rewrites the one of pass p - 2 only after
    // the cluster barrier of pass p - 1, which every CTA reaches after its
    // reads of pass p - 2
    uint32_t* hb = hist + (pass & 1) * kRadixBins;
    for (int j = tid; j < kRadixBins; j += NT) hb[j] = 0u;
    __syncthreads();
    const int rounds = (len + NT - 1) / NT;
#pragma unroll 1
    for (int r = 0; r < rounds; ++r) {
      const int e = r * NT + tid;
      uint32_t key = 0;
      bool match = false;
      if (e < len) {
        key = order_key(sc[e]);
        match = upper >= 32 || (key >> upper) == prefix;
      }
      const uint32_t digit = (key >> shift) & mask;
      const uint32_t active = __ballot_sync(FULL, match);
      if (match) {
        const uint32_t peers = __match_any_sync(active, digit);
        if ((__ffs(peers) - 1) == lane) atomicAdd(&hb[digit], static_cast<uint32_t>(__popc(peers)));
      }
    }
    __syncthreads();
    cluster_sync();          // every CTA's histogram of this pass is complete and visible
    // cluster-wide counts of bins 2047 - (4 tid + j), j = 0..3 (descending digits)
    uint32_t v[4] = {0u, 0u, 0u, 0u};
    if (tid < kRadixBins / 4) {
      const uint32_t a = smem_u32(hb + kRadixBins - 4 - 4 * tid);
      for (int r = 0; r < C; ++r) {
        const uint4 h = ld_shared_cluster_v4(mapa_shared(a, static_cast<uint32_t>(r)));
        v[0] += h.w;
        v[1] += h.z;
        v[2] += h.y;
        v[3] += h.x;
      }
    }
    uint32_t total;
    uint32_t above = block_excl_scan<NT>(v[0] + v[1] + v[2] + v[3], s_warp, total);
    // the digit d with count(digits above d) < remaining <= count(digits >= d)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (above < remaining && above + v[j] >= remaining) {
        s_bc[0] = static_cast<uint32_t>(kRadixBins - 1 - (4 * tid + j));
        s_bc[1] = above;
      }
      above += v[j];
    }
    __syncthreads();
    prefix = (prefix << width) | s_bc[0];
    remaining -= s_bc[1];
    __syncthreads();
  }
  // T = the k-th largest key; `remaining` positions of key T are needed, the
  // lowest positions first.  Each thread takes a contiguous run of positions
  // (odd length: consecutive lanes hit different banks).
  const uint32_t T = prefix;
  const int seg = ((len + NT - 1) / NT) | 1;
  const int e0 = min(tid * seg, len), e1 = min(e0 + seg, len);
  uint32_t gt = 0, eq = 0;
  for (int e = e0; e < e1; ++e) {
    const uint32_t key = order_key(sc[e]);
    gt += key > T;
    eq += key == T;
  }
  uint32_t tot;
  const uint32_t off = block_excl_scan<NT>((gt << 16) | eq, s_warp, tot);   // per-CTA counts < 2^16
  if (tid == 0) {
    cnt[0] = tot >> 16;
    cnt[1] = tot & 0xFFFFu;
  }
  __syncthreads();
  cluster_sync();            // every CTA's counts are visible
  if (tid == 0) {
    // ties go to the lower ranks (lower positions) first
    uint32_t rem = remaining, base = 0;
    for (uint32_t r = 0; r < crank; ++r) {
      const uint2 c = ld_shared_cluster_v2(mapa_shared(smem_u32(cnt), r));
      const uint32_t q = min(rem, c.y);
      rem -= q;
      base += c.x + q;
    }
    s_bc[2] = min(rem, cnt[1]);
    s_bc[3] = base;
  }
  __syncthreads();
  const uint32_t quota = s_bc[2];
  int32_t* dst = out + s_bc[3];
  uint32_t o_gt = off >> 16, o_eq = off & 0xFFFFu;
  for (int e = e0; e < e1; ++e) {
    const uint32_t key = order_key(sc[e]);
    if (key > T) {
      dst[o_gt + min(o_eq, quota)] = p0 + e;
      ++o_gt;
    } else if (key == T) {
      if (o_eq < quota) dst[o_gt + o_eq] = p0 + e;
      ++o_eq;
    }
  }
  __syncthreads();           // s_bc / s_warp are reused by the next row
}

// The row's top k by value bins, the common case.  Scratch (16 KB of shared
// memory per CTA): [0, 8K) histogram, later the chunk's bitmask of selected
// boundary positions; [8K, 12K) this CTA's boundary candidates (values,
// positions); [12K, 16K) every CTA's candidates.  slots[0..5] are read by the
// other CTAs of the cluster; slots[6] is local.
//   1. cluster-wide range [lo, hi] of the scores (and whether any is not finite);
//   2. a 2048-bin histogram over equal-width value bins of [lo, hi] (an fma
//      of the value, so bins are ordered like the scores), all-reduced over
//      the cluster: the bin b* holding the k-th largest score;
//   3. every position above b* is selected; the positions inside b* (tens on
//      indexer rows) are gathered from all CTAs and ranked exactly (higher
//      score, then lower position) by every CTA alike;
//   4. each CTA writes its selected positions, ascending, at its offset.
// Rows with a non-finite score, a single value, or more than kCandCap
// positions in b* return false before writing anything (uniformly across the
// cluster); the caller then runs the radix select.
constexpr int kCandCap = 512;

__device__ __forceinline__ float key_to_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__device__ bool cluster_value_topk(const float* __restrict__ sc, int len, int p0, int k, int32_t* __restrict__ out,
                                   uint8_t* scratch, uint32_t* slots, uint32_t* s_warp, uint32_t* s_bc, int C,
                                   uint32_t crank) {
  constexpr int NT = kThreads;
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t FULL = 0xffffffffu;
  uint32_t* hist = reinterpret_cast<uint32_t*>(scratch);
  float* own_v = reinterpret_cast<float*>(scratch + 8192);
  int32_t* own_p = reinterpret_cast<int32_t*>(scratch + 10240);
  float* all_v = reinterpret_cast<float*>(scratch + 12288);
  int32_t* all_p = reinterpret_cast<int32_t*>(scratch + 14336);

  // ---- 1. range ----
  if (tid == 0) {
    slots[0] = 0u;            // max key
    slots[1] = 0xFFFFFFFFu;   // min key
    slots[2] = 0u;            // any non-finite
    slots[4] = 0u;            // positions above b*
    slots[5] = 0u;            // boundary candidates
  }
  __syncthreads();
  {
    uint32_t kmax = 0u, kmin = 0xFFFFFFFFu, bad = 0u;
    for (int e = tid; e < len; e += NT) {
      const float x = sc[e];
      if (!(fabsf(x) <= 3.402823466e38f)) {
        bad = 1u;
      } else {
        const uint32_t key = order_key(x);
        kmax = max(kmax, key);
        kmin = min(kmin, key);
      }
    }
    kmax = __reduce_max_sync(FULL, kmax);
    kmin = __reduce_min_sync(FULL, kmin);
    bad = __reduce_or_sync(FULL, bad);
    if (lane == 0) {
      atomicMax(&slots[0], kmax);
      atomicMin(&slots[1], kmin);
      atomicOr(&slots[2], bad);
    }
  }
  __syncthreads();
  cluster_sync();                          // (1) every CTA's range is visible
  uint32_t gmax = 0u, gmin = 0xFFFFFFFFu, gbad = 0u;
  for (int r = 0; r < C; ++r) {
    const uint4 v = ld_shared_cluster_v4(mapa_shared(smem_u32(slots), static_cast<uint32_t>(r)));
    gmax = max(gmax, v.x);
    gmin = min(gmin, v.y);
    gbad |= v.z;
  }
  if (gbad != 0u || gmax <= gmin) return false;   // uniform: every CTA read the same slots
  const float lo = key_to_float(gmin), hi = key_to_float(gmax);
  const float scale = static_cast<float>(kRadixBins) / (hi - lo);
  if (!(scale <= 3.0e38f)) return false;           // a range too narrow for float bins
  const float off = 8388608.0f - lo * scale;
  auto bin_of = [&](float x) -> int {
    const int bb = static_cast<int>(__float_as_uint(__fmaf_rn(x, scale, off))) - 0x4B000000;
    return min(max(bb, 0), kRadixBins - 1);
  };

  // ---- 2. histogram of value bins, cluster-wide ----
  for (int j = tid; j < kRadixBins; j += NT) hist[j] = 0u;
  __syncthreads();
  for (int e = tid; e < len; e += NT) atomicAdd(&hist[bin_of(sc[e])], 1u);
  __syncthreads();
  cluster_sync();                          // (2) every CTA's histogram is complete
  uint32_t v[4] = {0u, 0u, 0u, 0u};        // bins 2047 - (4 tid + j), summed over the cluster
  if (tid < kRadixBins / 4) {
    const uint32_t a = smem_u32(hist + kRadixBins - 4 - 4 * tid);
    for (int r = 0; r < C; ++r) {
      const uint4 h = ld_shared_cluster_v4(mapa_shared(a, static_cast<uint32_t>(r)));
      v[0] += h.w;
      v[1] += h.z;
      v[2] += h.y;
      v[3] += h.x;
    }
  }
  uint32_t total;
  uint32_t above = block_excl_scan<NT>(v[0] + v[1] + v[2] + v[3], s_warp, total);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (above < static_cast<uint32_t>(k) && above + v[j] >= static_cast<uint32_t>(k)) {
      s_bc[0] = static_cast<uint32_t>(kRadixBins - 1 - (4 * tid + j));
      s_bc[1] = above;
      s_bc[2] = v[j];
    }
    above += v[j];
  }
  __syncthreads();
  const int bstar = static_cast<int>(s_bc[0]);
  const uint32_t above_all = s_bc[1];
  if (s_bc[2] > static_cast<uint32_t>(kCandCap)) {
    cluster_sync();                        // nobody reads our histogram any more
    return false;
  }
  const uint32_t rem = static_cast<uint32_t>(k) - above_all;

  // ---- 3. above b*: counted; inside b*: candidates ----
  {
    uint32_t n_above = 0;
    for (int e = tid; e < len; e += NT) {
      const float x = sc[e];
      const int bb = bin_of(x);
      n_above += bb > bstar;
      if (bb == bstar) {
        const uint32_t slot = atomicAdd(&slots[5], 1u);    // < kCandCap: the cluster's b* count is
        own_v[slot] = x;
        own_p[slot] = p0 + e;
      }
    }
    n_above = __reduce_add_sync(FULL, n_above);
    if (lane == 0 && n_above) atomicAdd(&slots[4], n_above);
  }
  __syncthreads();
  cluster_sync();                          // (3) every CTA's candidates and counts are visible
  // gather all candidates (in rank order of their CTAs) and every CTA's count above b*
  uint32_t n_all = 0, my_base = 0, my_n = 0, base_above = 0;
  {
    for (int r = 0; r < C; ++r) {
      const uint2 c = ld_shared_cluster_v2(mapa_shared(smem_u32(slots + 4), static_cast<uint32_t>(r)));
      const uint32_t src_v = mapa_shared(smem_u32(own_v), static_cast<uint32_t>(r));
      const uint32_t src_p = mapa_shared(smem_u32(own_p), static_cast<uint32_t>(r));
      for (uint32_t i = tid; i < c.y; i += NT) {
        uint32_t vb, pb;
        asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(vb) : "r"(src_v + 4 * i) : "memory");
        asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(pb) : "r"(src_p + 4 * i) : "memory");
        all_v[n_all + i] = __uint_as_float(vb);
        all_p[n_all + i] = static_cast<int32_t>(pb);
      }
      if (static_cast<uint32_t>(r) == crank) {
        my_base = n_all;
        my_n = c.y;
      }
      if (static_cast<uint32_t>(r) < crank) base_above += c.x;
      n_all += c.y;
    }
  }
  __syncthreads();
  // ---- 4. rank the candidates (every CTA ranks the same list the same way);
  // this CTA's output offset and the bitmap of its selected candidates ----
  uint32_t* bits = hist;                   // the histogram is dead: every CTA read it before (3)
  for (int j = tid; j < (len + 31) / 32; j += NT) bits[j] = 0u;
  if (tid == 0) slots[6] = 0u;             // selected candidates of lower ranks (local only)
  __syncthreads();
  for (uint32_t i = tid; i < n_all; i += NT) {
    const float x = all_v[i];
    const int pos = all_p[i];
    uint32_t rk = 0;
    for (uint32_t j = 0; j < n_all; ++j) {
      const float y = all_v[j];
      rk += (y > x) || (y == x && all_p[j] < pos);
    }
    if (rk < rem) {
      if (i < my_base) {
        atomicAdd(&slots[6], 1u);          // candidates come grouped by rank, lower ranks first
      } else if (i < my_base + my_n) {
        const int e = pos - p0;
        atomicOr(&bits[e >> 5], 1u << (e & 31));
      }
    }
  }
  __syncthreads();
  // ---- 5. ordered write: each thread a contiguous run (odd length) ----
  const uint32_t base = base_above + slots[6];
  const int seg = ((len + NT - 1) / NT) | 1;
  const int e0 = min(tid * seg, len), e1 = min(e0 + seg, len);
  auto chosen = [&](int e) {
    const int bb = bin_of(sc[e]);
    return bb > bstar || (bb == bstar && ((bits[e >> 5] >> (e & 31)) & 1u));
  };
  uint32_t n_sel = 0;
  for (int e = e0; e < e1; ++e) n_sel += chosen(e);
  uint32_t tot;
  uint32_t o = base + block_excl_scan<NT>(n_sel, s_warp, tot);
  for (int e = e0; e < e1; ++e)
    if (chosen(e)) out[o++] = p0 + e;
  __syncthreads();
  return true;
}

template <int TOK>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_topk_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const IndexerTopkParams fp) {
  using C = FusedCfg<TOK>;
  const IndexerParams& p = fp.ix;
  extern __shared__ uint8_t smem_raw[];

  // ---- work unit: sequence b, token group, this CTA's chunk of key tiles.
  // Every early exit below depends on (b, group) only: the whole cluster
  // takes it together. ----
  const uint32_t crank = cluster_ctarank();
  const int ncl = static_cast<int>(gridDim.x);         // CTAs per cluster (the cluster spans x)
  const int b = blockIdx.z;
  const int qblock = static_cast<int>(blockIdx.y);
  const int q0 = __ldg(&p.cu_q[b]);
  const int q_len = __ldg(&p.cu_q[b + 1]) - q0;
  const int kv = __ldg(&p.kv_len[b]);
  const int first = qblock * TOK;
  if (first >= q_len) return;
  const int64_t kstart = seq_start(p.pt, p.kv_start, b);
  if (q_len > kv || kv > fp.max_kv_len || !seq_rows_ok(p.pt, kstart, kv, p.total_keys)) {
    if (threadIdx.x == 0 && crank == 0) report_error(p.err, kDevErrBounds, 151, b);
    return;
  }
  const int ntok = min(TOK, q_len - first);
  const int t_first = kv - q_len + first;
  const int t_last = t_first + ntok - 1;
  const int tiles_total = (t_last + 1 + 127) / 128;
  const int tpc = (tiles_total + ncl - 1) / ncl;       // <= CAPT / 128 (checked on the host via max_kv_len)
  const int tile_begin = min(static_cast<int>(crank) * tpc, tiles_total);
  const int n_tiles = min(tile_begin + tpc, tiles_total) - tile_begin;   // may be 0
  const int p0 = tile_begin * 128;
  const int row0 = q0 + first;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = sm + C::OFF_Q;
  uint8_t* sK = sm + C::OFF_K;
  float* sS = reinterpret_cast<float*>(sm + C::OFF_S);
  uint32_t* hist = reinterpret_cast<uint32_t*>(sm + C::OFF_HIST);
  uint8_t* scratch = sm + C::OFF_HIST;      // the selection's 16 KB (histograms or candidates)
  float* sW = reinterpret_cast<float*>(sm + C::OFF_W);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* q_full = bars + 2 * C::STAGES;
  uint64_t* acc_full = q_full + 1;
  uint64_t* acc_empty = q_full + 1 + kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  uint32_t* slots = reinterpret_cast<uint32_t*>(sm + C::OFF_CNT);
  uint32_t* s_warp = reinterpret_cast<uint32_t*>(sm + C::OFF_WARP);
  uint32_t* s_bc = reinterpret_cast<uint32_t*>(sm + C::OFF_BC);
  int32_t* sPage = reinterpret_cast<int32_t*>(sm + C::OFF_PAGE);
  const bool paged = p.pt.table != nullptr;

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (paged) stage_half_tile_rows(p.pt, b, kv, tile_begin, n_tiles, p.total_keys, sPage, p.err);

  for (int i = threadIdx.x; i < TOK * 64; i += kThreads) {
    const int tk = i >> 6;
    float v = 0.f;
    if (tk < ntok) {
      const int64_t o = static_cast<int64_t>(row0 + tk) * 64 + (i & 63);
      v = __ldg(&p.w[o]) * __ldg(&p.q_scale[o]);
    }
    sW[i] = v;
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer --
    if (elect_one()) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      tma_load_2d(sQ, &tmap_q, q_full, 0, row0 * 64);
      for (int it = 0; it < n_tiles; ++it) {
        const int s = it % C::STAGES;
        if (!mbar_wait(&empty[s], ((it / C::STAGES) & 1) ^ 1, p.budget)) {
          report_error(p.err, kDevErrTimeout, 160, it);
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::K_BYTES);
        load_k_tile(sK + s * C::K_BYTES, &tmap_k, &full[s], paged, sPage, it,
                    kstart + static_cast<int64_t>(tile_begin + it) * 128);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer --
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, C::N, 0, 0);
      bool ok = mbar_wait(q_full, 0, p.budget);
      if (!ok) report_error(p.err, kDevErrTimeout, 161, 0);
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int s = it % C::STAGES;
        const int buf = it % kAccBufs;
        if (!mbar_wait(&full[s], (it / C::STAGES) & 1, p.budget) ||
            !mbar_wait(&acc_empty[buf], ((it / kAccBufs) & 1) ^ 1, p.budget)) {
          report_error(p.err, kDevErrTimeout, 162, it);
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sK + s * C::K_BYTES);
        const uint32_t b_base = smem_u32(sQ);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          umma_e4m3(tmem + buf * C::N, smem_desc(a_base + k * 32, 16, 1024, kSwizzle128B),
                    smem_desc(b_base + k * 32, 16, 1024, kSwizzle128B), idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&acc_full[buf]);
        umma_commit(&empty[s]);
      }
    }
  } else {
    // --------------------------------------------------- epilogue --
    // as in the indexer kernel, but each score goes to this CTA's chunk in
    // shared memory (a warp stores 32 consecutive floats)
    const int ew = static_cast<int>(warp) - 2;
    const int g = ew >> 2;
    const uint32_t quarter = warp & 3u;
    const int key_in_tile = static_cast<int>(quarter * 32 + lane);
    const uint32_t lane_addr = (quarter * 32u) << 16;
    auto key_scale = [&](int it) {
      const int s = (tile_begin + it) * 128 + key_in_tile;
      return (it < n_tiles && s < kv)
                 ? scale_of_key(p.k_scale, paged, sPage, it, key_in_tile, kstart + s, p.total_keys)
                 : 0.f;
    };
    float ks_next = key_scale(g);
    for (int it = g; it < n_tiles; it += kAccBufs) {
      const float ks = ks_next;
      ks_next = key_scale(it + kAccBufs);
      if (!mbar_wait(&acc_full[g], (it / kAccBufs) & 1, p.budget)) {
        report_error(p.err, kDevErrTimeout, 170, it);
        break;
      }
      tc_fence_after();
      const int e = it * 128 + key_in_tile;             // chunk-local position
#pragma unroll 1
      for (int tk = 0; tk < TOK; ++tk) {
        uint32_t ra[32], rb[32];
        const uint32_t taddr = tmem + lane_addr + static_cast<uint32_t>(g * C::N + tk * 64);
        tmem_ld32(taddr, ra);
        tmem_ld32(taddr + 32, rb);
        tmem_ld_wait();
        const ulonglong2* w2 = reinterpret_cast<const ulonglong2*>(sW + tk * 64);
        unsigned long long a01 = 0ull, a23 = 0ull;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const ulonglong2 wv = w2[j];
          a01 = ffma2(wv.x, pack2(fmaxf(__uint_as_float(ra[4 * j + 0]), 0.f),
                                  fmaxf(__uint_as_float(ra[4 * j + 1]), 0.f)), a01);
          a23 = ffma2(wv.y, pack2(fmaxf(__uint_as_float(ra[4 * j + 2]), 0.f),
                                  fmaxf(__uint_as_float(ra[4 * j + 3]), 0.f)), a23);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const ulonglong2 wv = w2[8 + j];
          a01 = ffma2(wv.x, pack2(fmaxf(__uint_as_float(rb[4 * j + 0]), 0.f),
                                  fmaxf(__uint_as_float(rb[4 * j + 1]), 0.f)), a01);
          a23 = ffma2(wv.y, pack2(fmaxf(__uint_as_float(rb[4 * j + 2]), 0.f),
                                  fmaxf(__uint_as_float(rb[4 * j + 3]), 0.f)), a23);
        }
        const float2 s01 = unpack2(a01), s23 = unpack2(a23);
        sS[tk * C::CAPT + e] = ((s01.x + s01.y) + (s23.x + s23.y)) * ks;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[g]);
    }
  }

  tc_fence_before();
  __syncthreads();           // every score of the chunk is in shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }

  // ---- selection, token by token ----
  const int k = fp.k_sel;
#pragma unroll 1
  for (int tk = 0; tk < ntok; ++tk) {
    const int n = t_first + tk + 1;                  // positions 0 .. t
    int32_t* out = fp.idx + static_cast<int64_t>(row0 + tk) * k;
    if (n <= k) {                                     // the whole prefix, then -1 (same in every CTA)
      if (crank == 0)
        for (int j = threadIdx.x; j < k; j += kThreads) out[j] = j < n ? j : -1;
      continue;
    }
    const int len = min(max(n - p0, 0), n_tiles * 128);
    const float* sc = sS + tk * C::CAPT;
    if (!cluster_value_topk(sc, len, p0, k, out, scratch, slots, s_warp, s_bc, ncl, crank))
      cluster_radix_topk(sc, len, p0, k, out, hist, slots + 6, s_warp, s_bc, ncl, crank);
    cluster_sync();          // every CTA is done reading this row's slots and candidates
  }
  cluster_sync();            // no CTA leaves while a peer may still read its shared memory
}

template <int TOK>
cudaError_t launch_fused_tok(int cluster, dim3 grid, const CUtensorMap& tq, const CUtensorMap& tk,
                             const IndexerTopkParams& p, cudaStream_t stream) {
  using C = FusedCfg<TOK>;
  auto kern = indexer_topk_kernel<TOK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  if (cluster > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int TOK>
cudaError_t launch_tok(dim3 grid, const CUtensorMap& tq, const CUtensorMap& tk, const IndexerParams& p,
                       cudaStream_t stream) {
  using C = IdxCfg<TOK>;
  const size_t smem = C::SMEM + (p.pt.table != nullptr ? 8 * static_cast<size_t>(p.tiles_per_chunk) : 0);
  if (smem > 232448) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(indexer_kernel<TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  indexer_kernel<TOK><<<grid, kThreads, smem, stream>>>(tq, tk, p);
  return cudaGetLastError();
}

}  // namespace

int indexer_tokens_per_cta(int max_q_per_seq) {
  if (max_q_per_seq >= 8) return 8;
  if (max_q_per_seq >= 4) return 4;
  if (max_q_per_seq >= 2) return 2;
  return 1;
}

size_t indexer_smem_bytes(int tok) {
  switch (tok) {
    case 1: return IdxCfg<1>::SMEM;
    case 2: return IdxCfg<2>::SMEM;
    case 4: return IdxCfg<4>::SMEM;
    default: return IdxCfg<8>::SMEM;
  }
}

int indexer_box_rows_q(int tok) {
  switch (tok) {
    case 1: return IdxCfg<1>::BOXQ;
    case 2: return IdxCfg<2>::BOXQ;
    case 4: return IdxCfg<4>::BOXQ;
    default: return IdxCfg<8>::BOXQ;
  }
}

// Clusters of `c` CTAs of the fused kernel (`tok` tokens) that can be
// resident at once on this device (cudaOccupancyMaxActiveClusters; 0 when the
// size cannot run).  Queried once per device and size.
static int fused_active_clusters(int tok, int c) {
  static std::atomic<int> cache[64][2][5];   // sizes 1, 2, 4, 8, 16
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return c <= 8 ? 1 : 0;
  const int li = c == 1 ? 0 : c == 2 ? 1 : c == 4 ? 2 : c == 8 ? 3 : 4;
  std::atomic<int>& slot = cache[dev][tok == 2 ? 1 : 0][li];
  int v = slot.load(std::memory_order_relaxed);
  if (v != 0) return v - 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(c), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(c);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  auto query = [&](auto kern, int smem) {
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return;
    if (c > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) return;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
  };
  if (tok == 2) query(indexer_topk_kernel<2>, FusedCfg<2>::SMEM);
  else query(indexer_topk_kernel<1>, FusedCfg<1>::SMEM);
  cudaGetLastError();   // a refused query leaves no sticky error behind
  slot.store(n + 1, std::memory_order_relaxed);
  return n;
}

int indexer_topk_cluster(int max_q_per_seq, int num_seqs, int max_kv_len) {
  if (max_q_per_seq < 1 || max_q_per_seq > 2 || num_seqs < 1 || max_kv_len < 1) return 0;
  const int tiles = (max_kv_len + 127) / 128;
  constexpr int cap_tiles = FusedCfg<1>::CAPT / 128;   // the same per token for both group sizes
  static_assert(FusedCfg<1>::CAPT == FusedCfg<2>::CAPT, "one chunk capacity");
  // enough CTAs for the row to fit in shared memory ...
  int c = 1;
  while (c <= 16 && (tiles + c - 1) / c > cap_tiles) c *= 2;
  if (c > 16) return 0;
  if (c > 8 && fused_active_clusters(max_q_per_seq, c) < 1) return 0;
  // ... and, while every cluster stays resident at once and each CTA keeps
  // >= 8 key tiles, more of them for bandwidth (each CTA streams its chunk)
  while (2 * c <= 16 && static_cast<int64_t>(num_seqs) * 2 * c <= sm_count() &&
         (tiles + 2 * c - 1) / (2 * c) >= 8 && fused_active_clusters(max_q_per_seq, 2 * c) >= num_seqs)
    c *= 2;
  return c;
}

bool indexer_topk_preferred(int max_q_per_seq, int num_seqs, int cluster) {
  // The fused kernel pays its cluster-wide selection once per token (~15 us
  // of passes and cluster barriers) and streams the keys with only
  // num_seqs x cluster CTAs; it beats the indexer + top-k pair (measured) for
  // one-token groups spread over at least ~2/3 of the SMs (64 x 16K-32K:
  // 70 vs 77 us; 16 x 32K: 40 vs 54 us), not for two-token groups on few
  // sequences (8 x 2 at 128K: 99 vs 81 us).
  return cluster > 0 && max_q_per_seq == 1 &&
         static_cast<int64_t>(num_seqs) * cluster * 3 >= static_cast<int64_t>(sm_count()) * 2;
}

cudaError_t launch_indexer_topk(int tok, int cluster, dim3 grid, const CUtensorMap& tmap_q,
                                const CUtensorMap& tmap_k, const IndexerTopkParams& p, cudaStream_t stream) {
  if (cluster < 1 || cluster > 16 || static_cast<int>(grid.x) != cluster) return cudaErrorInvalidValue;
  switch (tok) {
    case 1: return launch_fused_tok<1>(cluster, grid, tmap_q, tmap_k, p, stream);
    case 2: return launch_fused_tok<2>(cluster, grid, tmap_q, tmap_k, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_indexer(int tok, dim3 grid, const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                           const IndexerParams& p, cudaStream_t stream) {
  switch (tok) {
    case 1: return launch_tok<1>(grid, tmap_q, tmap_k, p, stream);
    case 2: return launch_tok<2>(grid, tmap_q, tmap_k, p, stream);
    case 4: return launch_tok<4>(grid, tmap_q, tmap_k, p, stream);
    case 8: return launch_tok<8>(grid, tmap_q, tmap_k, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
