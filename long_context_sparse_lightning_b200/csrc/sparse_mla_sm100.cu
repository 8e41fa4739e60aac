// Sparse MLA in MQA mode on sm_100a (tcgen05, TMEM operands and accumulators,
// a CTA pair per query token).
//
// "DeepSeek V3.2 稀疏注意力" (embedding DSA in MLA) and "NSA 与 DSA" §3.1: all
// query heads of a token share the same selected latent entries c_s (576-d =
// 512 latent + 64 RoPE; the value is the first 512 dims), so one gathered
// tile of entries feeds every head:
//     o[h] = sum_i softmax_i(sm_scale * q[h] . c[s_i]) * c[s_i][0:512].
//
// Work split: a cluster of two CTAs handles one token (or one split of its
// selection).  CTA r owns score dims [256r, 256r+256) U [512+32r, 544+32r)
// (288 of 576) and value dims [256r, 256r+256), so the 128 x 512 fp32 output
// accumulator is split 256 TMEM columns per CTA and each selected latent row is
// fetched once per pair.
//
// Tensor memory of one CTA (512 columns x 128 lanes, lane = head):
//   O [0,256) fp32, S [256,320) fp32, P [320,352) fp16 pairs, Q [352,496) fp16 pairs.
// Q and P are the A operands of their MMAs straight from TMEM, so the only
// shared-memory operand traffic is the gathered tile (B operand of both MMAs:
// K-major for Q.C^T, MN-major for P.V).
//
// Per tile of 64 selected entries:
//   gather     7 producer warps copy each row's 16-byte units with cp.async
//              straight into their swizzled slots, from an fp16 copy of the
//              latent cache (prefill: rows are reused across many tokens) or
//              from the bf16 cache (decode: Q.C^T then runs in bf16 on the
//              tile as it landed, and only afterwards do the producers convert
//              its value part to fp16 in place for P.V); 4-stage ring.  (TMA gather4 moves 4 rows x 128 B per
//              instruction and measured ~6 B/clk per SM on this pattern;
//              16-byte cp.async from 7 warps sustains several times that.)
//   MMA warp   S_r = Q_r . C_r^T (M=128, N=64, K=288) then O_r += P . V_r (N=256);
//   softmax    8 warps, 16 heads x 64 columns each: each warp ships its 4 KB of
//              fp32 partial scores to the peer with one bulk shared-to-shared
//              copy, one tile ahead of its own use so the transfer overlaps most
//              of an iteration, and adds the peer's fp32 partial to its own
//              (IEEE addition commutes, so both CTAs of the pair hold the same
//              fp32 scores bit for bit and compute one softmax: the same maxima,
//              probabilities, row sums and log-sum-exp); online softmax in log2
//              units with a lazily refreshed max (O rescaled in TMEM only when
//              the max grows by more than 2^8); P stored to TMEM as fp16.
//   MMA order  Q.C^T runs two tiles ahead of P.V.
// fp16 rather than bf16 inside the MMAs: with bf16 probabilities the rounding
// noise costs ~1e-3 mean relative error on the bf16 output; fp16 keeps ~1e-4.
// The conversion of q and the latent entries is exact in the normal fp16 range.
//
// Persistent pairs: each CTA pair walks a share of the (token, split) items.
// Per item the ring first carries the CTA's Q slice (two stage-sized TMA jobs,
// moved to TMEM as fp16 by the softmax warps), then the item's tiles; the
// producers stage the next item's positions and start its Q slice and first
// gathers while the current item's last tiles are still in the pipeline, and
// the next item's first Q.C^T runs during the current item's epilogue.  The
// bf16 output leaves by 16-byte stores of whole 64-byte runs per head (TMEM
// read with the .32x32b shape: lane = head).  A pair per token with a TMA
// store epilogue spent ~17K cycles per token outside the tile loop (prologue,
// epilogue, the next cluster's launch) against ~95K inside it.
//
// Decode shapes split a token's selection over several pairs; each writes a
// normalised partial output and its log-sum-exp, merged by mla_combine_kernel.
#include <atomic>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kTileKeys = 64;
constexpr int kStages = 4;
constexpr int KV_STAGE = 36864;          // 64 rows x (4 x 128 B latent + 64 B RoPE)
constexpr int KV_ROPE = 32768;
constexpr int XBLK = 4096;               // one softmax warp's partial scores: 16 heads x 64 keys fp32
constexpr int XBUF = 8 * XBLK;           // one tile's partial scores of all 8 softmax warps

constexpr uint32_t TM_O = 0;
constexpr uint32_t TM_S = 256;
constexpr uint32_t TM_P = 320;
constexpr uint32_t TM_Q = 352;
constexpr uint32_t kTmemCols = 512;

constexpr int OFF_KV = 0;
constexpr int OFF_STG = kStages * KV_STAGE;          // 147456: outgoing partial scores (one tile)
constexpr int OFF_X = OFF_STG + XBUF;                // 180224: incoming partial scores (one tile)
constexpr int OFF_IDX = OFF_X + XBUF;                // 212992: int32[2048]
constexpr int OFF_VALID = OFF_IDX + 2048 * 4;        // 221184: uint32[2][64] validity bits (item parity)
constexpr int OFF_BAR = OFF_VALID + 2 * 64 * 4;      // 221696
constexpr int OFF_INV = OFF_BAR + 512;               // 222208: float[2][128] inverse row sums (epilogue parity)
constexpr int OFF_MISC = OFF_INV + 2 * 128 * 4;      // 223232: TMEM address, ItemMeta[2]
constexpr int kSmem = OFF_MISC + 64 + 1024;

constexpr int kUnitsPerRow = 36;                     // 16-byte units of a row's 288-dim half
constexpr int kTileUnits = kTileKeys * kUnitsPerRow; // 2304
constexpr int kQBox = 16384;                         // one (up to) 128-row x 128-byte TMA box of Q

struct Bars {
  uint64_t q_full;          // the item's Q slice is in TMEM (8 softmax warps)
  uint64_t q_free;          // the MMA thread has seen that phase of q_full (one per Q slice)
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t qk_done[kStages];   // bf16 source: Q.C^T of the stage's tile has read it (MMA commit)
  uint64_t v_full[kStages];    // bf16 source: the stage's value part converted to fp16 in place
  uint64_t s_full, s_empty;
  uint64_t x_full[8], x_free[8];   // per softmax warp: peer's partial landed / peer has read ours
  uint64_t p_full, pv_done;
  uint64_t red;            // all softmax warps have published their inverse row sums
  uint64_t meta_full[2];   // item parity: selected positions staged (producers)
  uint64_t meta_free[2];   // item parity: the softmax warps are done with the validity bits
  uint64_t pbar;           // producer warps' own barrier (bounded, unlike bar.sync)
};
static_assert(sizeof(Bars) <= 512, "");

// Warp roles: 7 producer warps, 1 MMA warp, 8 softmax warps (two warpgroups,
// so warp w reaches TMEM lane quarter w % 4 as the hardware requires).
struct Cfg {
  static constexpr int NPROD = 7;
  static constexpr int MMA_WARP = NPROD;
  static constexpr int SOFT0 = NPROD + 1;
  static constexpr int THREADS = (NPROD + 1 + 8) * 32;
  static constexpr int PTHREADS = NPROD * 32;
  // registers per thread: 128 at launch; the producer + MMA warpgroups give up
  // 32 each so the softmax warpgroups get 160 (2 x 128 x 96 + 2 x 128 x 160 =
  // 512 x 128)
  static constexpr uint32_t REG_LOW = 96, REG_HIGH = 160;
};
static_assert(2 * 128 * Cfg::REG_LOW + 2 * 128 * Cfg::REG_HIGH == Cfg::THREADS * 128, "register split");
static_assert(Cfg::SOFT0 % 4 == 0, "softmax warps must start a warpgroup");
// Index staging: producer thread t takes slots t + 224 q; the last pass (q = 9)
// covers slots 2016..2047, i.e. exactly warp 0, so every pass is warp-uniform.
static_assert(9 * Cfg::PTHREADS + 32 == 2048, "index staging passes");
// A Q slice takes two ring jobs: latent boxes 0-1 (or 2-3) and RoPE rows 0-63 (64-127).
static_assert(2 * kQBox + 64 * 64 <= KV_STAGE, "half a Q slice must fit one ring stage");

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float lo = __uint_as_float(w << 16);
  const float hi = __uint_as_float(w & 0xFFFF0000u);
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint4 cvt_unit(uint4 v) {
  return make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// f32x2 register pairs (low element first) and their packed fma / add
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack_f32x2(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return make_float2(lo, hi);
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Global dim of 16-byte unit u (0..35) of CTA r's 288-dim half of a 576-d row.
__device__ __forceinline__ int unit_dim(int u, uint32_t r) {
  return u < 32 ? static_cast<int>(r) * 256 + u * 8 : 512 + static_cast<int>(r) * 32 + (u - 32) * 8;
}

// Shared-memory offset of unit u of row j inside a stage: units 0..31 form four
// 64-dim chunks (8 KB each, 128-byte swizzle), units 32..35 the RoPE chunk
// (64-byte swizzle): the canonical K-major SW128 / SW64 operand layouts.
__device__ __forceinline__ uint32_t tile_unit_offset(int j, int u) {
  if (u < 32) {
    const int c = u >> 3, cu = u & 7;
    return c * 8192 + j * 128 + ((cu ^ (j & 7)) << 4);
  }
  const int ru = u - 32;
  return KV_ROPE + j * 64 + ((ru ^ ((j >> 1) & 3)) << 4);
}

// What the producers publish about an item (one per item parity, before
// meta_full): the other roles read it from shared memory instead of
// recomputing it with dependent global loads.
struct ItemMeta {
  int32_t last;     // last valid slot of the selection, -1: none
  int32_t row, split, status;
};
static_assert(16 + 2 * sizeof(ItemMeta) <= 64, "item metadata fits the misc area");

// Work item w of a launch: token row w / nsplit of the batch, split w % nsplit.
// status 0: valid; 301: the sequence's descriptors are out of range (the row
// attends to nothing: out = 0, lse = -inf); 302: the row lies in no sequence
// of cu_q (the same: out = 0, lse = -inf).  Both record DSA_ERR_DEVICE_BOUNDS.
struct MlaItem {
  int row, split, b, kv, status;
  int e_begin, e_count;   // the split's slots of the selection
  int64_t kstart;
};

// Slots of the selection that split `split` covers.
__device__ __forceinline__ int split_slots(const MlaParams& p, int split) {
  const int e_begin = split * p.keys_per_split;
  return max(0, min(p.k_sel, e_begin + p.keys_per_split) - e_begin);
}

// Whether item w carries a Q slice through the ring: a function of the launch
// alone (no loads), so every role decides it at once and alike; an item whose
// sequence turns out to be invalid still takes (and drops) its slice.
__device__ __forceinline__ bool item_has_q(const MlaParams& p, int w) { return split_slots(p, w % p.nsplit) > 0; }

// The load-free part of an item: its row and slots.
__device__ __forceinline__ MlaItem mla_item_base(const MlaParams& p, int w) {
  MlaItem it;
  it.row = w / p.nsplit;
  it.split = w - it.row * p.nsplit;
  it.e_begin = it.split * p.keys_per_split;
  it.e_count = split_slots(p, it.split);
  it.b = 0;
  it.kv = 0;
  it.kstart = 0;
  it.status = 0;
  return it;
}

// The row's sequence and its descriptors (dependent loads).
// Called by whole warps (every lane gets the same result).
__device__ __forceinline__ void mla_item_seq(const MlaParams& p, MlaItem& it) {
  // The row's sequence: the last b with cu_q[b] <= row (empty sequences
  // skipped).  The 32 lanes sample the remaining range at once and a ballot
  // narrows it, so one round of loads covers 32 sequences and two cover 1024
  // (a binary search took one dependent load per halving: ~7 cold loads for
  // a 64-sequence decode batch).  An unsorted cu_q still yields some b in
  // range, which the check below rejects.
  const uint32_t lane = threadIdx.x & 31u;
  int lo = 0, hi = p.num_seqs - 1;
  while (lo < hi) {
    const int step = (hi - lo + 32) / 32;   // ceil((hi - lo + 1) / 32)
    const int idx = lo + static_cast<int>(lane) * step;
    const bool le = idx <= hi && __ldg(&p.cu_q[idx]) <= it.row;
    const uint32_t m = __ballot_sync(0xffffffffu, le);
    if (m == 0u) break;                     // cu_q[lo] > row: no sequence holds the row
    const int L = 31 - __clz(static_cast<int>(m));
    lo += L * step;
    hi = min(hi, lo + step - 1);
  }
  it.b = lo;
  const int q0 = __ldg(&p.cu_q[lo]);
  const int q_len = __ldg(&p.cu_q[lo + 1]) - q0;
  if (q0 < 0 || it.row < q0 || it.row >= q0 + q_len) {
    it.status = 302;
    return;
  }
  it.kv = __ldg(&p.kv_len[lo]);
  it.kstart = seq_start(p.pt, p.kv_start, lo);
  if (q_len > it.kv || !seq_rows_ok(p.pt, it.kstart, it.kv, p.total_keys)) it.status = 301;
}

// FP16_SRC: p.kv is an fp16 copy of the latent cache (rows land ready for the
// MMAs); otherwise p.kv is the bf16 cache: Q.C^T runs in bf16 and the producers
// convert the value part in place between Q.C^T and P.V.
//
// Persistent: gridDim.x / 2 CTA pairs; pair c takes items c, c + pairs, ...
// Every role walks the same item sequence and keeps the same counters (ring
// jobs, tiles, items with a Q slice), so the barrier phases agree across
// items.  Per item with n > 0 tiles the ring carries two Q jobs (the CTA's Q
// slice by TMA), then the n tiles.  The producers stage the next item's
// positions and issue its Q slice and first tiles while the current item's
// last tiles are still in the MMA / softmax pipeline; the softmax warps move
// the next Q slice into TMEM before the current item's epilogue, so the next
// item's first Q.C^T overlaps that epilogue.
template <bool FP16_SRC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg::THREADS, 1)
    sparse_mla_kernel(const MlaParams p, const __grid_constant__ MlaMaps maps) {
  using C = Cfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int n_pairs = static_cast<int>(gridDim.x >> 1);
  const int n_items = p.total_q * p.nsplit;
  const int H = p.n_heads;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sKV = sm + OFF_KV;
  int32_t* sIdx = reinterpret_cast<int32_t*>(sm + OFF_IDX);
  uint32_t* sValid = reinterpret_cast<uint32_t*>(sm + OFF_VALID);
  Bars* bar = reinterpret_cast<Bars*>(sm + OFF_BAR);
  float* sInv = reinterpret_cast<float*>(sm + OFF_INV);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  ItemMeta* meta = reinterpret_cast<ItemMeta*>(sm + OFF_MISC + 16);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int tid = threadIdx.x;

  if (tid == 0) {
    mbar_init(&bar->q_full, 8);
    mbar_init(&bar->q_free, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->kv_full[s], C::NPROD);
      mbar_init(&bar->kv_empty[s], 1);
      mbar_init(&bar->qk_done[s], 1);
      mbar_init(&bar->v_full[s], C::NPROD);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_empty, 8);
    for (int w = 0; w < 8; ++w) {
      mbar_init(&bar->x_full[w], 1);   // the receiving warp's expect_tx arrival + the peer's 4 KB copy
      mbar_init(&bar->x_free[w], 1);   // the peer warp's remote arrival once it has read the block
    }
    mbar_init(&bar->p_full, 8);
    mbar_init(&bar->pv_done, 1);
    mbar_init(&bar->red, 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->meta_full[i], 1);
      mbar_init(&bar->meta_free[i], 8);
    }
    mbar_init(&bar->pbar, C::NPROD);
    fence_mbar_init();
    prefetch_tmap(&maps.q_lat);
    prefetch_tmap(&maps.q_rope);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Our barriers are initialised: arrive on the cluster barrier now; each role
  // waits for the peer's arrival only before its first remote access (the
  // softmax warps' first score exchange) or at its end.
  cluster_arrive();
  const uint32_t tmem = *tmem_slot;

  if (warp < C::NPROD) {
    setmaxnreg_dec<C::REG_LOW>();
    // ------------------------------------------------------------ producers --
    // Each 16-byte unit goes straight to its swizzled slot with cp.async;
    // consecutive lanes take consecutive units of a row, so one warp request
    // covers a few whole 128-byte lines.  bf16 sources are converted to fp16 in
    // place by the thread that loaded them.
    const uint8_t* kvbase = reinterpret_cast<const uint8_t*>(p.kv);   // sIdx holds cache rows
    // this thread's units (the same slots in every tile): unit g = tid + m * PTHREADS
    // of the tile is row j = g / 36, 16-byte unit u = g % 36
    constexpr int UPT = (kTileUnits + C::PTHREADS - 1) / C::PTHREADS;
    uint32_t soff[UPT], goff[UPT], jrow[UPT];
#pragma unroll
    for (int m = 0; m < UPT; ++m) {
      const int g = min(tid + m * C::PTHREADS, kTileUnits - 1);
      const int j = g / kUnitsPerRow, u = g % kUnitsPerRow;
      soff[m] = tile_unit_offset(j, u);
      goff[m] = static_cast<uint32_t>(unit_dim(u, rank)) * 2u;
      jrow[m] = static_cast<uint32_t>(j);
    }
    auto mine = [&](int m) { return m + 1 < UPT || tid + m * C::PTHREADS < kTileUnits; };
    bool ok = true;
    uint32_t pb = 0;        // uses of the producer barrier
    // all producer warps (an mbarrier, so that a warp that gave up on an
    // earlier wait cannot leave the others blocked for good)
    auto pbar = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->pbar);
      const bool r = mbar_wait(&bar->pbar, pb & 1u, p.budget);
      ++pb;
      if (!__all_sync(0xffffffffu, r)) {
        if (lane == 0) report_error(p.err, kDevErrTimeout, 314, static_cast<int>(pb));
        ok = false;
      }
    };
    // ring job r: stage r % kStages, its use number r / kStages
    auto slot_wait = [&](int r) {
      if (ok && !mbar_wait(&bar->kv_empty[r % kStages], ((r / kStages) & 1) ^ 1, p.budget)) {
        report_error(p.err, kDevErrTimeout, 311, r);
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
    };
    int ring = 0;           // ring jobs issued so far (Q halves and tiles)
    // The next item: its row and slots need no loads; its sequence is looked
    // up while the current item's Q slice is in flight (the first item's while
    // its own slice and positions are).
    MlaItem nxt;
    if (pair < n_items) nxt = mla_item_base(p, pair);
    for (int k = 0; ok; ++k) {
      const int w = pair + k * n_pairs;
      if (w >= n_items) break;
      MlaItem it = nxt;
      // this item's positions: loads first (one memory latency)
      const int32_t* idx_row = p.idx + static_cast<int64_t>(it.row) * p.k_sel + it.e_begin;
      int v[10];
#pragma unroll
      for (int q = 0; q < 10; ++q) {
        const int j = tid + q * C::PTHREADS;
        v[q] = (j < 2048 && j < it.e_count) ? __ldg(&idx_row[j]) : -1;
      }
      // The CTA's Q slice: two ring jobs by TMA (latent boxes 2h, 2h+1 and RoPE
      // rows 64h..64h+63), issued before the positions are staged so that it
      // lands while the previous item's last tiles are still being processed.
      // Every warp waits for the slot before its arrival.
      if (item_has_q(p, w)) {
        const int rope_rows = H < 64 ? H : 64;
        for (int h = 0; ok && h < 2; ++h, ++ring) {
          slot_wait(ring);
          if (!ok) break;
          const int st = ring % kStages;
          if (lane == 0) {
            // bf16: close the stage's conversion phase for this job first, so
            // that the job's kv_full completion implies every warp's v_full arrival
            if constexpr (!FP16_SRC) mbar_arrive(&bar->v_full[st]);
            if (warp == 0) {
              const bool rope = h == 0 || H > 64;
              uint8_t* dst = sKV + st * KV_STAGE;
              mbar_arrive_expect_tx(&bar->kv_full[st],
                                    static_cast<uint32_t>(2 * H * 128 + (rope ? rope_rows * 64 : 0)));
              tma_load_2d(dst, &maps.q_lat, &bar->kv_full[st], static_cast<int>(rank) * 256 + 128 * h, it.row * H);
              tma_load_2d(dst + kQBox, &maps.q_lat, &bar->kv_full[st], static_cast<int>(rank) * 256 + 128 * h + 64,
                          it.row * H);
              if (rope)
                tma_load_2d(dst + 2 * kQBox, &maps.q_rope, &bar->kv_full[st], 512 + static_cast<int>(rank) * 32,
                            it.row * H + 64 * h);
            } else {
              mbar_arrive(&bar->kv_full[st]);
            }
          }
        }
        if (!ok) break;
      }
      if (k == 0) mla_item_seq(p, it);
      if (w + n_pairs < n_items) {
        nxt = mla_item_base(p, w + n_pairs);
        mla_item_seq(p, nxt);
      }
      if (it.status != 0 && tid == 0 && rank == 0) report_error(p.err, kDevErrBounds, it.status, it.b);
      // The previous item's tiles are issued and landed by every warp (sIdx is
      // free), and the validity buffer of this item's parity is free once the
      // softmax warps are done with item k - 2.
      if (tid == 0) {
        if (k >= 2 && !mbar_wait(&bar->meta_free[k & 1], ((k >> 1) + 1) & 1, p.budget)) {
          report_error(p.err, kDevErrTimeout, 315, k);
          ok = false;
        }
        ItemMeta& m = meta[k & 1];
        m.last = -1;
        m.row = it.row;
        m.split = it.split;
        m.status = it.status;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      pbar();
      if (!ok) break;
      // each selected position -> its cache row (flat or paged), invalid -> -1,
      // per-32 validity bits, the last valid slot
      uint32_t* sV = sValid + (k & 1) * 64;
      int my_last = -1;
#pragma unroll
      for (int q = 0; q < 10; ++q) {
        const int j = tid + q * C::PTHREADS;
        if (j < 2048) {
          int e = (it.status != 0 || v[q] < 0 || v[q] >= it.kv) ? -1 : v[q];
          if (e >= 0) {
            const int64_t r = cache_row(p.pt, it.b, it.kstart, e);
            if (r < 0) report_error(p.err, kDevErrBounds, 303, it.b);   // a page id outside the pool: skipped
            e = static_cast<int>(r);
          }
          sIdx[j] = e;
          const uint32_t bits = __ballot_sync(0xffffffffu, e >= 0);
          if (lane == 0) sV[j >> 5] = bits;
          if (e >= 0) my_last = j;
        }
      }
      if (my_last >= 0) atomicMax(&meta[k & 1].last, my_last);
      pbar();
      if (!ok) break;
      const int n_tiles = (meta[k & 1].last + 1 + kTileKeys - 1) / kTileKeys;
      if (tid == 0) mbar_arrive(&bar->meta_full[k & 1]);
      if (n_tiles == 0) continue;

      // the item's tiles: ring jobs r0 .. r0 + n_tiles - 1
      const int r0 = ring;
      const int32_t* sI = sIdx;
      auto issue = [&](int tile) {
        const int r = r0 + tile;
        slot_wait(r);
        if (ok) {
          const uint32_t base = smem_u32(sKV + (r % kStages) * KV_STAGE);
          const int32_t* e = sI + tile * kTileKeys;
#pragma unroll
          for (int m = 0; m < UPT; ++m) {
            if (mine(m)) {
              const int pos = max(e[jrow[m]], 0);
              cp_async_16(base + soff[m], kvbase + static_cast<int64_t>(pos) * 1152 + goff[m]);
            }
          }
        }
        cp_async_commit();
      };
      auto land = [&](int tile) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->kv_full[(r0 + tile) % kStages]);
      };
      if constexpr (FP16_SRC) {
        // Up to three tiles in flight (copies committed, not yet landed).  A
        // warp blocks on a ring slot only when it has nothing left to land:
        // landing tile t lets Q.C^T(t) run, and the P.V that frees a slot
        // comes after Q.C^T of the newer tiles, so waiting for a slot while
        // holding an unlanded tile would hold up the scores of that tile
        // (3.62 -> 3.43 ms at 4096 queries of 32K context).
        auto slot_free = [&](int tile) {
          const int r = r0 + tile;
          const bool f = mbar_test(smem_u32(&bar->kv_empty[r % kStages]), ((r / kStages) & 1) ^ 1);
          return __shfl_sync(0xffffffffu, f, 0);   // lane 0 decides for the warp
        };
        constexpr int kAhead = 3;
        int n_issued = 0;
        for (int n_landed = 0; ok && n_landed < n_tiles;) {
          const int in_flight = n_issued - n_landed;
          if (n_issued < n_tiles && in_flight < kAhead && (in_flight == 0 || slot_free(n_issued))) {
            issue(n_issued++);
            continue;
          }
          // the oldest tile's group completes once at most in_flight - 1
          // younger groups are pending
          if (in_flight >= 3) {
            cp_async_wait<2>();
          } else if (in_flight == 2) {
            cp_async_wait<1>();
          } else {
            cp_async_wait<0>();
          }
          land(n_landed++);
        }
      } else {
        // bf16 source (decode-shaped batches, a few tiles per pair): two tiles
        // ahead in program order -- land tile i, convert tile i-1, then wait
        // for tile i+2's slot.  (The fp16 schedule above measured slower here:
        // 82 -> 86 us for 64 decode tokens, tile 2's gather waiting for the
        // conversion of tile 0.)  Q.C^T reads the tile as bf16 (exact
        // products, like fp16); once it has, the value part (units 0..31)
        // becomes fp16 in place for P.V.
        auto convert = [&](int tile) {
          const int r = r0 + tile, st = r % kStages;
          if (ok && !mbar_wait(&bar->qk_done[st], (r / kStages) & 1, p.budget)) {
            report_error(p.err, kDevErrTimeout, 313, r);
            ok = false;
          }
          ok = __all_sync(0xffffffffu, ok);
          if (ok) {
            uint8_t* base = sKV + st * KV_STAGE;
#pragma unroll
            for (int m = 0; m < UPT; ++m) {
              if (mine(m) && soff[m] < static_cast<uint32_t>(KV_ROPE)) {   // a value unit
                uint4* q = reinterpret_cast<uint4*>(base + soff[m]);
                *q = cvt_unit(*q);
              }
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar->v_full[st]);
        };
        issue(0);
        if (n_tiles > 1) issue(1);
        for (int i = 0; ok && i < n_tiles; ++i) {
          if (i + 1 < n_tiles) {
            cp_async_wait<1>();
          } else {
            cp_async_wait<0>();
          }
          land(i);
          if (i > 0) convert(i - 1);
          if (i + 2 < n_tiles) issue(i + 2);
        }
        if (ok) convert(n_tiles - 1);
      }
      ring += n_tiles;
    }
    cp_async_wait<0>();
    cluster_wait();
  } else if (warp == C::MMA_WARP) {
    setmaxnreg_dec<C::REG_LOW>();
    // ----------------------------------------------------------- MMA issuer --
    if (elect_one()) {
      // Q.C^T in the source's type (bf16 Q in TMEM for a bf16 cache), P.V in fp16
      constexpr uint32_t kQkFmt = FP16_SRC ? 0u : kFmtBF16;
      constexpr uint32_t idesc_qk = idesc_f32acc(kQkFmt, kQkFmt, 128, 64, 0, 0);   // K-major
      constexpr uint32_t idesc_pv = idesc_f32acc(0, 0, 128, 256, 0, 1);    // P K-major, V MN-major
      int ring = 0, G = 0, qc = 0;   // ring jobs, tiles, Q slices so far
      for (int k = 0;; ++k) {
        const int w = pair + k * n_pairs;
        if (w >= n_items) break;
        if (!mbar_wait(&bar->meta_full[k & 1], (k >> 1) & 1, p.budget)) {
          report_error(p.err, kDevErrTimeout, 324, k);
          break;
        }
        const int n_tiles = (meta[k & 1].last + 1 + kTileKeys - 1) / kTileKeys;
        if (item_has_q(p, w)) {
          if (!mbar_wait(&bar->q_full, qc & 1, p.budget)) {
            report_error(p.err, kDevErrTimeout, 320, k);
            break;
          }
          // the Q slice is in TMEM: the softmax warps may convert the next
          // one once this phase has been seen, and its two ring stages are free
          // (bf16: their Q.C^T phase is closed too, keeping the per-stage
          // phases in step)
          mbar_arrive(&bar->q_free);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int st = (ring + h) % kStages;
            if constexpr (!FP16_SRC) mbar_arrive(&bar->qk_done[st]);
            mbar_arrive(&bar->kv_empty[st]);
          }
          ring += 2;
          ++qc;
        }
        if (n_tiles == 0) continue;
        // QK^T runs two tiles ahead of PV: the softmax reads S(i+1) while it
        // still works on tile i, so S(i+2) can be computed meanwhile.  Across
        // items the last two P.V of an item come before the next item's first
        // Q.C^T, which waits for the next Q slice (converted by the softmax
        // warps only once this item's tile loop is over).
        bool ok = true;
        for (int i = 0; ok && i < n_tiles + 2; ++i) {
          if (i < n_tiles) {
            const int r = ring + i, st = r % kStages, gt = G + i;
            if (!mbar_wait(&bar->kv_full[st], (r / kStages) & 1, p.budget) ||
                (gt > 0 && !mbar_wait(&bar->s_empty, (gt - 1) & 1, p.budget))) {
              report_error(p.err, kDevErrTimeout, 321, gt);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t kv_addr = smem_u32(sKV + st * KV_STAGE);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                umma_f16_ts(tmem + TM_S, tmem + TM_Q + c * 32 + kk * 8,
                            smem_desc(kv_addr + c * 8192 + kk * 32, 16, 1024, kSwizzle128B), idesc_qk,
                            (c | kk) ? 1u : 0u);
              }
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              umma_f16_ts(tmem + TM_S, tmem + TM_Q + 128 + kk * 8,
                          smem_desc(kv_addr + KV_ROPE + kk * 32, 16, 512, kSwizzle64B), idesc_qk, 1u);
            }
            umma_commit(&bar->s_full);
            if constexpr (!FP16_SRC) umma_commit(&bar->qk_done[st]);
          }
          if (i >= 2) {
            const int j = i - 2;
            const int r = ring + j, st = r % kStages, gt = G + j;
            if (!mbar_wait(&bar->p_full, gt & 1, p.budget)) {
              report_error(p.err, kDevErrTimeout, 322, gt);
              ok = false;
              break;
            }
            if (!FP16_SRC && !mbar_wait(&bar->v_full[st], (r / kStages) & 1, p.budget)) {
              report_error(p.err, kDevErrTimeout, 323, gt);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t kv_addr = smem_u32(sKV + st * KV_STAGE);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              umma_f16_ts(tmem + TM_O, tmem + TM_P + kk * 8,
                          smem_desc(kv_addr + kk * 2048, 8192, 1024, kSwizzle128B), idesc_pv,
                          (j | kk) ? 1u : 0u);
            }
            umma_commit(&bar->pv_done);
            umma_commit(&bar->kv_empty[st]);
          }
        }
        if (!ok) break;
        ring += n_tiles;
        G += n_tiles;
      }
    }
    cluster_wait();
  } else {
    setmaxnreg_inc<C::REG_HIGH>();
    // -------------------------------------------------------------- softmax --
    // Warp sw owns 16 heads -- TMEM lanes [32q + 16*(sw/4), +16) of its lane
    // quarter q = warp % 4 -- across all 64 columns of a tile, read with the
    // .16x256b shape: lane t holds heads rA = L + t/4 and rB = rA + 8, keys
    // 8k + 2(t%4) + {0, 1} for k = 0..7.  A head's 64 scores sit in the 4 lanes
    // of one group, so row max and sum need two shuffles and no other warp.
    const int sw = static_cast<int>(warp) - C::SOFT0;   // 0..7
    const uint32_t quarter = warp & 3u;
    const int L = static_cast<int>(quarter) * 32 + 16 * (sw >> 2);
    const int hA = L + static_cast<int>(lane >> 2), hB = hA + 8;
    const int ku = 2 * static_cast<int>(lane & 3u);     // this lane's key offset inside each group of 8
    const uint32_t tbase = tmem + (static_cast<uint32_t>(L) << 16);
    // partial-score blocks: 4 KB per warp per tile; lane l's 16-byte unit q at q*512 + l*16
    const uint32_t stg_base = smem_u32(sm + OFF_STG) + sw * XBLK;
    const uint32_t x_base = smem_u32(sm + OFF_X) + sw * XBLK;
    const uint32_t x_base_remote = mapa_shared(x_base, peer);
    const uint32_t x_full_remote = mapa_shared(smem_u32(&bar->x_full[sw]), peer);
    const uint32_t x_free_remote = mapa_shared(smem_u32(&bar->x_free[sw]), peer);
    const float NEG_INF = __int_as_float(0xff800000);
    const float scale = p.scale_log2;
    bool ok = true;
    // bounded wait polled by every lane (each lane acquires for itself); the
    // vote makes the outcome warp-uniform.  On an already completed phase this
    // costs ~55-80 cycles, against ~280 when lane 0 polls and broadcasts.
    auto wwait = [&](uint64_t* b_, uint32_t parity, bool cluster, uint32_t site, int info) -> bool {
      const bool r = cluster ? mbar_wait_cluster(b_, parity, p.budget) : mbar_wait(b_, parity, p.budget);
      const bool all = __all_sync(0xffffffffu, r);
      if (!all && lane == 0) report_error(p.err, kDevErrTimeout, site, info);
      return all;
    };
    // S of global tile t, this warp's 16 heads, this CTA's fp32 partial over
    // its 288 dims: s[4k], s[4k+1] = head rA, keys 8k+ku, 8k+ku+1; s[4k+2],
    // s[4k+3] = head rB.  Split in two so the TMEM load's latency overlaps
    // other work.
    auto load_s_issue = [&](int t, uint32_t (&s)[32]) -> bool {
      if (!wwait(&bar->s_full, t & 1, false, 330, t)) return false;
      tc_fence_after();
      tmem_ld_16x256b_x8(tbase + TM_S, s);
      return true;
    };
    auto load_s_finish = [&]() {
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->s_empty);
    };
    // ship this warp's block of S(t) to the peer: one 4 KB bulk copy of the
    // raw fp32 values.  One buffer each way: the peer's arrival on x_free
    // (it has read our block of tile t-1) also means that copy has finished
    // reading our staging block.
    auto send = [&](int t, const uint32_t (&s)[32]) -> bool {
      if (!wwait(&bar->x_free[sw], (t & 1) ^ 1, true, 331, t)) return false;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg_base + q * 512 + lane * 16), "r"(s[4 * q]),
                     "r"(s[4 * q + 1]), "r"(s[4 * q + 2]), "r"(s[4 * q + 3])
                     : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) bulk_copy_to_peer(x_base_remote, stg_base, XBLK, x_full_remote);
      return true;
    };
    // The Q slice of the item whose Q jobs are ring jobs rq, rq + 1 -> TMEM
    // (shape .32x32b: lane = head): warps of the first warpgroup write dims
    // [0, 144) of the CTA's 288, the second [144, 288).  Stage A holds latent
    // boxes 0-1 and RoPE rows 0-63, stage B boxes 2-3 and RoPE rows 64-127.
    int qn = 0;   // Q slices converted so far
    auto convert_q = [&](int rq, int info) -> bool {
      const int sa = rq % kStages, sb = (rq + 1) % kStages;
      // the MMA thread has seen the previous slice's q_full phase (so this
      // slice's arrivals cannot run a phase ahead of it), and the slice landed
      if ((qn > 0 && !wwait(&bar->q_free, (qn - 1) & 1, false, 337, info)) ||
          !wwait(&bar->kv_full[sa], (rq / kStages) & 1, false, 338, info) ||
          !wwait(&bar->kv_full[sb], ((rq + 1) / kStages) & 1, false, 338, info))
        return false;
      const uint8_t* qa = sKV + sa * KV_STAGE;
      const uint8_t* qb = sKV + sb * KV_STAGE;
      const int g = sw >> 2;
      const int h = static_cast<int>(quarter * 32 + lane);
      const int hl = h & 63;
      uint32_t qv[72];
#pragma unroll
      for (int m = 0; m < 18; ++m) {
        const int u = 18 * g + m;        // unit of the CTA's 288 dims: 0..31 latent, 32..35 RoPE
        const uint8_t* src;
        if (u < 32) {
          const int c = u >> 3;
          src = ((c >> 1) ? qb : qa) + (c & 1) * kQBox + h * 128 + (((u & 7) ^ (h & 7)) << 4);
        } else {
          src = ((h >> 6) ? qb : qa) + 2 * kQBox + hl * 64 + (((u - 32) ^ ((hl >> 1) & 3)) << 4);
        }
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (h < H) raw = *reinterpret_cast<const uint4*>(src);
        const uint4 v = FP16_SRC ? cvt_unit(raw) : raw;   // Q in the type of the gathered entries
        qv[4 * m + 0] = v.x;
        qv[4 * m + 1] = v.y;
        qv[4 * m + 2] = v.z;
        qv[4 * m + 3] = v.w;
      }
      const uint32_t qaddr = tmem + ((quarter * 32u) << 16) + TM_Q + 72 * g;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t t16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) t16[e] = qv[16 * c + e];
        tmem_st16(qaddr + 16 * c, t16);
      }
      {
        uint32_t t8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t8[e] = qv[64 + e];
        tmem_st8(qaddr + 64, t8);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->q_full);
      ++qn;
      return true;
    };

    cluster_wait();          // the peer's barriers exist: exchanges may start

    int G = 0, ring = 0, ke = 0;   // tiles, ring jobs, epilogues so far
    bool have_q = false;           // this item's Q slice is already in TMEM
    for (int k = 0; ok; ++k) {
      const int w = pair + k * n_pairs;
      if (w >= n_items) break;
      // the Q slice first: it needs no metadata (the first item's lands while
      // the producers are still staging its positions)
      if (item_has_q(p, w)) {
        if (!have_q && !convert_q(ring, k)) {
          ok = false;
          break;
        }
        ring += 2;
      }
      if (!wwait(&bar->meta_full[k & 1], (k >> 1) & 1, false, 336, k)) {
        ok = false;
        break;
      }
      // the item's metadata in registers: the buffer is restaged for item k + 2
      // once this warp's tile loop is over
      const ItemMeta it = meta[k & 1];
      const int n_tiles = (it.last + 1 + kTileKeys - 1) / kTileKeys;
      const uint32_t* sV = sValid + (k & 1) * 64;
      float m_runA = NEG_INF, m_runB = NEG_INF;   // running maxima (log2 domain), refreshed lazily
      float l_runA = 0.f, l_runB = 0.f;           // this lane's share of the row sums
      uint32_t cur[32];        // this CTA's fp32 partial scores of the current tile
      if (n_tiles > 0) {
        ok = load_s_issue(G, cur);
        if (ok) {
          load_s_finish();
          ok = send(G, cur);
        }
      }
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int gt = G + i;
        // 1. start loading the next tile's partial scores; they are shipped to
        //    the peer once this tile's scores are assembled
        const bool more = i + 1 < n_tiles;
        uint32_t snext[32];
        if (more && !load_s_issue(gt + 1, snext)) {
          ok = false;
          break;
        }
        // ... and release the S buffer as soon as the load has completed: the
        // MMA warp's Q.C^T of tile i+2 waits for it (releasing it after this
        // tile's maxima, to hide the load's latency, held that Q.C^T back by
        // ~1K cycles per tile)
        if (more) load_s_finish();
        // 2. the peer's partial scores of tile i (this warp's own barrier)
        if (lane == 0) mbar_arrive_expect_tx(&bar->x_full[sw], XBLK);
        if (!wwait(&bar->x_full[sw], gt & 1, true, 332, gt)) {
          ok = false;
          break;
        }
        uint32_t xp[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(xp[4 * q]), "=r"(xp[4 * q + 1]), "=r"(xp[4 * q + 2]), "=r"(xp[4 * q + 3])
                       : "r"(x_base + q * 512 + lane * 16)
                       : "memory");
        }
        // own + peer partial in fp32 (f32x2 pairs; each lane the IEEE fp32 add):
        // the peer computes peer + own, the same sum
        float sv[32];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float2 v = unpack_f32x2(add_f32x2(pack_f32x2(__uint_as_float(cur[2 * c]), __uint_as_float(cur[2 * c + 1])),
                                                  pack_f32x2(__uint_as_float(xp[2 * c]), __uint_as_float(xp[2 * c + 1]))));
          sv[2 * c] = v.x;
          sv[2 * c + 1] = v.y;
        }
        __syncwarp();
        // the values are in registers: the peer may refill the buffer
        if (lane == 0) mbar_arrive_remote_relaxed(x_free_remote);
        // 3. mask positions past the selection / padding: key 8k + ku + e
        const uint64_t vmask = static_cast<uint64_t>(sV[2 * i]) | (static_cast<uint64_t>(sV[2 * i + 1]) << 32);
        if (vmask != ~uint64_t(0)) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              if (!((vmask >> (8 * kk + ku + e)) & 1u)) {
                sv[4 * kk + e] = NEG_INF;
                sv[4 * kk + 2 + e] = NEG_INF;
              }
            }
          }
        }
        // 4. row maxima over the 64 columns: 16 per lane, then the lane group
        float mA = fmaxf(sv[0], sv[1]), mB = fmaxf(sv[2], sv[3]);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk) {
          mA = fmaxf(mA, fmaxf(sv[4 * kk], sv[4 * kk + 1]));
          mB = fmaxf(mB, fmaxf(sv[4 * kk + 2], sv[4 * kk + 3]));
        }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, o));
          mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, o));
        }
        float alphaA = 1.f, alphaB = 1.f;
        bool grow = false;
        {
          const float nA = fmaxf(m_runA, mA * scale), nB = fmaxf(m_runB, mB * scale);
          if (nA > m_runA + 8.0f) {                      // true on the first finite tile
            alphaA = fast_exp2(m_runA - nA);             // exp2(-inf) = 0
            m_runA = nA;
            grow = true;
          }
          if (nB > m_runB + 8.0f) {
            alphaB = fast_exp2(m_runB - nB);
            m_runB = nB;
            grow = true;
          }
        }
        const float refA = m_runA == NEG_INF ? 0.f : m_runA;
        const float refB = m_runB == NEG_INF ? 0.f : m_runB;
        // next tile's partial scores to the peer
        if (more) {
          if (!send(gt + 1, snext)) {
            ok = false;
            break;
          }
        }
        // 5. probabilities (fp16 pairs, in the .16x128b order of P's columns) and row sums
        // (exponent arguments and row sums on f32x2 pairs: half the FMA/add
        // instructions; each lane is the fp32 operation of the scalar form)
        uint32_t pk[16];
        const uint64_t sc2 = pack_f32x2(scale, scale);
        const uint64_t nA2 = pack_f32x2(-refA, -refA), nB2 = pack_f32x2(-refB, -refB);
        uint64_t sA2 = 0ull, sB2 = 0ull;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const float2 xa = unpack_f32x2(fma_f32x2(pack_f32x2(sv[4 * kk], sv[4 * kk + 1]), sc2, nA2));
          const float2 xb = unpack_f32x2(fma_f32x2(pack_f32x2(sv[4 * kk + 2], sv[4 * kk + 3]), sc2, nB2));
          const float a0 = fast_exp2(xa.x), a1 = fast_exp2(xa.y);
          const float b0 = fast_exp2(xb.x), b1 = fast_exp2(xb.y);
          sA2 = add_f32x2(sA2, pack_f32x2(a0, a1));
          sB2 = add_f32x2(sB2, pack_f32x2(b0, b1));
          pk[2 * kk] = pack_half2(a0, a1);
          pk[2 * kk + 1] = pack_half2(b0, b1);
        }
        const float2 sa = unpack_f32x2(sA2), sb = unpack_f32x2(sB2);
        l_runA = l_runA * alphaA + (sa.x + sa.y);
        l_runB = l_runB * alphaB + (sb.x + sb.y);
        // 6. PV(i-1) must be done before P and O are touched (the previous
        //    item's last P.V was waited for by its epilogue)
        if (i > 0 && !wwait(&bar->pv_done, (gt - 1) & 1, false, 333, gt)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (i > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld_16x256b_x8(tbase + TM_O + 64 * c, o);
            tmem_ld_wait();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              o[4 * kk] = __float_as_uint(__uint_as_float(o[4 * kk]) * alphaA);
              o[4 * kk + 1] = __float_as_uint(__uint_as_float(o[4 * kk + 1]) * alphaA);
              o[4 * kk + 2] = __float_as_uint(__uint_as_float(o[4 * kk + 2]) * alphaB);
              o[4 * kk + 3] = __float_as_uint(__uint_as_float(o[4 * kk + 3]) * alphaB);
            }
            tmem_st_16x256b_x8(tbase + TM_O + 64 * c, o);
          }
        }
        tmem_st_16x128b_x8(tbase + TM_P, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->p_full);
#pragma unroll
        for (int c = 0; c < 32; ++c) cur[c] = snext[c];
      }
      if (!ok) break;
      // the validity bits of this parity may be restaged (item k + 2)
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->meta_free[k & 1]);
      ring += n_tiles;
      // The next item's Q slice into TMEM now -- every Q.C^T issued so far has
      // completed (this warp loaded its scores) -- so that item's first Q.C^T
      // runs during this epilogue.
      have_q = false;
      if (w + n_pairs < n_items && item_has_q(p, w + n_pairs)) {
        if (!convert_q(ring, k + 1)) {
          ok = false;
          break;
        }
        have_q = true;
      }

      // ---- epilogue: O / l -> bf16 (or fp32 partial).  An item without
      // tiles -- a row whose selection holds no usable entry, or whose
      // sequence is invalid (301) or absent (302) -- writes out = 0, lse =
      // -inf (split partials: lse = -inf, which the merge turns into the
      // same), so no stale partial of an earlier call is ever merged ----
      {
        if (n_tiles > 0 && !wwait(&bar->pv_done, (G + n_tiles - 1) & 1, false, 335, G + n_tiles)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float lA = l_runA, lB = l_runB;
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          lA += __shfl_xor_sync(0xffffffffu, lA, o);
          lB += __shfl_xor_sync(0xffffffffu, lB, o);
        }
        const bool anyA = n_tiles > 0 && lA > 0.f, anyB = n_tiles > 0 && lB > 0.f;
        const float invA = anyA ? 1.f / lA : 0.f, invB = anyB ? 1.f / lB : 0.f;
        const float lseA = anyA ? (m_runA + __log2f(lA)) * 0.69314718055994531f : NEG_INF;
        const float lseB = anyB ? (m_runB + __log2f(lB)) * 0.69314718055994531f : NEG_INF;
        if (p.nsplit == 1) {
          // Each lane stores whole 64-byte runs of one head: the inverse row
          // sums go through shared memory to the .32x32b layout (lane = head),
          // the two warps of a lane quarter taking 128 value dims each.
          float* inv_s = sInv + (ke & 1) * 128;
          if ((lane & 3u) == 0) {
            inv_s[hA] = invA;
            inv_s[hB] = invB;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar->red);
          if (!wwait(&bar->red, ke & 1, false, 339, ke)) {
            ok = false;
            break;
          }
          // This warp's 4 KB staging block transposes the stores: our last
          // bulk copy out of it has been read once the peer arrived on x_free
          // for the last tile we sent.
          const int t_last = G + n_tiles - 1;
          if (t_last >= 0 && !wwait(&bar->x_free[sw], t_last & 1, true, 334, t_last)) {
            ok = false;
            break;
          }
          const int h = static_cast<int>(quarter * 32 + lane);
          const float inv = inv_s[h];
          const int cb = 128 * (sw >> 2);   // this warp's 128 of the CTA's 256 value dims
          // row r of the block: head 32q + r, 64 dims = 8 units, unit u at (u ^ (r & 7)) * 16
          const uint32_t blk = stg_base;
          uint16_t* obase = p.out + (static_cast<int64_t>(it.row) * H + quarter * 32) * 512 + rank * 256 + cb;
#pragma unroll 1
          for (int j = 0; j < 2; ++j) {
            uint32_t o0[32], o1[32];
            if (n_tiles > 0) {
              tmem_ld32(tmem + ((quarter * 32u) << 16) + TM_O + cb + 64 * j, o0);
              tmem_ld32(tmem + ((quarter * 32u) << 16) + TM_O + cb + 64 * j + 32, o1);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) o0[e] = o1[e] = 0u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              uint32_t wv[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = 8 * (u & 3) + 2 * e;   // column pair inside o0 (u < 4) or o1
                const float x0 = __uint_as_float(u < 4 ? o0[c] : o1[c]) * inv;
                const float x1 = __uint_as_float(u < 4 ? o0[c + 1] : o1[c + 1]) * inv;
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
                wv[e] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(blk + lane * 128 + ((u ^ (lane & 7)) << 4)),
                           "r"(wv[0]), "r"(wv[1]), "r"(wv[2]), "r"(wv[3])
                           : "memory");
            }
            __syncwarp();
            // eight lanes per head row: each store instruction writes four whole 128-byte runs
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 4 * i + static_cast<int>(lane >> 3), uu = static_cast<int>(lane & 7u);
              uint4 val;
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                           : "r"(blk + r * 128 + ((uu ^ (r & 7)) << 4))
                           : "memory");
              if (static_cast<int>(quarter) * 32 + r < H)
                *reinterpret_cast<uint4*>(obase + static_cast<int64_t>(r) * 512 + 64 * j + 8 * uu) = val;
            }
            __syncwarp();
          }
          if (rank == 0 && (lane & 3u) == 0 && p.lse != nullptr) {
            if (hA < H) p.lse[static_cast<int64_t>(it.row) * H + hA] = lseA;
            if (hB < H) p.lse[static_cast<int64_t>(it.row) * H + hB] = lseB;
          }
          ++ke;
        } else {
          const int64_t prow = (static_cast<int64_t>(it.row) * p.nsplit + it.split) * 128;
          float* oA = p.part_o + (prow + hA) * 512 + rank * 256 + ku;
          float* oB = p.part_o + (prow + hB) * 512 + rank * 256 + ku;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            if (n_tiles > 0) {
              tmem_ld_16x256b_x8(tbase + TM_O + 64 * c, o);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = 0u;
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              *reinterpret_cast<float2*>(oA + 64 * c + 8 * kk) =
                  make_float2(__uint_as_float(o[4 * kk]) * invA, __uint_as_float(o[4 * kk + 1]) * invA);
              *reinterpret_cast<float2*>(oB + 64 * c + 8 * kk) =
                  make_float2(__uint_as_float(o[4 * kk + 2]) * invB, __uint_as_float(o[4 * kk + 3]) * invB);
            }
          }
          if ((lane & 3u) == 0) {        // each value half with its own log-sum-exp
            p.part_lse[(prow * 2 + rank * 128) + hA] = lseA;
            p.part_lse[(prow * 2 + rank * 128) + hB] = lseB;
          }
        }
      }
      G += n_tiles;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // the peer no longer touches our shared memory
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// bf16 -> fp16 copy of the latent cache (saturating, exact in the normal range).
__global__ void __launch_bounds__(256) latent_to_fp16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                             int64_t n_units) {
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n_units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    dst[u] = cvt_unit(__ldg(&src[u]));
  }
}

// Merge the per-split partial outputs of each token: weights exp(lse_s - lse).
__global__ void __launch_bounds__(256) mla_combine_kernel(const MlaParams p) {
  const int row = blockIdx.x;
  const int H = p.n_heads;
  const int S = p.nsplit;
  for (int u = blockIdx.y * blockDim.x + threadIdx.x; u < H * 128; u += blockDim.x * gridDim.y) {
    const int h = u >> 7, d4 = u & 127;
    // dims [4 d4, 4 d4 + 4) belong to value half d4 / 64, which has its own lse
    const float* lse_s = p.part_lse + (static_cast<int64_t>(row) * S * 2 + (d4 >> 6)) * 128 + h;
    float m = __int_as_float(0xff800000);
    for (int s = 0; s < S; ++s) m = fmaxf(m, lse_s[s * 256]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (m != __int_as_float(0xff800000)) {
      for (int s = 0; s < S; ++s) {
        const float w = __expf(lse_s[s * 256] - m);
        wsum += w;
        const float4 o = reinterpret_cast<const float4*>(
            p.part_o + ((static_cast<int64_t>(row) * S + s) * 128 + h) * 512)[d4];
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    const __nv_bfloat162 v0 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    const __nv_bfloat162 v1 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t*>(&v0);
    packed.y = *reinterpret_cast<const uint32_t*>(&v1);
    *reinterpret_cast<uint2*>(p.out + (static_cast<int64_t>(row) * H + h) * 512 + d4 * 4) = packed;
    if (d4 == 0 && p.lse != nullptr) {
      p.lse[static_cast<int64_t>(row) * H + h] = wsum > 0.f ? m + __logf(wsum) : __int_as_float(0xff800000);
    }
  }
}

// CTA pairs of the kernel that can be resident at once on this device (an
// occupancy query, cached per device and variant): a persistent pair that
// waited for a free slot would start after the others had finished.
template <bool FP16_SRC>
int resident_pairs() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v != 0) return v - 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(kSmem);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, sparse_mla_kernel<FP16_SRC>, &cfg) != cudaSuccess) n = 0;
  cudaGetLastError();   // a refused query leaves no sticky error behind
  cache[dev].store(n + 1, std::memory_order_relaxed);
  return n;
}

template <bool FP16_SRC>
cudaError_t launch_variant(const MlaParams& p, const MlaMaps& maps, cudaStream_t stream) {
  const int64_t items = static_cast<int64_t>(p.total_q) * p.nsplit;
  if (items <= 0) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(sparse_mla_kernel<FP16_SRC>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  int pairs = resident_pairs<FP16_SRC>();
  if (pairs < 1) pairs = sm_count() / 2;
  if (pairs < 1) pairs = 1;
  const int cap = mla_pair_cap();
  if (cap > 0 && cap < pairs) pairs = cap;
  if (items < pairs) pairs = static_cast<int>(items);
  sparse_mla_kernel<FP16_SRC><<<dim3(static_cast<unsigned>(2 * pairs)), Cfg::THREADS, kSmem, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace

int mla_num_splits(int total_q, int max_q_per_seq, int num_seqs, int k_sel) {
  // A token's selection is split over several CTA pairs while the doubled
  // number of pairs still fits one wave (74 pairs on 148 SMs) and every split
  // keeps >= 8 tiles: one pair per token leaves most SMs idle on small
  // batches, and a split's fixed cost (prologue/epilogue ~17K cycles, about
  // five tiles, plus the log-sum-exp merge) is far below the idle time it
  // recovers (measured, 32-tile selections: 16 tokens at 32K context 83 us
  // unsplit vs 44 us in four splits; 8 x 2 tokens at 128K 82 vs 42 us; 64
  // tokens stay unsplit: 91 us vs 216 us in four splits over two waves).
  (void)max_q_per_seq;
  (void)num_seqs;
  const int max_tiles = (k_sel + kTileKeys - 1) / kTileKeys;
  int s = 1;
  while (s * 2 <= max_tiles / 8 && static_cast<int64_t>(total_q) * s * 2 * 2 <= 148) s *= 2;
  return s;
}

int mla_keys_per_split(int k_sel, int nsplit) {
  const int tiles = (k_sel + kTileKeys - 1) / kTileKeys;
  return ((tiles + nsplit - 1) / nsplit) * kTileKeys;
}

bool mla_use_fp16_copy(int total_q, int max_kv_len, int64_t total_keys, int k_sel) {
  // the copy reads and writes every cache row once; worth it when each row is
  // gathered about 8 times or more
  const int64_t gathers = static_cast<int64_t>(total_q) * (k_sel < max_kv_len ? k_sel : max_kv_len);
  return gathers >= 8 * total_keys;
}

size_t mla_smem_bytes() { return kSmem; }

cudaError_t launch_sparse_mla(const MlaParams& p, const MlaMaps& maps, cudaStream_t stream) {
  return launch_variant<false>(p, maps, stream);
}

cudaError_t launch_sparse_mla_fp16(const MlaParams& p, const MlaMaps& maps, cudaStream_t stream) {
  return launch_variant<true>(p, maps, stream);
}

cudaError_t launch_latent_to_fp16(const uint16_t* src, uint16_t* dst, int64_t n_elems, cudaStream_t stream) {
  const int64_t units = n_elems / 8;
  latent_to_fp16_kernel<<<148 * 8, 256, 0, stream>>>(reinterpret_cast<const uint4*>(src),
                                                     reinterpret_cast<uint4*>(dst), units);
  return cudaGetLastError();
}

cudaError_t launch_mla_combine(int total_q, const MlaParams& p, cudaStream_t stream) {
  // 64 CTAs per token: few tokens, many SMs, one unit of (head, 4 dims) per thread
  mla_combine_kernel<<<dim3(total_q, 64), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dsa
