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
// Per token, around the tile loop: the CTA's Q slice arrives by TMA boxes into
// ring stages 2-3 (converted to fp16 into TMEM by the softmax warps before the
// producers reuse those stages), and the bf16 output leaves by TMA box stores
// staged, swizzled, in the idle ring.
//
// Decode shapes split a token's selection over several pairs; each writes a
// normalised partial output and its log-sum-exp, merged by mla_combine_kernel.
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
constexpr int OFF_VALID = OFF_IDX + 2048 * 4;        // 221184: uint32[64] validity bits
constexpr int OFF_BAR = OFF_VALID + 64 * 4;          // 221440
constexpr int OFF_MISC = OFF_BAR + 512;
constexpr int kSmem = OFF_MISC + 64 + 1024;

constexpr int kUnitsPerRow = 36;                     // 16-byte units of a row's 288-dim half
constexpr int kTileUnits = kTileKeys * kUnitsPerRow; // 2304
constexpr int kQBox = 16384;                         // one 128-row x 128-byte TMA box of Q or O

struct Bars {
  uint64_t q_tma;           // this CTA's Q slice landed in shared memory (TMA)
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t qk_done[kStages];   // bf16 source: Q.C^T of the stage's tile has read it (MMA commit)
  uint64_t v_full[kStages];    // bf16 source: the stage's value part converted to fp16 in place
  uint64_t s_full, s_empty;
  uint64_t x_full[8], x_free[8];   // per softmax warp: peer's partial landed / peer has read ours
  uint64_t p_full, pv_done;
  uint64_t red;            // all softmax warps have staged the output
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
static_assert(2048 % Cfg::THREADS == 0, "index staging assumes whole warps per pass");
static_assert(4 * kQBox + 128 * 64 <= 2 * KV_STAGE, "Q slice must fit ring stages 2-3");

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

// FP16_SRC: p.kv is an fp16 copy of the latent cache (rows land ready for the
// MMAs); otherwise p.kv is the bf16 cache: Q.C^T runs in bf16 and the producers
// convert the value part in place between Q.C^T and P.V.
template <bool FP16_SRC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg::THREADS, 1)
    sparse_mla_kernel(const MlaParams p, const __grid_constant__ MlaMaps maps) {
  using C = Cfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;

  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int tok = pair / p.nsplit;
  const int split = pair % p.nsplit;
  const int b = blockIdx.y;
  const int q0 = __ldg(&p.cu_q[b]);
  const int q_len = __ldg(&p.cu_q[b + 1]) - q0;
  // Every early exit depends only on launch indices and on device inputs that
  // do not change during the kernel, so both CTAs of a pair take it together
  // (a one-sided exit would leave the peer waiting in barrier.cluster).
  if (tok >= q_len) return;
  const int row = q0 + tok;
  const int H = p.n_heads;
  if (q0 < 0 || row >= p.total_q) {          // inconsistent cu_q: nothing of this row is written
    if (threadIdx.x == 0 && rank == 0) report_error(p.err, kDevErrBounds, 302, b);
    return;
  }
  const int kv = __ldg(&p.kv_len[b]);
  const int64_t kstart = seq_start(p.pt, p.kv_start, b);
  if (q_len > kv || !seq_rows_ok(p.pt, kstart, kv, p.total_keys)) {
    if (threadIdx.x == 0 && rank == 0) report_error(p.err, kDevErrBounds, 301, b);
    // The row attends to nothing: out = 0 and lse = -inf (split partials:
    // lse = -inf, which the merge turns into the same), so no stale partial
    // of an earlier call is ever merged into this row.
    const float NI = __int_as_float(0xff800000);
    if (p.nsplit == 1) {
      for (int u = threadIdx.x; u < H * 32; u += blockDim.x) {      // 32 16-byte units of this CTA's half
        const int h = u >> 5, c = u & 31;
        *reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(row) * H + h) * 512 + rank * 256 + c * 8) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      if (rank == 0 && p.lse != nullptr)
        for (int h = threadIdx.x; h < H; h += blockDim.x) p.lse[static_cast<int64_t>(row) * H + h] = NI;
    } else {
      const int64_t prow = (static_cast<int64_t>(row) * p.nsplit + split) * 128;
      for (int h = threadIdx.x; h < 128; h += blockDim.x) p.part_lse[prow * 2 + rank * 128 + h] = NI;
    }
    return;
  }
  const int e_begin = split * p.keys_per_split;
  const int e_count = max(0, min(p.k_sel, e_begin + p.keys_per_split) - e_begin);

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sKV = sm + OFF_KV;
  int32_t* sIdx = reinterpret_cast<int32_t*>(sm + OFF_IDX);
  uint32_t* sValid = reinterpret_cast<uint32_t*>(sm + OFF_VALID);
  Bars* bar = reinterpret_cast<Bars*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  int32_t* s_last = reinterpret_cast<int32_t*>(sm + OFF_MISC + 4);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int tid = threadIdx.x;

  // ---- this split's selected positions: loads first (one memory latency,
  // overlapping the set-up below) ----
  const int32_t* idx_row = p.idx + static_cast<int64_t>(row) * p.k_sel + e_begin;
  // (positions are checked against kv_len and mapped to cache rows below)
  constexpr int PER = (2048 + C::THREADS - 1) / C::THREADS;
  int v[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int j = tid + q * C::THREADS;
    v[q] = (j < 2048 && j < e_count) ? __ldg(&idx_row[j]) : -1;
  }

  // ---- barriers, then this CTA's Q slice by TMA into ring stages 2-3 (free
  // until the producers' third tile, which waits for q_full) ----
  uint8_t* sQ = sKV + 2 * KV_STAGE;
  if (tid == 0) {
    *s_last = -1;
    mbar_init(&bar->q_tma, 1);
    mbar_init(&bar->q_full, 8);
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
    mbar_init(&bar->red, 256);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar->q_tma, static_cast<uint32_t>(H) * (4 * 128 + 64));
#pragma unroll
    for (int c = 0; c < 4; ++c)
      tma_load_2d(sQ + c * kQBox, &maps.q_lat, &bar->q_tma, static_cast<int>(rank) * 256 + c * 64, row * H);
    tma_load_2d(sQ + 4 * kQBox, &maps.q_rope, &bar->q_tma, 512 + static_cast<int>(rank) * 32, row * H);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();

  // ---- each selected position -> its cache row (flat or paged), invalid -> -1,
  // per-32 validity bits, the last valid slot ----
  int my_last = -1;
  {
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int j = tid + q * C::THREADS;
      if (j < 2048) {
        int e = (v[q] < 0 || v[q] >= kv) ? -1 : v[q];
        if (e >= 0) {
          const int64_t r = cache_row(p.pt, b, kstart, e);
          if (r < 0) report_error(p.err, kDevErrBounds, 303, b);   // a page id outside the pool: skipped
          e = static_cast<int>(r);
        }
        sIdx[j] = e;
        const uint32_t bits = __ballot_sync(0xffffffffu, e >= 0);
        if (lane == 0) sValid[j >> 5] = bits;
        if (e >= 0) my_last = j;
      }
    }
  }
  if (my_last >= 0) atomicMax(s_last, my_last);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Our barriers are initialised: arrive on the cluster barrier now; each role
  // waits for the peer's arrival only before its first remote access (the
  // softmax warps' first score exchange) or at its end, so the set-up of
  // both CTAs overlaps the first gathers and the Q conversion.
  cluster_arrive();
  const uint32_t tmem = *tmem_slot;
  const int n_ent = *s_last + 1;
  const int n_tiles = (n_ent + kTileKeys - 1) / kTileKeys;

  if (warp < C::NPROD) {
    setmaxnreg_dec<C::REG_LOW>();
    // ------------------------------------------------------------ producers --
    // Each 16-byte unit goes straight to its swizzled slot with cp.async;
    // consecutive lanes take consecutive units of a row, so one warp request
    // covers a few whole 128-byte lines.  bf16 sources are converted to fp16 in
    // place by the thread that loaded them.
    if (n_tiles > 0) {
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
      // the tile's ring slot is free: P.V of the slot's previous tile has read
      // it, and stages 2-3 no longer hold the Q slice (the softmax warps have
      // moved it to TMEM)
      auto slot_free = [&](int tile) {
        const int st = tile % kStages;
        bool f = mbar_test(smem_u32(&bar->kv_empty[st]), ((tile / kStages) & 1) ^ 1);
        if (tile == 2 || tile == 3) f = f && mbar_test(smem_u32(&bar->q_full), 0);
        return __shfl_sync(0xffffffffu, f, 0);   // lane 0 decides for the warp
      };
      auto issue = [&](int tile) {
        const int st = tile % kStages;
        if (ok && !mbar_wait(&bar->kv_empty[st], ((tile / kStages) & 1) ^ 1, p.budget)) {
          report_error(p.err, kDevErrTimeout, 311, tile);
          ok = false;
        }
        if (ok && (tile == 2 || tile == 3) && !mbar_wait(&bar->q_full, 0, p.budget)) {
          report_error(p.err, kDevErrTimeout, 312, tile);
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          const uint32_t base = smem_u32(sKV + st * KV_STAGE);
          const int32_t* e = sIdx + tile * kTileKeys;
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
        if (lane == 0) mbar_arrive(&bar->kv_full[tile % kStages]);
      };
      // bf16 source: Q.C^T reads the tile as bf16 (exact products, like fp16);
      // once it has, the value part (units 0..31) becomes fp16 in place for
      // P.V, off the path from the gather to the scores
      auto convert = [&](int tile) {
        if constexpr (!FP16_SRC) {
          const int st = tile % kStages;
          if (ok && !mbar_wait(&bar->qk_done[st], (tile / kStages) & 1, p.budget)) {
            report_error(p.err, kDevErrTimeout, 313, tile);
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
        }
      };
      if constexpr (FP16_SRC) {
        // Up to three tiles in flight (copies committed, not yet landed).  A
        // warp blocks on a ring slot only when it has nothing left to land:
        // landing tile t lets Q.C^T(t) run, and the P.V that frees a slot
        // comes after Q.C^T of the newer tiles, so waiting for a slot while
        // holding an unlanded tile would hold up the scores of that tile
        // (3.62 -> 3.43 ms at 4096 queries of 32K context).
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
        // conversion of tile 0.)
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
      cp_async_wait<0>();
    }
    cluster_wait();
  } else if (warp == C::MMA_WARP) {
    setmaxnreg_dec<C::REG_LOW>();
    // ----------------------------------------------------------- MMA issuer --
    if (n_tiles > 0 && elect_one()) {
      // Q.C^T in the source's type (bf16 Q in TMEM for a bf16 cache), P.V in fp16
      constexpr uint32_t kQkFmt = FP16_SRC ? 0u : kFmtBF16;
      constexpr uint32_t idesc_qk = idesc_f32acc(kQkFmt, kQkFmt, 128, 64, 0, 0);   // K-major
      constexpr uint32_t idesc_pv = idesc_f32acc(0, 0, 128, 256, 0, 1);    // P K-major, V MN-major
      bool ok = mbar_wait(&bar->q_full, 0, p.budget);
      if (!ok) report_error(p.err, kDevErrTimeout, 320, 0);
      // QK^T runs two tiles ahead of PV: the softmax reads S(i+1) while it
      // still works on tile i, so S(i+2) can be computed meanwhile.
      for (int i = 0; ok && i < n_tiles + 2; ++i) {
        if (i < n_tiles) {
          const int st = i % kStages;
          if (!mbar_wait(&bar->kv_full[st], (i / kStages) & 1, p.budget) ||
              (i > 0 && !mbar_wait(&bar->s_empty, (i - 1) & 1, p.budget))) {
            report_error(p.err, kDevErrTimeout, 321, i);
            break;
          }
          tc_fence_after();
          const uint32_t kv_addr = smem_u32(sKV + st * KV_STAGE);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              umma_f16_ts(tmem + TM_S, tmem + TM_Q + c * 32 + k * 8,
                          smem_desc(kv_addr + c * 8192 + k * 32, 16, 1024, kSwizzle128B), idesc_qk,
                          (c | k) ? 1u : 0u);
            }
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            umma_f16_ts(tmem + TM_S, tmem + TM_Q + 128 + k * 8,
                        smem_desc(kv_addr + KV_ROPE + k * 32, 16, 512, kSwizzle64B), idesc_qk, 1u);
          }
          umma_commit(&bar->s_full);
          if constexpr (!FP16_SRC) umma_commit(&bar->qk_done[st]);
        }
        if (i >= 2) {
          const int j = i - 2;
          if (!mbar_wait(&bar->p_full, j & 1, p.budget)) {
            report_error(p.err, kDevErrTimeout, 322, j);
            break;
          }
          const int st = j % kStages;
          if (!FP16_SRC && !mbar_wait(&bar->v_full[st], (j / kStages) & 1, p.budget)) {
            report_error(p.err, kDevErrTimeout, 323, j);
            break;
          }
          tc_fence_after();
          const uint32_t kv_addr = smem_u32(sKV + st * KV_STAGE);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            umma_f16_ts(tmem + TM_O, tmem + TM_P + k * 8,
                        smem_desc(kv_addr + k * 2048, 8192, 1024, kSwizzle128B), idesc_pv, (j | k) ? 1u : 0u);
          }
          umma_commit(&bar->pv_done);
          umma_commit(&bar->kv_empty[st]);
        }
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
    float m_runA = NEG_INF, m_runB = NEG_INF;   // running maxima (log2 domain), refreshed lazily
    float l_runA = 0.f, l_runB = 0.f;           // this lane's share of the row sums
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
    // S(t) of this warp's 16 heads, this CTA's fp32 partial over its 288 dims:
    // s[4k], s[4k+1] = head rA, keys 8k+ku, 8k+ku+1; s[4k+2], s[4k+3] = head rB.
    // Split in two so the TMEM load's latency overlaps other work.
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

    // every softmax warp waits for the Q slice, also when there is nothing to
    // attend, so no TMA write is still in flight when the CTA exits
    if (!wwait(&bar->q_tma, 0, false, 338, 0)) ok = false;
    if (n_tiles > 0) {
      // Q_r row h into TMEM (shape .32x32b: lane = head): warps of the first
      // warpgroup write dims [0, 144) of the CTA's 288, the second [144, 288)
      const int g = sw >> 2;
      const int h = static_cast<int>(quarter * 32 + lane);
      uint32_t qv[72];
#pragma unroll
      for (int m = 0; m < 18; ++m) {
        const int u = 18 * g + m;        // unit of the CTA's 288 dims: 0..31 latent, 32..35 RoPE
        const uint32_t off = u < 32 ? (u >> 3) * kQBox + h * 128 + (((u & 7) ^ (h & 7)) << 4)
                                    : 4 * kQBox + h * 64 + (((u - 32) ^ ((h >> 1) & 3)) << 4);
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (ok && h < H) raw = *reinterpret_cast<const uint4*>(sQ + off);
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
    }
    cluster_wait();          // the peer's barriers exist: exchanges may start

    uint32_t cur[32];        // this CTA's fp32 partial scores of the current tile
    if (n_tiles > 0) {
      ok = ok && load_s_issue(0, cur);
      if (ok) {
        load_s_finish();
        ok = send(0, cur);
      }
    }
    for (int i = 0; ok && i < n_tiles; ++i) {
      // 1. start loading the next tile's partial scores; they are shipped to
      //    the peer once this tile's scores are assembled
      const bool more = i + 1 < n_tiles;
      uint32_t snext[32];
      if (more && !load_s_issue(i + 1, snext)) {
        ok = false;
        break;
      }
      // 2. the peer's partial scores of tile i (this warp's own barrier)
      if (lane == 0) mbar_arrive_expect_tx(&bar->x_full[sw], XBLK);
      if (!wwait(&bar->x_full[sw], i & 1, true, 332, i)) {
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
      const uint64_t vmask = static_cast<uint64_t>(sValid[2 * i]) | (static_cast<uint64_t>(sValid[2 * i + 1]) << 32);
      if (vmask != ~uint64_t(0)) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            if (!((vmask >> (8 * k + ku + e)) & 1u)) {
              sv[4 * k + e] = NEG_INF;
              sv[4 * k + 2 + e] = NEG_INF;
            }
          }
        }
      }
      // 4. row maxima over the 64 columns: 16 per lane, then the lane group
      float mA = fmaxf(sv[0], sv[1]), mB = fmaxf(sv[2], sv[3]);
#pragma unroll
      for (int k = 1; k < 8; ++k) {
        mA = fmaxf(mA, fmaxf(sv[4 * k], sv[4 * k + 1]));
        mB = fmaxf(mB, fmaxf(sv[4 * k + 2], sv[4 * k + 3]));
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
      // next tile's partial scores: wait for the TMEM load, ship
      if (more) {
        load_s_finish();
        if (!send(i + 1, snext)) {
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
      for (int k = 0; k < 8; ++k) {
        const float2 xa = unpack_f32x2(fma_f32x2(pack_f32x2(sv[4 * k], sv[4 * k + 1]), sc2, nA2));
        const float2 xb = unpack_f32x2(fma_f32x2(pack_f32x2(sv[4 * k + 2], sv[4 * k + 3]), sc2, nB2));
        const float a0 = fast_exp2(xa.x), a1 = fast_exp2(xa.y);
        const float b0 = fast_exp2(xb.x), b1 = fast_exp2(xb.y);
        sA2 = add_f32x2(sA2, pack_f32x2(a0, a1));
        sB2 = add_f32x2(sB2, pack_f32x2(b0, b1));
        pk[2 * k] = pack_half2(a0, a1);
        pk[2 * k + 1] = pack_half2(b0, b1);
      }
      const float2 sa = unpack_f32x2(sA2), sb = unpack_f32x2(sB2);
      l_runA = l_runA * alphaA + (sa.x + sa.y);
      l_runB = l_runB * alphaB + (sb.x + sb.y);
      // 6. PV(i-1) must be done before P and O are touched
      if (i > 0 && !wwait(&bar->pv_done, (i - 1) & 1, false, 333, i)) {
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
          for (int k = 0; k < 8; ++k) {
            o[4 * k] = __float_as_uint(__uint_as_float(o[4 * k]) * alphaA);
            o[4 * k + 1] = __float_as_uint(__uint_as_float(o[4 * k + 1]) * alphaA);
            o[4 * k + 2] = __float_as_uint(__uint_as_float(o[4 * k + 2]) * alphaB);
            o[4 * k + 3] = __float_as_uint(__uint_as_float(o[4 * k + 3]) * alphaB);
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

    // ---- epilogue: O / l -> bf16 (or fp32 partial) ----
    if (ok && n_tiles > 0 && !wwait(&bar->pv_done, (n_tiles - 1) & 1, false, 335, n_tiles)) ok = false;
    tc_fence_after();
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      l_runA += __shfl_xor_sync(0xffffffffu, l_runA, o);
      l_runB += __shfl_xor_sync(0xffffffffu, l_runB, o);
    }
    const bool anyA = n_tiles > 0 && l_runA > 0.f, anyB = n_tiles > 0 && l_runB > 0.f;
    const float invA = anyA ? 1.f / l_runA : 0.f, invB = anyB ? 1.f / l_runB : 0.f;
    const float lseA = anyA ? (m_runA + __log2f(l_runA)) * 0.69314718055994531f : NEG_INF;
    const float lseB = anyB ? (m_runB + __log2f(l_runB)) * 0.69314718055994531f : NEG_INF;
    // O chunk c (64 of the CTA's 256 value dims) of this warp's 16 heads
    auto load_o = [&](int c, uint32_t (&o)[32]) {
      if (n_tiles > 0) {
        tmem_ld_16x256b_x8(tbase + TM_O + 64 * c, o);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0u;
      }
    };
    if (p.nsplit == 1) {
      // O / l as bf16 into ring stages 0-1 (idle now) in the 128-byte-swizzled
      // layout of four [H x 64-dim] TMA boxes, then one thread stores the boxes:
      // whole rows leave the SM instead of pieces strided by a head row.
      uint8_t* sO = sKV;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        load_o(c, o);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          // dims 64c + 8k + ku, +1: box c, 16-byte unit k, byte 2*ku
          if (hA < H) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[4 * k]) * invA,
                                                           __uint_as_float(o[4 * k + 1]) * invA);
            *reinterpret_cast<__nv_bfloat162*>(sO + c * kQBox + hA * 128 + ((k ^ (hA & 7)) << 4) + 2 * ku) = v;
          }
          if (hB < H) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[4 * k + 2]) * invB,
                                                           __uint_as_float(o[4 * k + 3]) * invB);
            *reinterpret_cast<__nv_bfloat162*>(sO + c * kQBox + hB * 128 + ((k ^ (hB & 7)) << 4) + 2 * ku) = v;
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar->red);
      const bool staged = wwait(&bar->red, 0, false, 339, n_tiles);
      if (staged && sw == 0 && lane == 0) {
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          tma_store_2d(&maps.out, sO + bx * kQBox, static_cast<int>(rank) * 256 + bx * 64, row * H);
        bulk_commit_group();
        bulk_wait_read_all();    // the CTA may leave once the boxes are read
      }
      if (rank == 0 && (lane & 3u) == 0 && p.lse != nullptr) {
        if (hA < H) p.lse[static_cast<int64_t>(row) * H + hA] = lseA;
        if (hB < H) p.lse[static_cast<int64_t>(row) * H + hB] = lseB;
      }
    } else {
      const int64_t prow = (static_cast<int64_t>(row) * p.nsplit + split) * 128;
      float* oA = p.part_o + (prow + hA) * 512 + rank * 256 + ku;
      float* oB = p.part_o + (prow + hB) * 512 + rank * 256 + ku;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        load_o(c, o);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          *reinterpret_cast<float2*>(oA + 64 * c + 8 * k) =
              make_float2(__uint_as_float(o[4 * k]) * invA, __uint_as_float(o[4 * k + 1]) * invA);
          *reinterpret_cast<float2*>(oB + 64 * c + 8 * k) =
              make_float2(__uint_as_float(o[4 * k + 2]) * invB, __uint_as_float(o[4 * k + 3]) * invB);
        }
      }
      if ((lane & 3u) == 0) {        // each value half with its own log-sum-exp
        p.part_lse[(prow * 2 + rank * 128) + hA] = lseA;
        p.part_lse[(prow * 2 + rank * 128) + hB] = lseB;
      }
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

template <bool FP16_SRC>
cudaError_t launch_variant(dim3 grid, const MlaParams& p, const MlaMaps& maps, cudaStream_t stream) {
  cudaError_t e =
      cudaFuncSetAttribute(sparse_mla_kernel<FP16_SRC>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  sparse_mla_kernel<FP16_SRC><<<grid, Cfg::THREADS, kSmem, stream>>>(p, maps);
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

cudaError_t launch_sparse_mla(dim3 grid, const MlaParams& p, const MlaMaps& maps, cudaStream_t stream) {
  return launch_variant<false>(grid, p, maps, stream);
}

cudaError_t launch_sparse_mla_fp16(dim3 grid, const MlaParams& p, const MlaMaps& maps, cudaStream_t stream) {
  return launch_variant<true>(grid, p, maps, stream);
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
