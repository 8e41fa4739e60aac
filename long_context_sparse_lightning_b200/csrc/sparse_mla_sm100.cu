// Sparse MLA in MQA mode on sm_100a (tcgen05, TMEM accumulators, a CTA pair
// per query token).
//
// "DeepSeek V3.2 稀疏注意力" (embedding DSA in MLA) and "NSA 与 DSA" §3.1: all
// query heads of a token share the same selected latent entries c_s (576-d =
// 512 latent + 64 RoPE; the value is the first 512 dims), so one gathered
// tile of entries feeds every head:
//     o[h] = sum_i softmax_i(sm_scale * q[h] . c[s_i]) * c[s_i][0:512].
//
// Layout of the work: a cluster of two CTAs handles one token (or one split of
// its selected entries).  CTA r owns latent dims [256r, 256r+256) and RoPE
// dims [512+32r, 512+32r+32) -- 288 of the 576 score dims and 256 of the 512
// value dims -- so the 128 x 512 fp32 output accumulator is split 256 TMEM
// columns per CTA and every latent byte is gathered exactly once per pair.
// Per tile of 64 selected entries:
//   producers (6 warps)  gather this CTA's 288 dims of each selected row with
//                        16-byte loads, convert bf16 -> fp16 (exact for the
//                        normal fp16 range) and store them 128/64-byte
//                        swizzled; the same tile serves QK^T as a K-major B
//                        operand and PV as an MN-major B operand;
//   MMA warp             S_r = Q_r . C_r^T (M=128 heads, N=64, K=288, fp16 in,
//                        fp32 in TMEM), later O_r += P . V_r (N=256);
//   softmax (4 warps)    thread h owns head h: exchanges its 64 partial scores
//                        with the partner CTA through distributed shared memory,
//                        adds them (both CTAs get bit-identical S), runs the
//                        online softmax in the log2 domain with a lazily
//                        refreshed running max (rescale of O only when the max
//                        grows by more than 2^8), writes P as fp16.
// P is fp16 rather than bf16: with bf16 probabilities the rounding noise alone
// costs ~1e-3 mean relative error on the bf16 output; fp16 keeps it ~1e-4.
//
// Decode shapes split a token's selection over several pairs; each writes a
// normalised partial output and its log-sum-exp, merged by mla_combine_kernel.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kProdWarps = 6;
constexpr int kProdThreads = kProdWarps * 32;
constexpr int kMmaWarp = kProdWarps;              // warp 8
constexpr int kThreads = (kProdWarps + 1 + 4) * 32;
constexpr int kTileKeys = 64;
constexpr int kUnitsPerRow = 36;                  // 16-byte units per gathered row half (288 dims)
constexpr int kTileUnits = kTileKeys * kUnitsPerRow;
constexpr int kUnitsPerThread = kTileUnits / kProdThreads;   // 9
static_assert(kTileUnits % kProdThreads == 0, "");
constexpr int kQUnits = 128 * kUnitsPerRow;
constexpr int kQUnitsPerThread = kQUnits / kProdThreads;     // 18

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int OFF_Q = 0;                 // 4 x [128 x 128 B] SW128 + [128 x 64 B] SW64
constexpr int Q_ROPE = 65536;
constexpr int OFF_KV = 73728;            // 2 stages x 36864
constexpr int KV_STAGE = 36864;
constexpr int KV_ROPE = 32768;
constexpr int OFF_P = OFF_KV + 2 * KV_STAGE;     // 147456: 2 x [128 x 128 B] SW128 fp16
constexpr int P_BYTES = 16384;
constexpr int OFF_X = OFF_P + 2 * P_BYTES;       // 180224: incoming partial S, 128 rows x 272 B
constexpr int X_PITCH = 272;
constexpr int OFF_IDX = OFF_X + 128 * X_PITCH;   // 215040
constexpr int OFF_BAR = OFF_IDX + 2048 * 4;      // 223232
constexpr int OFF_MISC = OFF_BAR + 128;
constexpr int kSmem = OFF_MISC + 64 + 1024;
constexpr uint32_t kTmemCols = 512;              // O: cols [0,256), S: [256,384)

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t x_full;
  uint64_t x_free;
  uint64_t p_full[2];
  uint64_t pv_done[2];
};
static_assert(sizeof(Bars) <= 128, "");

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

// smem offset (within a 288-dim row group) of 16-byte unit u of row j:
// units 0..31 = latent dims (4 chunks of 8 units, 128-byte swizzle),
// units 32..35 = RoPE dims (64-byte swizzle).
__device__ __forceinline__ uint32_t tile_unit_offset(int j, int u, int chunk_bytes, int rope_off) {
  if (u < 32) {
    const int c = u >> 3, cu = u & 7;
    return c * chunk_bytes + j * 128 + ((cu ^ (j & 7)) << 4);
  }
  const int ru = u - 32;
  return rope_off + j * 64 + ((ru ^ ((j >> 1) & 3)) << 4);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1) sparse_mla_kernel(const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;

  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int tok = pair / p.nsplit;
  const int split = pair % p.nsplit;
  const int b = blockIdx.y;
  const int q0 = __ldg(&p.cu_q[b]);
  const int q_len = __ldg(&p.cu_q[b + 1]) - q0;
  // Every early exit below depends only on launch indices and device inputs
  // that do not change during the kernel, so both CTAs of a pair take it
  // together; a one-sided exit would leave the partner in barrier.cluster.
  if (tok >= q_len) return;
  const int row = q0 + tok;
  const int kv = __ldg(&p.kv_len[b]);
  const int64_t kstart = __ldg(&p.kv_start[b]);
  if (q_len > kv || kstart < 0 || kstart + kv > p.total_keys) {
    if (threadIdx.x == 0 && rank == 0) report_error(p.err, kDevErrBounds, 301, b);
    return;                             // both CTAs of the pair take this branch
  }
  const int H = p.n_heads;
  const int e_begin = split * p.keys_per_split;
  const int e_count = max(0, min(p.k_sel, e_begin + p.keys_per_split) - e_begin);

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = sm + OFF_Q;
  uint8_t* sKV = sm + OFF_KV;
  uint8_t* sP = sm + OFF_P;
  float* sX = reinterpret_cast<float*>(sm + OFF_X);
  int32_t* sIdx = reinterpret_cast<int32_t*>(sm + OFF_IDX);
  Bars* bar = reinterpret_cast<Bars*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  int32_t* s_last = reinterpret_cast<int32_t*>(sm + OFF_MISC + 4);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int tid = threadIdx.x;

  // ---- selected positions of this split; invalid ones become -1 ----
  if (tid == 0) *s_last = -1;
  __syncthreads();
  const int32_t* idx_row = p.idx + static_cast<int64_t>(row) * p.k_sel + e_begin;
  int my_last = -1;
  for (int j = tid; j < 2048; j += kThreads) {
    int v = -1;
    if (j < e_count) {
      v = __ldg(&idx_row[j]);
      if (v < 0 || v >= kv) v = -1;
    }
    sIdx[j] = v;
    if (v >= 0) my_last = j;
  }
  if (my_last >= 0) atomicMax(s_last, my_last);

  if (tid == 0) {
    mbar_init(&bar->q_full, kProdWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->kv_full[i], kProdWarps);
      mbar_init(&bar->kv_empty[i], 1);
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->s_empty[i], 4);
    }
    mbar_init(&bar->x_full, 128);
    mbar_init(&bar->x_free, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->p_full[i], 128);
      mbar_init(&bar->pv_done[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_ent = *s_last + 1;
  const int n_tiles = (n_ent + kTileKeys - 1) / kTileKeys;

  if (warp < kProdWarps) {
    // ------------------------------------------ gather + convert producers --
    if (n_tiles > 0) {
      // Q_r: this token's 128 head rows (rows >= H are zero)
      {
        const uint16_t* qrow = p.q + static_cast<int64_t>(row) * H * 576;
#pragma unroll 4
        for (int m = 0; m < kQUnitsPerThread; ++m) {
          const int g = tid + m * kProdThreads;
          const int h = g / kUnitsPerRow, u = g % kUnitsPerRow;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (h < H) {
            const int dim = u < 32 ? static_cast<int>(rank) * 256 + u * 8 : 512 + static_cast<int>(rank) * 32 + (u - 32) * 8;
            v = cvt_unit(__ldg(reinterpret_cast<const uint4*>(qrow + h * 576 + dim)));
          }
          *reinterpret_cast<uint4*>(sQ + tile_unit_offset(h, u, 16384, Q_ROPE)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->q_full);
      }
      const uint16_t* kvbase = p.kv + kstart * 576;
      uint4 bufA[kUnitsPerThread], bufB[kUnitsPerThread];
      auto issue = [&](int tile, uint4 (&buf)[kUnitsPerThread]) {
#pragma unroll
        for (int m = 0; m < kUnitsPerThread; ++m) {
          const int g = tid + m * kProdThreads;
          const int j = g / kUnitsPerRow, u = g % kUnitsPerRow;
          const int s = sIdx[tile * kTileKeys + j];
          const int pos = s >= 0 ? s : 0;
          const int dim = u < 32 ? static_cast<int>(rank) * 256 + u * 8 : 512 + static_cast<int>(rank) * 32 + (u - 32) * 8;
          buf[m] = __ldg(reinterpret_cast<const uint4*>(kvbase + static_cast<int64_t>(pos) * 576 + dim));
        }
      };
      bool ok = true;
      auto commit = [&](int tile, const uint4 (&buf)[kUnitsPerThread]) {
        const int st = tile & 1;
        if (ok && !mbar_wait(&bar->kv_empty[st], ((tile >> 1) & 1) ^ 1, p.budget)) {
          report_error(p.err, kDevErrTimeout, 310, tile);
          ok = false;
        }
        if (!ok) return;
        uint8_t* base = sKV + st * KV_STAGE;
#pragma unroll
        for (int m = 0; m < kUnitsPerThread; ++m) {
          const int g = tid + m * kProdThreads;
          const int j = g / kUnitsPerRow, u = g % kUnitsPerRow;
          *reinterpret_cast<uint4*>(base + tile_unit_offset(j, u, 8192, KV_ROPE)) = cvt_unit(buf[m]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->kv_full[st]);
      };
      issue(0, bufA);
      for (int i = 0; i < n_tiles && ok; i += 2) {
        if (i + 1 < n_tiles) issue(i + 1, bufB);
        commit(i, bufA);
        if (i + 1 < n_tiles) {
          if (i + 2 < n_tiles) issue(i + 2, bufA);
          commit(i + 1, bufB);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------- MMA issuer --
    if (n_tiles > 0 && elect_one()) {
      constexpr uint32_t idesc_qk = idesc_f32acc(0, 0, 128, 64, 0, 0);     // fp16 x fp16, K-major both
      constexpr uint32_t idesc_pv = idesc_f32acc(0, 0, 128, 256, 0, 1);    // P K-major, V MN-major
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t p_addr = smem_u32(sP);
      bool ok = mbar_wait(&bar->q_full, 0, p.budget);
      if (!ok) report_error(p.err, kDevErrTimeout, 320, 0);
      for (int i = 0; ok && i <= n_tiles; ++i) {
        if (i < n_tiles) {
          const int st = i & 1;
          if (!mbar_wait(&bar->kv_full[st], (i >> 1) & 1, p.budget) ||
              !mbar_wait(&bar->s_empty[st], ((i >> 1) & 1) ^ 1, p.budget)) {
            report_error(p.err, kDevErrTimeout, 321, i);
            break;
          }
          tc_fence_after();
          const uint32_t kv_addr = smem_u32(sKV + st * KV_STAGE);
          const uint32_t tS = tmem + 256 + st * 64;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              umma_bf16(tS, smem_desc(q_addr + c * 16384 + k * 32, 16, 1024, kSwizzle128B),
                        smem_desc(kv_addr + c * 8192 + k * 32, 16, 1024, kSwizzle128B), idesc_qk,
                        (c | k) ? 1u : 0u);
            }
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            umma_bf16(tS, smem_desc(q_addr + Q_ROPE + k * 32, 16, 512, kSwizzle64B),
                      smem_desc(kv_addr + KV_ROPE + k * 32, 16, 512, kSwizzle64B), idesc_qk, 1u);
          }
          umma_commit(&bar->s_full[st]);
        }
        if (i >= 1) {
          const int j = i - 1;
          const int st = j & 1;
          if (!mbar_wait(&bar->p_full[st], (j >> 1) & 1, p.budget)) {
            report_error(p.err, kDevErrTimeout, 322, j);
            break;
          }
          tc_fence_after();
          const uint32_t kv_addr = smem_u32(sKV + st * KV_STAGE);
          const uint32_t pb_addr = p_addr + st * P_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            umma_bf16(tmem, smem_desc(pb_addr + k * 32, 16, 1024, kSwizzle128B),
                      smem_desc(kv_addr + k * 2048, 8192, 1024, kSwizzle128B), idesc_pv, (j | k) ? 1u : 0u);
          }
          umma_commit(&bar->pv_done[st]);
          umma_commit(&bar->kv_empty[st]);
        }
      }
    }
  } else {
    // ------------------------------------------------ softmax warpgroup --
    const uint32_t quarter = warp & 3u;
    const int h = static_cast<int>(quarter * 32 + lane);
    const uint32_t lane_addr = (quarter * 32u) << 16;
    const uint32_t x_local = smem_u32(sX) + h * X_PITCH;
    const uint32_t x_remote = mapa_shared(x_local, peer);
    const uint32_t x_full_remote = mapa_shared(smem_u32(&bar->x_full), peer);
    const uint32_t x_free_remote = mapa_shared(smem_u32(&bar->x_free), peer);
    const float NEG_INF = __int_as_float(0xff800000);
    float m_run = NEG_INF;    // running max (log2 domain), refreshed lazily
    float l_run = 0.f;
    bool ok = true;
    // bounded wait whose outcome is the same for every lane of the warp
    auto wwait = [&](uint64_t* b_, uint32_t parity, bool cluster, uint32_t site, int info) -> bool {
      const bool r = cluster ? mbar_wait_cluster(b_, parity, p.budget) : mbar_wait(b_, parity, p.budget);
      if (!r) report_error(p.err, kDevErrTimeout, site, info);
      return __all_sync(0xffffffffu, r);
    };
    for (int i = 0; ok && i < n_tiles; ++i) {
      const int st = i & 1;
      // 1. this CTA's partial scores for head h
      if (!wwait(&bar->s_full[st], (i >> 1) & 1, false, 330, i)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sa[32], sb[32];
      tmem_ld32(tmem + lane_addr + 256 + st * 64, sa);
      tmem_ld32(tmem + lane_addr + 256 + st * 64 + 32, sb);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->s_empty[st]);
      // 2. send them to the partner, 3. receive the partner's
      if (!wwait(&bar->x_free, (i & 1) ^ 1, true, 331, i)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        st_cluster_v4(x_remote + q * 16, __uint_as_float(sa[4 * q]), __uint_as_float(sa[4 * q + 1]),
                      __uint_as_float(sa[4 * q + 2]), __uint_as_float(sa[4 * q + 3]));
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        st_cluster_v4(x_remote + 128 + q * 16, __uint_as_float(sb[4 * q]), __uint_as_float(sb[4 * q + 1]),
                      __uint_as_float(sb[4 * q + 2]), __uint_as_float(sb[4 * q + 3]));
      }
      mbar_arrive_remote(x_full_remote);
      if (!wwait(&bar->x_full, i & 1, true, 332, i)) {
        ok = false;
        break;
      }
      const float4* xr = reinterpret_cast<const float4*>(reinterpret_cast<const uint8_t*>(sX) + h * X_PITCH);
      const int* tidx = sIdx + i * kTileKeys;
      float mz = NEG_INF;
      // own + peer partial scores (the peer adds them in the other order: fp add
      // commutes, so both CTAs hold bit-identical S), masked, in log2 units
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 x = xr[q];
        uint32_t* src = q < 8 ? &sa[4 * q] : &sb[4 * (q - 8)];
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float zz = tidx[4 * q + e] >= 0 ? (__uint_as_float(src[e]) + xs[e]) * p.scale_log2 : NEG_INF;
          src[e] = __float_as_uint(zz);
          mz = fmaxf(mz, zz);
        }
      }
      mbar_arrive_remote(x_free_remote);   // our buffer may be refilled by the peer
      const float m_new = fmaxf(m_run, mz);
      const bool grow = m_new > m_run + 8.0f;         // true on the first finite tile
      float alpha = 1.f;
      if (grow) {
        alpha = fast_exp2(m_run - m_new);              // exp2(-inf) = 0
        m_run = m_new;
      }
      const float m_ref = m_run == NEG_INF ? 0.f : m_run;
      // P buffer (i & 1) is free once PV(i - 2) finished
      if (i >= 2 && !wwait(&bar->pv_done[st], ((i - 2) >> 1) & 1, false, 333, i)) {
        ok = false;
        break;
      }
      // O may only be rescaled between PV(i - 1) and PV(i)
      if (i > 0 && __any_sync(0xffffffffu, grow)) {
        if (!wwait(&bar->pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, false, 334, i)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_addr + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(tmem + lane_addr + c * 32, o);
        }
        tmem_st_wait();
      }
      // P row h: fp16, 64 keys = 128 bytes, 128-byte swizzle
      uint8_t* prow = sP + st * P_BYTES + h * 128;
      float rs = 0.f;
#pragma unroll
      for (int cu = 0; cu < 8; ++cu) {
        const uint32_t* src = cu < 4 ? &sa[8 * cu] : &sb[8 * (cu - 4)];
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pa = fast_exp2(__uint_as_float(src[2 * e]) - m_ref);
          const float pb = fast_exp2(__uint_as_float(src[2 * e + 1]) - m_ref);
          rs += pa + pb;
          const __half2 hv = __floats2half2_rn(pa, pb);
          w4[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(prow + ((cu ^ (h & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      l_run = l_run * alpha + rs;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar->p_full[st]);
    }
    // ---- epilogue: O / l -> bf16 (or fp32 partial) ----
    if (ok && n_tiles > 0 && !wwait(&bar->pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, false, 335, n_tiles)) {
      ok = false;
    }
    tc_fence_after();
    const float inv_l = (n_tiles > 0 && l_run > 0.f) ? 1.f / l_run : 0.f;
    const float lse_val = (n_tiles > 0 && l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : NEG_INF;
    if (p.nsplit == 1) {
      uint16_t* orow = p.out + (static_cast<int64_t>(row) * H + h) * 512 + rank * 256;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        if (n_tiles > 0) {
          tmem_ld32(tmem + lane_addr + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
        if (h < H) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[8 * q + 2 * e]) * inv_l,
                                                             __uint_as_float(o[8 * q + 2 * e + 1]) * inv_l);
              w4[e] = *reinterpret_cast<const uint32_t*>(&v);
            }
            *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      if (rank == 0 && h < H && p.lse != nullptr) p.lse[static_cast<int64_t>(row) * H + h] = lse_val;
    } else {
      const int64_t prow_i = (static_cast<int64_t>(row) * p.nsplit + split) * 128 + h;
      float* orow = p.part_o + prow_i * 512 + rank * 256;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        if (n_tiles > 0) {
          tmem_ld32(tmem + lane_addr + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          *reinterpret_cast<float4*>(orow + c * 32 + q * 4) =
              make_float4(__uint_as_float(o[4 * q]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                          __uint_as_float(o[4 * q + 2]) * inv_l, __uint_as_float(o[4 * q + 3]) * inv_l);
        }
      }
      if (rank == 0) p.part_lse[prow_i] = lse_val;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();          // the peer no longer touches our shared memory
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the per-split partial outputs of each token: weights exp(lse_s - lse).
__global__ void __launch_bounds__(256) mla_combine_kernel(const MlaParams p) {
  const int row = blockIdx.x;
  const int H = p.n_heads;
  const int S = p.nsplit;
  for (int u = threadIdx.x; u < H * 128; u += blockDim.x) {
    const int h = u >> 7, d4 = u & 127;
    const float* lse_s = p.part_lse + (static_cast<int64_t>(row) * S) * 128 + h;
    float m = __int_as_float(0xff800000);
    for (int s = 0; s < S; ++s) m = fmaxf(m, lse_s[s * 128]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (m != __int_as_float(0xff800000)) {
      for (int s = 0; s < S; ++s) {
        const float w = __expf(lse_s[s * 128] - m);
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

}  // namespace

int mla_num_splits(int total_q, int max_q_per_seq, int num_seqs, int k_sel) {
  // fill ~2 waves of CTA pairs (74 pairs per wave on 148 SMs); keep >= 4 tiles per split
  (void)max_q_per_seq;
  (void)num_seqs;
  const int max_tiles = (k_sel + kTileKeys - 1) / kTileKeys;
  int s = 1;
  while (s * 2 <= max_tiles / 4 && static_cast<int64_t>(total_q) * s < 148) s *= 2;
  return s;
}

int mla_keys_per_split(int k_sel, int nsplit) {
  const int tiles = (k_sel + kTileKeys - 1) / kTileKeys;
  return ((tiles + nsplit - 1) / nsplit) * kTileKeys;
}

size_t mla_smem_bytes() { return kSmem; }

cudaError_t launch_sparse_mla(dim3 grid, const MlaParams& p, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  sparse_mla_kernel<<<grid, kThreads, kSmem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_mla_combine(int total_q, const MlaParams& p, cudaStream_t stream) {
  mla_combine_kernel<<<total_q, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dsa
