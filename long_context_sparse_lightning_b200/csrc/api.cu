// C ABI of the DSA hot path: argument validation, workspace carving, TMA
// descriptor encoding and kernel launches.  No allocation, no synchronisation
// (except dsa_check_device_error), no fallback path.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/dsa.h"
#include "kernels.cuh"

namespace {

using dsa::IndexerParams;
using dsa::wait_budget;
using dsa::MlaParams;
using dsa::TopkParams;

constexpr size_t kHeaderBytes = 256;      // device error word + reserved
constexpr long long kDefaultBudget = 2000000000LL;   // clock64 cycles per bounded wait (~1 s)

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }


// ---- cuTensorMapEncodeTiled through the runtime's driver entry point ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
    }
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] of `elem` bytes, box [box_rows, box_cols].
bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, size_t elem, uint64_t rows,
                  uint64_t cols, uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

dsa_status_t check_batch(const dsa_batch_t* b) {
  if (b == nullptr) return DSA_ERR_INVALID_ARG;
  if (b->num_seqs < 1 || b->num_seqs > 65535 || b->total_q < 0 || b->max_q_per_seq < 0 || b->max_kv_len < 0 ||
      b->total_keys < 0)
    return DSA_ERR_INVALID_ARG;
  if (b->cu_q == nullptr || b->kv_len == nullptr) return DSA_ERR_INVALID_ARG;
  if (b->block_table == nullptr) {
    if (b->kv_start == nullptr) return DSA_ERR_INVALID_ARG;
  } else {
    // pages of a multiple of 64 rows (the key tiles load as 64-row halves), a
    // table row long enough for the longest sequence, a whole number of pages
    if (b->page_size < 64 || (b->page_size % 64) != 0 || b->blocks_per_seq < 1) return DSA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(b->blocks_per_seq) * b->page_size < b->max_kv_len) return DSA_ERR_INVALID_ARG;
    if (b->total_keys % b->page_size != 0) return DSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(b->block_table) & 3u) != 0) return DSA_ERR_INVALID_ARG;
  }
  if (b->total_q > 0 && (b->max_q_per_seq < 1 || b->max_kv_len < b->max_q_per_seq || b->total_keys < 1))
    return DSA_ERR_INVALID_ARG;
  if (b->max_q_per_seq > b->total_q || static_cast<int64_t>(b->max_kv_len) > b->total_keys)
    return DSA_ERR_INVALID_ARG;
  if (b->total_keys >= (int64_t(1) << 31) || static_cast<int64_t>(b->total_q) * 128 >= (int64_t(1) << 31))
    return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

dsa::PageTable page_table(const dsa_batch_t* b) {
  dsa::PageTable pt;
  if (b->block_table != nullptr) {
    pt.table = b->block_table;
    pt.page = b->page_size;
    pt.stride = b->blocks_per_seq;
    pt.num_pages = static_cast<int32_t>(b->total_keys / b->page_size);
  }
  return pt;
}

// key-tile box height of the indexer's key-cache descriptor: whole 128-key
// tiles (flat) or 64-row halves, one per page run (paged)
uint32_t k_box_rows(const dsa_batch_t* b) { return b->block_table != nullptr ? 64 : 128; }

dsa_status_t check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || !aligned16(ws)) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < need) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

int64_t forward_ld(const dsa_batch_t* b) { return static_cast<int64_t>(align_up(b->max_kv_len, 4)); }

// the [total_q, ld] fp32 score matrix the unfused indexer -> top-k keeps in ws
size_t scores_bytes(const dsa_batch_t* b) {
  return align_up(static_cast<size_t>(b->total_q) * forward_ld(b) * sizeof(float), 256);
}

struct MlaSplit {
  int nsplit;
  int keys_per_split;
};
MlaSplit mla_split(const dsa_batch_t* b, int k_sel) {
  const int s = dsa::mla_num_splits(b->total_q, b->max_q_per_seq, b->num_seqs, k_sel);
  return {s, dsa::mla_keys_per_split(k_sel, s)};
}

size_t mla_part_bytes(const dsa_batch_t* b, int k_sel) {
  const MlaSplit sp = mla_split(b, k_sel);
  if (sp.nsplit <= 1) return 0;
  const size_t rows = static_cast<size_t>(b->total_q) * sp.nsplit * 128;
  return align_up(rows * 512 * sizeof(float), 256) + align_up(rows * 2 * sizeof(float), 256);
}

bool mla_copy(const dsa_batch_t* b, int k_sel) {
  return dsa::mla_use_fp16_copy(b->total_q, b->max_kv_len, b->total_keys, k_sel);
}

// partial results + (prefill-shaped batches) the fp16 copy of the latent cache
size_t mla_ws_bytes(const dsa_batch_t* b, int k_sel) {
  size_t n = mla_part_bytes(b, k_sel);
  if (mla_copy(b, k_sel)) n += align_up(static_cast<size_t>(b->total_keys) * 576 * 2, 256);
  return n;
}

// ----------------------------------------------------------------- stages --
dsa_status_t run_indexer(const dsa_batch_t* b, const void* q_fp8, const float* q_scale, const float* w,
                         const void* k_fp8, const float* k_scale, float* scores, int64_t ld, uint32_t* err,
                         cudaStream_t stream) {
  const int tok = dsa::indexer_tokens_per_cta(b->max_q_per_seq);
  CUtensorMap tq, tk;
  if (!make_tmap_2d(&tq, q_fp8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(b->total_q) * 64, 128,
                    dsa::indexer_box_rows_q(tok), 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tk, k_fp8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(b->total_keys), 128,
                    k_box_rows(b), 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  const int qblocks = (b->max_q_per_seq + tok - 1) / tok;
  if (qblocks > 65535) return DSA_ERR_UNSUPPORTED;
  const int tiles = (b->max_kv_len + 127) / 128;
  // CTAs to aim for (one per SM at a time): each CTA pays a fixed setup, so
  // few long chunks win when there are few tokens per CTA; measured best: ~4
  // waves with 8-token blocks (prefill), 2 with 1 token (decode), 1 with 2
  const int64_t waves = tok >= 8 ? 4 : (tok >= 4 ? 2 : (tok == 2 ? 1 : 2));
  const int64_t target = waves * 148;
  int tpc = tiles;
  while (tpc > 8 && static_cast<int64_t>(b->num_seqs) * qblocks * ((tiles + tpc - 1) / tpc) < target)
    tpc = (tpc + 1) / 2;
  IndexerParams p;
  p.cu_q = b->cu_q;
  p.kv_len = b->kv_len;
  p.kv_start = b->kv_start;
  p.q_scale = q_scale;
  p.w = w;
  p.k_scale = k_scale;
  p.scores = scores;
  p.ld = ld;
  p.total_keys = b->total_keys;
  p.tiles_per_chunk = tpc;
  p.num_qblocks = qblocks;
  p.err = err;
  p.budget = wait_budget();
  p.pt = page_table(b);
  p.skip_arrival = dsa::test_skip_arrival();
  const dim3 grid((tiles + tpc - 1) / tpc, qblocks, b->num_seqs);
  return dsa::launch_indexer(tok, grid, tq, tk, p, stream) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// The fused decode indexer + top-k applies (CTAs per cluster), or 0.
int fused_cluster(const dsa_batch_t* b) {
  return dsa::indexer_topk_cluster(b->max_q_per_seq, b->num_seqs, b->max_kv_len);
}

// dsa_forward takes the fused kernel (it applies and is the faster path).
bool forward_fused(const dsa_batch_t* b) {
  return dsa::indexer_topk_preferred(b->max_q_per_seq, b->num_seqs, fused_cluster(b));
}

dsa_status_t run_indexer_topk(const dsa_batch_t* b, const void* q_fp8, const float* q_scale, const float* w,
                              const void* k_fp8, const float* k_scale, int k_sel, int32_t* idx, uint32_t* err,
                              cudaStream_t stream) {
  const int tok = b->max_q_per_seq;     // 1 or 2
  const int cl = fused_cluster(b);
  if (cl < 1) return DSA_ERR_UNSUPPORTED;
  CUtensorMap tq, tk;
  if (!make_tmap_2d(&tq, q_fp8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(b->total_q) * 64, 128,
                    dsa::indexer_box_rows_q(tok), 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tk, k_fp8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(b->total_keys), 128,
                    k_box_rows(b), 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  dsa::IndexerTopkParams p;
  p.ix.cu_q = b->cu_q;
  p.ix.kv_len = b->kv_len;
  p.ix.kv_start = b->kv_start;
  p.ix.q_scale = q_scale;
  p.ix.w = w;
  p.ix.k_scale = k_scale;
  p.ix.scores = nullptr;
  p.ix.ld = 0;
  p.ix.total_keys = b->total_keys;
  p.ix.tiles_per_chunk = 0;
  p.ix.num_qblocks = 1;
  p.ix.err = err;
  p.ix.budget = wait_budget();
  p.ix.pt = page_table(b);
  p.k_sel = k_sel;
  p.idx = idx;
  p.max_kv_len = b->max_kv_len;
  const dim3 grid(static_cast<unsigned>(cl), 1, static_cast<unsigned>(b->num_seqs));
  return dsa::launch_indexer_topk(tok, cl, grid, tq, tk, p, stream) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// candidate buffers of the two-phase top-k (rows longer than 32768 positions)
size_t topk_ws_bytes(const dsa_batch_t* b, int k_sel) {
  const dsa::TopkSegments t = dsa::topk_segments(b->max_kv_len, k_sel, b->total_q);
  if (t.segs == 0) return 0;
  return 2 * align_up(static_cast<size_t>(b->total_q) * t.segs * k_sel * sizeof(float), 256);
}

dsa_status_t run_topk(const dsa_batch_t* b, const float* scores, int64_t ld, int k_sel, int32_t* idx,
                      uint8_t* seg, uint32_t* err, cudaStream_t stream) {
  TopkParams p;
  p.cu_q = b->cu_q;
  p.kv_len = b->kv_len;
  p.scores = scores;
  p.ld = ld;
  p.k_sel = k_sel;
  p.idx = idx;
  p.total_q = b->total_q;
  p.num_seqs = b->num_seqs;
  p.err = err;
  p.budget = wait_budget();
  const dsa::TopkSegments t = dsa::topk_segments(b->max_kv_len, k_sel, b->total_q);
  if (t.segs > 0) {
    const size_t half = align_up(static_cast<size_t>(b->total_q) * t.segs * k_sel * sizeof(float), 256);
    p.seg_pos = reinterpret_cast<int32_t*>(seg);
    p.seg_val = reinterpret_cast<float*>(seg + half);
    p.n_seg = t.segs;
    p.seg_len = t.len;
  }
  return dsa::launch_topk(b->max_kv_len, p, stream) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status_t run_mla(const dsa_batch_t* b, const void* q, int n_heads, const void* kv, const int32_t* idx,
                     int k_sel, float sm_scale, void* out, float* lse, uint8_t* part, uint32_t* err,
                     cudaStream_t stream) {
  const MlaSplit sp = mla_split(b, k_sel);
  MlaParams p;
  p.cu_q = b->cu_q;
  p.kv_len = b->kv_len;
  p.kv_start = b->kv_start;
  p.q = static_cast<const uint16_t*>(q);
  p.kv = static_cast<const uint16_t*>(kv);
  p.idx = idx;
  p.total_keys = b->total_keys;
  p.total_q = b->total_q;
  p.num_seqs = b->num_seqs;
  p.pt = page_table(b);
  p.k_sel = k_sel;
  p.n_heads = n_heads;
  p.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.nsplit = sp.nsplit;
  p.keys_per_split = sp.keys_per_split;
  p.part_o = nullptr;
  p.part_lse = nullptr;
  if (sp.nsplit > 1) {
    const size_t rows = static_cast<size_t>(b->total_q) * sp.nsplit * 128;
    p.part_o = reinterpret_cast<float*>(part);
    p.part_lse = reinterpret_cast<float*>(part + align_up(rows * 512 * sizeof(float), 256));
  }
  p.err = err;
  p.budget = wait_budget();
  if (static_cast<int64_t>(b->total_q) * sp.nsplit >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  dsa::MlaMaps maps;
  if (!dsa::make_mla_maps(&maps, q, b->total_q, n_heads)) return DSA_ERR_CUDA;
  if (mla_copy(b, k_sel)) {
    uint16_t* kv16 = reinterpret_cast<uint16_t*>(part + mla_part_bytes(b, k_sel));
    const int64_t n = b->total_keys * 576;
    if (dsa::launch_latent_to_fp16(static_cast<const uint16_t*>(kv), kv16, n, stream) != cudaSuccess)
      return DSA_ERR_CUDA;
    p.kv = kv16;
    if (dsa::launch_sparse_mla_fp16(p, maps, stream) != cudaSuccess) return DSA_ERR_CUDA;
  } else if (dsa::launch_sparse_mla(p, maps, stream) != cudaSuccess) {
    return DSA_ERR_CUDA;
  }
  if (sp.nsplit > 1 && dsa::launch_mla_combine(b->total_q, p, stream) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t check_indexer_args(const dsa_batch_t* b, const void* q_fp8, const float* q_scale, const float* w,
                                const void* k_fp8, const float* k_scale) {
  if (q_fp8 == nullptr || q_scale == nullptr || w == nullptr || k_fp8 == nullptr || k_scale == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp8) || !aligned16(k_fp8) || !aligned16(q_scale) || !aligned16(w)) return DSA_ERR_INVALID_ARG;
  (void)b;
  return DSA_OK;
}

dsa_status_t check_mla_args(const void* q, int n_heads, const void* kv, int k_sel, float sm_scale, void* out) {
  if (q == nullptr || kv == nullptr || out == nullptr) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return DSA_ERR_INVALID_ARG;
  if (n_heads < 1 || n_heads > 128) return DSA_ERR_UNSUPPORTED;
  if (k_sel < 1 || k_sel > DSA_MAX_K_SEL) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

}  // namespace

namespace dsa {
dsa_status_t validate_batch(const dsa_batch_t* b) { return check_batch(b); }

int test_skip_arrival() {
  const char* s = std::getenv("DSA_TEST_SKIP_ARRIVAL");
  if (s == nullptr || *s == '\0') return -1;
  const long v = std::atol(s);
  return v >= 0 && v < (1L << 30) ? static_cast<int>(v) : -1;
}
PageTable batch_pages(const dsa_batch_t* b) { return page_table(b); }

int mla_pair_cap() {
  const char* s = std::getenv("DSA_MLA_MAX_PAIRS");
  if (s == nullptr || *s == '\0') return 0;
  const long v = std::atol(s);
  return v > 0 && v < (1L << 20) ? static_cast<int>(v) : 0;
}

long long wait_budget() {
  const char* s = std::getenv("DSA_WAIT_BUDGET_CYCLES");
  if (s != nullptr) {
    const long long v = std::atoll(s);
    if (v > 0) return v;
  }
  return kDefaultBudget;
}

bool make_mla_maps(MlaMaps* m, const void* q, int64_t total_q, int n_heads) {
  const uint64_t rows = static_cast<uint64_t>(total_q) * static_cast<uint64_t>(n_heads);
  const uint32_t h = static_cast<uint32_t>(n_heads);
  const uint32_t rope_rows = h < 64 ? h : 64;   // RoPE rows 0-63 and 64-127 travel in separate ring stages
  return make_tmap_2d(&m->q_lat, q, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, rows, 576, h, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_tmap_2d(&m->q_rope, q, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, rows, 576, rope_rows, 32,
                      CU_TENSOR_MAP_SWIZZLE_64B);
}
}  // namespace dsa

extern "C" {

size_t dsa_workspace_size(dsa_op_t op, const dsa_batch_t* batch, int32_t k_sel, int32_t n_heads) {
  if (check_batch(batch) != DSA_OK) return 0;
  switch (op) {
    case DSA_OP_INDEXER:
      return kHeaderBytes;
    case DSA_OP_TOPK:
      if (k_sel < 1 || k_sel > DSA_MAX_K_SEL) return 0;
      return kHeaderBytes + topk_ws_bytes(batch, k_sel);
    case DSA_OP_SPARSE_MLA:
      if (k_sel < 1 || k_sel > DSA_MAX_K_SEL || n_heads < 1 || n_heads > 128) return 0;
      return kHeaderBytes + mla_ws_bytes(batch, k_sel);
    case DSA_OP_CACHE_WRITE:
      return kHeaderBytes;
    case DSA_OP_INDEXER_TOPK:
      if (k_sel < 1 || k_sel > DSA_MAX_K_SEL) return 0;
      if (fused_cluster(batch) > 0) return kHeaderBytes;
      return kHeaderBytes + scores_bytes(batch) + topk_ws_bytes(batch, k_sel);
    case DSA_OP_FORWARD: {
      if (k_sel < 1 || k_sel > DSA_MAX_K_SEL || n_heads < 1 || n_heads > 128) return 0;
      if (forward_fused(batch)) return kHeaderBytes + mla_ws_bytes(batch, k_sel);
      // the top-k candidates and the MLA buffers are used one after the other
      return kHeaderBytes + scores_bytes(batch) + std::max(mla_ws_bytes(batch, k_sel), topk_ws_bytes(batch, k_sel));
    }
  }
  return 0;
}

dsa_status_t dsa_indexer_scores(const dsa_batch_t* batch, const void* q_fp8, const float* q_scale, const float* w,
                                const void* k_fp8, const float* k_scale, float* scores, int64_t ld_scores, void* ws,
                                size_t ws_bytes, dsa_stream_t stream) {
  dsa_status_t s = check_batch(batch);
  if (s != DSA_OK) return s;
  if ((s = check_indexer_args(batch, q_fp8, q_scale, w, k_fp8, k_scale)) != DSA_OK) return s;
  if (scores == nullptr || !aligned16(scores) || ld_scores < batch->max_kv_len || (ld_scores & 3) != 0)
    return DSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, kHeaderBytes)) != DSA_OK) return s;
  if (batch->total_q == 0) return DSA_OK;
  return run_indexer(batch, q_fp8, q_scale, w, k_fp8, k_scale, scores, ld_scores, static_cast<uint32_t*>(ws),
                     reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_topk(const dsa_batch_t* batch, const float* scores, int64_t ld_scores, int32_t k_sel, int32_t* idx,
                      void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status_t s = check_batch(batch);
  if (s != DSA_OK) return s;
  if (scores == nullptr || idx == nullptr || !aligned16(scores) || ld_scores < batch->max_kv_len ||
      (ld_scores & 3) != 0)
    return DSA_ERR_INVALID_ARG;
  if (k_sel < 1 || k_sel > DSA_MAX_K_SEL) return DSA_ERR_UNSUPPORTED;
  if ((s = check_ws(ws, ws_bytes, kHeaderBytes + topk_ws_bytes(batch, k_sel))) != DSA_OK) return s;
  if (batch->total_q == 0) return DSA_OK;
  return run_topk(batch, scores, ld_scores, k_sel, idx, static_cast<uint8_t*>(ws) + kHeaderBytes,
                  static_cast<uint32_t*>(ws), reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_sparse_mla(const dsa_batch_t* batch, const void* q, int32_t n_heads, const void* kv,
                            const int32_t* idx, int32_t k_sel, float sm_scale, void* out, float* lse, void* ws,
                            size_t ws_bytes, dsa_stream_t stream) {
  dsa_status_t s = check_batch(batch);
  if (s != DSA_OK) return s;
  if ((s = check_mla_args(q, n_heads, kv, k_sel, sm_scale, out)) != DSA_OK) return s;
  if (idx == nullptr) return DSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, kHeaderBytes + mla_ws_bytes(batch, k_sel))) != DSA_OK) return s;
  if (batch->total_q == 0) return DSA_OK;
  return run_mla(batch, q, n_heads, kv, idx, k_sel, sm_scale, out, lse, static_cast<uint8_t*>(ws) + kHeaderBytes,
                 static_cast<uint32_t*>(ws), reinterpret_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_forward(const dsa_batch_t* batch, const void* q_fp8, const float* q_scale, const float* w,
                         const void* k_fp8, const float* k_scale, int32_t k_sel, const void* q, int32_t n_heads,
                         const void* kv, float sm_scale, int32_t* idx, void* out, float* lse, void* ws,
                         size_t ws_bytes, dsa_stream_t stream) {
  dsa_status_t s = check_batch(batch);
  if (s != DSA_OK) return s;
  if ((s = check_indexer_args(batch, q_fp8, q_scale, w, k_fp8, k_scale)) != DSA_OK) return s;
  if ((s = check_mla_args(q, n_heads, kv, k_sel, sm_scale, out)) != DSA_OK) return s;
  if (idx == nullptr) return DSA_ERR_INVALID_ARG;
  const size_t need = dsa_workspace_size(DSA_OP_FORWARD, batch, k_sel, n_heads);
  if ((s = check_ws(ws, ws_bytes, need)) != DSA_OK) return s;
  if (batch->total_q == 0) return DSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  uint8_t* part;
  if (forward_fused(batch)) {              // decode: scores stay on chip
    part = base + kHeaderBytes;
    if ((s = run_indexer_topk(batch, q_fp8, q_scale, w, k_fp8, k_scale, k_sel, idx, err, st)) != DSA_OK) return s;
  } else {
    const int64_t ld = forward_ld(batch);
    float* scores = reinterpret_cast<float*>(base + kHeaderBytes);
    part = base + kHeaderBytes + scores_bytes(batch);
    if ((s = run_indexer(batch, q_fp8, q_scale, w, k_fp8, k_scale, scores, ld, err, st)) != DSA_OK) return s;
    if ((s = run_topk(batch, scores, ld, k_sel, idx, part, err, st)) != DSA_OK) return s;
  }
  return run_mla(batch, q, n_heads, kv, idx, k_sel, sm_scale, out, lse, part, err, st);
}

dsa_status_t dsa_indexer_topk(const dsa_batch_t* batch, const void* q_fp8, const float* q_scale, const float* w,
                              const void* k_fp8, const float* k_scale, int32_t k_sel, int32_t* idx, void* ws,
                              size_t ws_bytes, dsa_stream_t stream) {
  dsa_status_t s = check_batch(batch);
  if (s != DSA_OK) return s;
  if ((s = check_indexer_args(batch, q_fp8, q_scale, w, k_fp8, k_scale)) != DSA_OK) return s;
  if (idx == nullptr) return DSA_ERR_INVALID_ARG;
  if (k_sel < 1 || k_sel > DSA_MAX_K_SEL) return DSA_ERR_UNSUPPORTED;
  const size_t need = dsa_workspace_size(DSA_OP_INDEXER_TOPK, batch, k_sel, 1);
  if ((s = check_ws(ws, ws_bytes, need)) != DSA_OK) return s;
  if (batch->total_q == 0) return DSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  if (fused_cluster(batch) > 0)
    return run_indexer_topk(batch, q_fp8, q_scale, w, k_fp8, k_scale, k_sel, idx, err, st);
  const int64_t ld = forward_ld(batch);
  float* scores = reinterpret_cast<float*>(base + kHeaderBytes);
  if ((s = run_indexer(batch, q_fp8, q_scale, w, k_fp8, k_scale, scores, ld, err, st)) != DSA_OK) return s;
  return run_topk(batch, scores, ld, k_sel, idx, base + kHeaderBytes + scores_bytes(batch), err, st);
}

dsa_status_t dsa_topk_candidates(const dsa_batch_t* batch, const float* scores, int64_t ld_scores, int32_t k_sel,
                                 const int32_t* pos_offset, int32_t* cand_pos, float* cand_val, void* ws,
                                 size_t ws_bytes, dsa_stream_t stream) {
  dsa_status_t s = check_batch(batch);
  if (s != DSA_OK) return s;
  if (scores == nullptr || cand_pos == nullptr || cand_val == nullptr || !aligned16(scores) ||
      ld_scores < batch->max_kv_len || (ld_scores & 3) != 0)
    return DSA_ERR_INVALID_ARG;
  if (pos_offset != nullptr && (reinterpret_cast<uintptr_t>(pos_offset) & 3u) != 0) return DSA_ERR_INVALID_ARG;
  if (k_sel < 1 || k_sel > DSA_MAX_K_SEL) return DSA_ERR_UNSUPPORTED;
  if ((s = check_ws(ws, ws_bytes, kHeaderBytes + topk_ws_bytes(batch, k_sel))) != DSA_OK) return s;
  if (batch->total_q == 0) return DSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((s = run_topk(batch, scores, ld_scores, k_sel, cand_pos, static_cast<uint8_t*>(ws) + kHeaderBytes,
                    static_cast<uint32_t*>(ws), st)) != DSA_OK)
    return s;
  dsa::TopkParams p;
  p.cu_q = batch->cu_q;
  p.kv_len = batch->kv_len;
  p.scores = scores;
  p.ld = ld_scores;
  p.k_sel = k_sel;
  p.idx = cand_pos;
  p.total_q = batch->total_q;
  p.num_seqs = batch->num_seqs;
  p.err = static_cast<uint32_t*>(ws);
  p.budget = wait_budget();
  return dsa::launch_topk_values(p, pos_offset, cand_val, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status_t dsa_topk_merge(int32_t n_rows, int32_t n_src, int32_t k_sel, const int32_t* cand_pos,
                            const float* cand_val, int32_t* idx, dsa_stream_t stream) {
  if (n_rows < 0 || n_src < 1 || cand_pos == nullptr || cand_val == nullptr || idx == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(cand_pos) || !aligned16(cand_val)) return DSA_ERR_INVALID_ARG;
  if (k_sel < 1 || k_sel > DSA_MAX_K_SEL) return DSA_ERR_UNSUPPORTED;
  const int64_t m = static_cast<int64_t>(n_src) * k_sel;
  if (m > 32768 || (m & 3) != 0) return DSA_ERR_UNSUPPORTED;
  if (n_rows == 0) return DSA_OK;
  return dsa::launch_topk_merge_sources(n_rows, n_src, k_sel, cand_pos, cand_val, idx,
                                        reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DSA_OK
             : DSA_ERR_CUDA;
}

int32_t dsa_forward_launches(const dsa_batch_t* batch, int32_t k_sel, int32_t n_heads) {
  if (check_batch(batch) != DSA_OK) return 0;
  if (k_sel < 1 || k_sel > DSA_MAX_K_SEL || n_heads < 1 || n_heads > 128) return 0;
  if (batch->total_q == 0) return 0;
  int32_t n = 1;                                                             // indexer (fused: + top-k)
  if (!forward_fused(batch)) n += dsa::topk_segments(batch->max_kv_len, k_sel, batch->total_q).segs > 0 ? 2 : 1;
  if (mla_copy(batch, k_sel)) n += 1;                                        // fp16 latent copy
  n += 1;                                                                    // sparse MLA
  if (mla_split(batch, k_sel).nsplit > 1) n += 1;                            // merge
  return n;
}

dsa_status_t dsa_quantize_fp8(const void* x, int64_t n_vec, void* codes, float* scales, dsa_stream_t stream) {
  if (n_vec < 0 || x == nullptr || codes == nullptr || scales == nullptr) return DSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return DSA_ERR_INVALID_ARG;
  if (n_vec >= (int64_t(1) << 40)) return DSA_ERR_UNSUPPORTED;
  if (n_vec == 0) return DSA_OK;
  return dsa::launch_quantize_fp8(x, n_vec, codes, scales, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DSA_OK
             : DSA_ERR_CUDA;
}

dsa_status_t dsa_indexer_prep(const void* x, int64_t n_vec, int32_t vecs_per_pos, const int32_t* pos,
                              const float* rope_cos, const float* rope_sin, int32_t n_pos, void* codes, float* scales,
                              void* ws, size_t ws_bytes, dsa_stream_t stream) {
  if (n_vec < 0 || vecs_per_pos < 1 || n_pos < 1 || x == nullptr || pos == nullptr || rope_cos == nullptr ||
      rope_sin == nullptr || codes == nullptr || scales == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(rope_cos) || !aligned16(rope_sin) ||
      (reinterpret_cast<uintptr_t>(pos) & 3u) != 0 || n_vec % vecs_per_pos != 0)
    return DSA_ERR_INVALID_ARG;
  if (n_vec >= (int64_t(1) << 40)) return DSA_ERR_UNSUPPORTED;
  dsa_status_t s;
  if ((s = check_ws(ws, ws_bytes, kHeaderBytes)) != DSA_OK) return s;
  if (n_vec == 0) return DSA_OK;
  return dsa::launch_indexer_prep(x, n_vec, vecs_per_pos, pos, rope_cos, rope_sin, n_pos, codes, scales,
                                  static_cast<uint32_t*>(ws), reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DSA_OK
             : DSA_ERR_CUDA;
}

dsa_status_t dsa_cache_write(const dsa_batch_t* batch, const void* k, const void* latent, void* k_cache,
                             float* k_scale, void* latent_cache, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status_t s = check_batch(batch);
  if (s != DSA_OK) return s;
  if (k == nullptr || latent == nullptr || k_cache == nullptr || k_scale == nullptr || latent_cache == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(latent) || !aligned16(k_cache) || !aligned16(k_scale) || !aligned16(latent_cache))
    return DSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, kHeaderBytes)) != DSA_OK) return s;
  if (batch->total_q == 0) return DSA_OK;
  return dsa::launch_cache_write(batch->num_seqs, batch->max_q_per_seq, batch->total_q, batch->total_keys,
                                 batch->cu_q, batch->kv_len, batch->kv_start, page_table(batch), k, latent, k_cache,
                                 k_scale, latent_cache, static_cast<uint32_t*>(ws),
                                 reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? DSA_OK
             : DSA_ERR_CUDA;
}

dsa_status_t dsa_check_device_error(void* ws, dsa_stream_t stream, uint32_t* site, uint32_t* info) {
  if (ws == nullptr) return DSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  uint32_t word[4] = {0, 0, 0, 0};
  if (cudaMemcpy(word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (word[0] != 0) {
    if (cudaMemset(ws, 0, sizeof(word)) != cudaSuccess) return DSA_ERR_CUDA;
  }
  if (site != nullptr) *site = word[1];
  if (info != nullptr) *info = word[2];
  switch (word[0]) {
    case 0: return DSA_OK;
    case DSA_ERR_DEVICE_TIMEOUT: return DSA_ERR_DEVICE_TIMEOUT;
    case DSA_ERR_DEVICE_BOUNDS: return DSA_ERR_DEVICE_BOUNDS;
    default: return DSA_ERR_CUDA;
  }
}

const char* dsa_status_string(dsa_status_t status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case DSA_ERR_DEVICE_BOUNDS: return "device index out of range";
  }
  return "unknown status";
}

int32_t dsa_version(void) { return 200; }

}  // extern "C"
