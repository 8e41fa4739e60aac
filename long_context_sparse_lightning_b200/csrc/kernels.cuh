// Kernel parameter blocks and host-side launch entry points shared between
// the kernels' translation units and the C ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// SMs of the current device (queried once per device)
int sm_count();

// Flat or paged caches.  Flat (table == nullptr): position s of sequence b is
// row kv_start[b] + s.  Paged: row table[b * stride + s / page] * page +
// s % page of a pool of num_pages pages.
struct PageTable {
  const int32_t* table = nullptr;
  int32_t page = 0;        // rows per page, a multiple of 64
  int32_t stride = 0;      // entries per sequence in the table
  int32_t num_pages = 0;
};

// Host side, shared by the C ABI translation units: the batch descriptor's
// argument checks (DSA_OK or the status to return) and its page table.
dsa_status_t validate_batch(const dsa_batch_t* b);
PageTable batch_pages(const dsa_batch_t* b);
#ifdef __CUDACC__
// First cache row of sequence b (flat caches; 0 when paged, where kv_start
// may be null).
__device__ __forceinline__ int64_t seq_start(const PageTable& pt, const int64_t* kv_start, int b) {
  return pt.table == nullptr ? __ldg(&kv_start[b]) : 0;
}

// Every position 0 .. kv-1 of the sequence has a cache row: inside the flat
// cache, or inside the sequence's block-table row.
__device__ __forceinline__ bool seq_rows_ok(const PageTable& pt, int64_t kstart, int kv, int64_t total_keys) {
  if (pt.table == nullptr) return kstart >= 0 && kstart + kv <= total_keys;
  return static_cast<int64_t>(kv) <= static_cast<int64_t>(pt.stride) * pt.page;
}

// Cache row of position s (>= 0) of sequence b, or -1 when the page id in the
// block table is outside the pool.
__device__ __forceinline__ int64_t cache_row(const PageTable& pt, int b, int64_t kstart, int s) {
  if (pt.table == nullptr) return kstart + s;
  const int pg = __ldg(&pt.table[static_cast<int64_t>(b) * pt.stride + s / pt.page]);
  if (pg < 0 || pg >= pt.num_pages) return -1;
  return static_cast<int64_t>(pg) * pt.page + s % pt.page;
}
#endif

// clock64 cycles one bounded device wait may take before it records
// DSA_ERR_DEVICE_TIMEOUT: DSA_WAIT_BUDGET_CYCLES if set (> 0), else ~1 s
long long wait_budget();
// Test hook: DSA_MLA_MAX_PAIRS=n caps the sparse MLA's persistent grid at n CTA
// pairs, so that small batches drive many items through each pair; 0 = no cap.
int mla_pair_cap();

// ---------------------------------------------------------------- indexer --
struct IndexerParams {
  const int32_t* cu_q;
  const int32_t* kv_len;
  const int64_t* kv_start;
  const float* q_scale;   // [total_q, 64]
  const float* w;         // [total_q, 64]
  const float* k_scale;   // [total_keys]
  float* scores;          // [total_q, ld]
  int64_t ld;
  int64_t total_keys;
  int32_t tiles_per_chunk;  // 128-key tiles one CTA scores
  int32_t num_qblocks;      // gridDim.y
  uint32_t* err;
  long long budget;         // clock64 cycles per bounded wait
  PageTable pt;             // paged: the k tiles load as two 64-row boxes from their pages
  int32_t skip_arrival = -1;  // failure-path tests only: CTA (0,0,0) skips its epilogue's
                              // release of this accumulator item (see test_skip_arrival)
};

// Item whose accumulator release CTA (0,0,0) of the indexer skips, so that a
// bounded wait runs out: DSA_TEST_SKIP_ARRIVAL, read per call; -1 (unset) in
// normal use.  For tests of the device error path only.
int test_skip_arrival();

// tokens per CTA: 1, 2, 4 or 8
int indexer_tokens_per_cta(int max_q_per_seq);
size_t indexer_smem_bytes(int tok);
int indexer_box_rows_q(int tok);
cudaError_t launch_indexer(int tok, dim3 grid, const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                           const IndexerParams& p, cudaStream_t stream);

// Fused decode indexer + top-k: a cluster of CTAs per (sequence, token
// group) scores the row's keys into shared memory, one contiguous chunk per
// CTA, and selects the row's top k with a cluster-wide radix select; no score
// leaves the chip.  For batches of 1-2 query tokens per sequence.
struct IndexerTopkParams {
  IndexerParams ix;        // scores / ld unused
  int32_t k_sel = 0;
  int32_t* idx = nullptr;  // [total_q, k_sel]
  int32_t max_kv_len = 0;  // host maximum over the batch (the chunk capacity was checked against it)
};
// CTAs per cluster for this batch, 0 when the fused kernel does not apply
// (more than 2 tokens per sequence, or a row too long for 16 CTAs).
int indexer_topk_cluster(int max_q_per_seq, int num_seqs, int max_kv_len);
// Whether dsa_forward should take the fused kernel (it is not always faster
// than the indexer + top-k pair; dsa_indexer_topk takes it whenever it applies).
bool indexer_topk_preferred(int max_q_per_seq, int num_seqs, int cluster);
cudaError_t launch_indexer_topk(int tok, int cluster, dim3 grid, const CUtensorMap& tmap_q,
                                const CUtensorMap& tmap_k, const IndexerTopkParams& p, cudaStream_t stream);

// ------------------------------------------------------------------ top-k --
struct TopkParams {
  const int32_t* cu_q;
  const int32_t* kv_len;
  const float* scores;
  int64_t ld;
  int32_t k_sel;
  int32_t* idx;           // [total_q, k_sel]
  int32_t total_q;
  int32_t num_seqs;
  uint32_t* err;
  long long budget;       // clock64 cycles a bulk-copy wait may take
  // two-phase path (topk_segments(...).segs > 0): n_seg segments of seg_len
  // positions per row; [total_q, n_seg, k_sel] candidate positions and scores
  int32_t* seg_pos = nullptr;
  float* seg_val = nullptr;
  int32_t n_seg = 0;
  int32_t seg_len = 0;
};

// Two-phase top-k plan: rows longer than 32768 positions are selected per
// segment and then merged.  segs == 0: the single-pass kernels.
struct TopkSegments {
  int segs;
  int len;
};
TopkSegments topk_segments(int max_kv_len, int k_sel, int total_q);
cudaError_t launch_topk(int max_kv_len, const TopkParams& p, cudaStream_t stream);
// p.idx (local positions, as launch_topk wrote them) -> global positions
// (+ pos_offset[sequence], may be null) in place, and their scores into vals
cudaError_t launch_topk_values(const TopkParams& p, const int32_t* pos_offset, float* vals, cudaStream_t stream);
// top k of n_src candidate lists of k entries per row (n_src * k <= 32768, a multiple of 4)
cudaError_t launch_topk_merge_sources(int n_rows, int n_src, int k, const int32_t* cand_pos, const float* cand_val,
                                      int32_t* idx, cudaStream_t stream);

// ------------------------------------------------------------- sparse MLA --
struct MlaParams {
  const int32_t* cu_q = nullptr;
  const int32_t* kv_len = nullptr;
  const int64_t* kv_start = nullptr;
  const uint16_t* q = nullptr;        // bf16 [total_q, H, 576]
  const uint16_t* kv = nullptr;       // [total_keys, 576]: bf16 cache, or its fp16 copy
  const int32_t* idx = nullptr;       // [total_q, k_sel]
  int64_t total_keys = 0;
  int32_t total_q = 0;                // rows of q / out / lse / idx
  int32_t num_seqs = 0;               // entries of kv_len; cu_q has num_seqs + 1
  PageTable pt;
  int32_t k_sel = 0;
  int32_t n_heads = 0;
  float scale_log2 = 0.f;             // sm_scale * log2(e)
  uint16_t* out = nullptr;            // bf16 [total_q, H, 512]
  float* lse = nullptr;               // [total_q, H] or nullptr
  float* part_o = nullptr;            // [total_q, nsplit, 128, 512] fp32 when nsplit > 1
  float* part_lse = nullptr;          // [total_q, nsplit, 2 value halves, 128]
  int32_t nsplit = 1;
  int32_t keys_per_split = 0;         // multiple of 64
  uint32_t* err = nullptr;
  long long budget = 2000000000LL;
};

int mla_num_splits(int total_q, int max_q_per_seq, int num_seqs, int k_sel);
int mla_keys_per_split(int k_sel, int nsplit);
// Gather from an fp16 copy of the latent cache (made once per call) when the
// selections reuse each latent row often enough to amortise the copy.
bool mla_use_fp16_copy(int total_q, int max_kv_len, int64_t total_keys, int k_sel);
size_t mla_smem_bytes();
// TMA descriptors of the sparse MLA kernel (bf16 bits as 16-bit elements):
//   q_lat  over q viewed as [total_q * H, 576], box [H rows x 64 cols], 128-byte swizzle
//   q_rope the same tensor, box [min(H, 64) rows x 32 cols], 64-byte swizzle
struct MlaMaps {
  CUtensorMap q_lat;
  CUtensorMap q_rope;
};
// Encodes both descriptors for q [total_q * n_heads, 576]; false if the driver
// refuses them.
bool make_mla_maps(MlaMaps* m, const void* q, int64_t total_q, int n_heads);
// p.kv is the bf16 cache: selected rows are gathered with 16-byte loads, Q.C^T
// runs in bf16 on them, and their value part is then converted to fp16 in
// shared memory for P.V (no extra buffers).
// Both launch a persistent grid: one CTA pair per resident cluster slot (at
// most total_q * nsplit pairs), each pair walking its share of the (token,
// split) items.
cudaError_t launch_sparse_mla(const MlaParams& p, const MlaMaps& maps, cudaStream_t stream);
// p.kv is an fp16 copy of the cache (launch_latent_to_fp16): rows are
// gathered ready for the MMAs.
cudaError_t launch_sparse_mla_fp16(const MlaParams& p, const MlaMaps& maps, cudaStream_t stream);
cudaError_t launch_latent_to_fp16(const uint16_t* src, uint16_t* dst, int64_t n_elems, cudaStream_t stream);
cudaError_t launch_mla_combine(int total_q, const MlaParams& p, cudaStream_t stream);

// ------------------------------------------------------------------- prep --
// per-128 FP8 quantiser: x bf16 [n_vec, 128] -> codes e4m3 [n_vec, 128], scales [n_vec]
cudaError_t launch_quantize_fp8(const void* x, int64_t n_vec, void* codes, float* scales, cudaStream_t stream);
// non-interleaved RoPE on dims 0..63 -> normalised Walsh-Hadamard -> per-128 FP8
cudaError_t launch_indexer_prep(const void* x, int64_t n_vec, int vecs_per_pos, const int32_t* pos,
                                const float* rope_cos, const float* rope_sin, int n_pos, void* codes, float* scales,
                                uint32_t* err, cudaStream_t stream);
// new tokens' keys (quantised) and latent rows into the flat caches
cudaError_t launch_cache_write(int num_seqs, int max_q_per_seq, int total_q, int64_t total_keys,
                               const int32_t* cu_q, const int32_t* kv_len, const int64_t* kv_start,
                               const PageTable& pt, const void* k, const void* latent, void* k_cache, float* k_scale,
                               void* latent_cache, uint32_t* err, cudaStream_t stream);

}  // namespace dsa
