// Kernel parameter blocks and host-side launch entry points shared between
// the kernels' translation units and the C ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

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
};

// tokens per CTA: 1, 2, 4 or 8
int indexer_tokens_per_cta(int max_q_per_seq);
size_t indexer_smem_bytes(int tok);
int indexer_box_rows_q(int tok);
cudaError_t launch_indexer(int tok, dim3 grid, const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                           const IndexerParams& p, cudaStream_t stream);

// ------------------------------------------------------------------ top-k --
struct TopkParams {
  const int32_t* cu_q;
  const int32_t* kv_len;
  const float* scores;
  int64_t ld;
  int32_t k_sel;
  int32_t* idx;           // [total_q, k_sel]
  uint32_t* err;
};

cudaError_t launch_topk(int max_kv_len, dim3 grid, const TopkParams& p, cudaStream_t stream);

// ------------------------------------------------------------- sparse MLA --
struct MlaParams {
  const int32_t* cu_q;
  const int32_t* kv_len;
  const int64_t* kv_start;
  const uint16_t* q;        // bf16 [total_q, H, 576]
  const uint16_t* kv;       // bf16 [total_keys, 576]
  const int32_t* idx;       // [total_q, k_sel]
  int64_t total_keys;
  int32_t k_sel;
  int32_t n_heads;
  float scale_log2;         // sm_scale * log2(e)
  uint16_t* out;            // bf16 [total_q, H, 512]
  float* lse;               // [total_q, H] or nullptr
  float* part_o;            // [total_q, nsplit, 128, 512] fp32 when nsplit > 1
  float* part_lse;          // [total_q, nsplit, 128]
  int32_t nsplit;
  int32_t keys_per_split;   // multiple of 64
  uint32_t* err;
  long long budget;
};

int mla_num_splits(int total_q, int max_q_per_seq, int num_seqs, int k_sel);
int mla_keys_per_split(int k_sel, int nsplit);
size_t mla_smem_bytes();
cudaError_t launch_sparse_mla(dim3 grid, const MlaParams& p, cudaStream_t stream);
cudaError_t launch_mla_combine(int total_q, const MlaParams& p, cudaStream_t stream);

}  // namespace dsa
