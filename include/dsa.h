/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * Three stages, each one hand-written CUDA kernel, plus their composition:
 *
 *   dsa_indexer_scores  Lightning-Indexer scores, Eq. (1) of "详解DSA":
 *                         I[t,s] = sum_{j<64} w[t,j] * ReLU(q[t,j] . k[s]),  s <= t,
 *                       on FP8 e4m3 q and k with one fp32 scale per 128-element
 *                       vector (the demo Indexer.forward of "详解DSA" quantises q
 *                       and k per 128 and hands codes + scales to its FP8 index
 *                       kernel).  The scales are folded exactly:
 *                         I = k_scale[s] * sum_j (w*q_scale)[t,j] * ReLU(q8[t,j] . k8[s]).
 *   dsa_topk            per query row, the k_sel positions of largest score among
 *                       s <= t, Eq. (2) of "详解DSA" (S_t = {s : I[t,s] in Top-k});
 *                       rows with at most k_sel positions keep all of them (the
 *                       demo takes topk(min(index_topk, end_pos))).
 *   dsa_sparse_mla      attention of all n_heads query heads of a token over the
 *                       selected latent entries, MQA mode ("DeepSeek V3.2
 *                       稀疏注意力", section on embedding DSA in MLA: every head of
 *                       a token shares the same top-k latent KV entries):
 *                         o[h] = sum_i softmax_i(sm_scale * q[h] . c[s_i]) * c[s_i][0:512]
 *                       over 576-d entries (512 latent + 64 RoPE), value = first 512.
 *   dsa_forward         indexer -> top-k -> sparse MLA on one stream
 *                       (T_DSA = T_index + T_topk + T_gather + T_sparse_attn,
 *                       "DeepSeek V3.2 稀疏注意力", complexity section).
 *   dsa_quantize_fp8,   upstream of the three: the per-128 FP8 quantiser of q / k
 *   dsa_cache_write     and the write of new tokens into the key and latent caches.
 *
 * Conventions (all entry points):
 *   - Every tensor pointer is caller-owned DEVICE memory, row-major and
 *     contiguous, 16-byte aligned.  The library never allocates, never frees
 *     and keeps no per-call global state.
 *   - Every call is asynchronous on `stream` and never synchronises, except
 *     dsa_check_device_error.  Argument errors are returned before any launch.
 *   - Positions (indices) are sequence-relative int32, as torch.topk returns
 *     positions in the demo; a selection is a set: valid entries first, then -1.
 *   - Unsupported shapes return DSA_ERR_UNSUPPORTED; there is no fallback path.
 *   - `ws` is a caller-provided device workspace of at least
 *     dsa_workspace_size(op, ...) bytes.  Its first 16 bytes are a device error
 *     word that kernels set when a bounded wait times out or an index is out of
 *     range; zero the workspace once after allocating it, and read (and clear)
 *     the word with dsa_check_device_error.
 *
 * Ragged batches: query row r belongs to sequence b with cu_q[b] <= r < cu_q[b+1];
 * its i-th query (i = r - cu_q[b]) sits at position t = kv_len[b] - q_len[b] + i,
 * q_len[b] = cu_q[b+1] - cu_q[b], and may see positions 0..t.  Key/latent row of
 * position s of sequence b is kv_start[b] + s in the flat caches.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL = the legacy default stream. */
typedef struct CUstream_st* dsa_stream_t;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misaligned pointer          */
  DSA_ERR_UNSUPPORTED = 2,     /* a shape the kernels do not implement                */
  DSA_ERR_CUDA = 3,            /* a CUDA runtime/driver call failed                   */
  DSA_ERR_WORKSPACE = 4,       /* ws too small                                        */
  DSA_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait ran out (device error word) */
  DSA_ERR_DEVICE_BOUNDS = 6    /* a kernel met an out-of-range index (device word)    */
} dsa_status_t;

typedef enum {
  DSA_OP_INDEXER = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_SPARSE_MLA = 2,
  DSA_OP_FORWARD = 3,
  DSA_OP_CACHE_WRITE = 4,
  DSA_OP_INDEXER_TOPK = 5
} dsa_op_t;

/* Host struct describing a ragged batch; the arrays are DEVICE memory.
 *
 * Caches are flat (block_table == NULL: position s of sequence b is cache row
 * kv_start[b] + s) or paged (block_table != NULL: the key, key-scale and
 * latent caches are pools of total_keys / page_size pages of page_size rows,
 * and position s of sequence b is pool row
 *     block_table[b * blocks_per_seq + s / page_size] * page_size + s % page_size;
 * kv_start is then ignored and may be NULL).  "DeepSeek V3.2 稀疏注意力" lists
 * this logical-position -> block/offset map among what a decode kernel must
 * define.  A page id outside [0, total_keys / page_size) is a device-side
 * bounds error (DSA_ERR_DEVICE_BOUNDS); the row it would address is not read. */
typedef struct {
  int32_t num_seqs;          /* B >= 1                                             */
  int32_t total_q;           /* cu_q[B]; query rows of every per-row tensor       */
  int32_t max_q_per_seq;     /* max_b q_len[b] (host copy, sizes the grids)       */
  int32_t max_kv_len;        /* max_b kv_len[b] (host copy)                       */
  int64_t total_keys;        /* rows of the key / latent caches or pools (< 2^31) */
  const int32_t* cu_q;       /* [B+1] query-row offsets, cu_q[0] = 0              */
  const int32_t* kv_len;     /* [B] positions present, including the new queries  */
  const int64_t* kv_start;   /* [B] first flat cache row of each sequence          */
  const int32_t* block_table;  /* [B, blocks_per_seq] page ids, or NULL (flat)     */
  int32_t page_size;         /* paged: rows per page, a positive multiple of 64    */
  int32_t blocks_per_seq;    /* paged: row stride of block_table,
                                >= ceil(max_kv_len / page_size)                    */
} dsa_batch_t;

/* Fixed sizes of the hot path (the pages' indexer: 64 heads of dim 128). */
#define DSA_INDEX_HEADS 64
#define DSA_INDEX_DIM 128
#define DSA_LATENT_DIM 576
#define DSA_VALUE_DIM 512
#define DSA_MAX_K_SEL 2048

/* Bytes of device workspace the call `op` needs for this batch.  Returns 0
 * when the arguments are invalid.  For DSA_OP_FORWARD and DSA_OP_INDEXER_TOPK
 * this includes the [total_q, ld] fp32 score matrix, ld = max_kv_len rounded
 * up to 4 -- except for decode batches (at most 2 query tokens per sequence,
 * rows the fused kernel's clusters hold), whose scores never leave the chip.
 * (dsa_forward: only where it takes the fused kernel, see dsa_indexer_topk).
 * For DSA_OP_TOPK (and the unfused forward) rows longer than 32768 positions
 * with k_sel a multiple of 4 add 8 * k_sel bytes per row and 32768-position
 * segment: the candidates of the two-phase selection. */
DSA_API size_t dsa_workspace_size(dsa_op_t op, const dsa_batch_t* batch, int32_t k_sel, int32_t n_heads);

/* Indexer scores.
 *   q_fp8   [total_q, 64, 128] e4m3 codes      q_scale [total_q, 64] fp32 (> 0)
 *   w       [total_q, 64] fp32                 k_fp8   [total_keys, 128] e4m3 codes
 *   k_scale [total_keys] fp32 (> 0)
 *   scores  [total_q, ld_scores] fp32 out; row r holds I[t, s] for s = 0..t of its
 *           sequence; entries beyond t are not written.  ld_scores >= max_kv_len,
 *           a multiple of 4. */
DSA_API dsa_status_t dsa_indexer_scores(const dsa_batch_t* batch, const void* q_fp8, const float* q_scale,
                                const float* w, const void* k_fp8, const float* k_scale, float* scores,
                                int64_t ld_scores, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Top-k positions per query row.
 *   scores [total_q, ld_scores] fp32 (only s <= t is read)
 *   idx    [total_q, k_sel] int32 out: the k_sel highest-scoring positions
 *          (equal scores: the lower s wins; -0 and +0 are equal) in ascending
 *          order of s, then -1 padding when t + 1 < k_sel.
 *   1 <= k_sel <= 2048. */
DSA_API dsa_status_t dsa_topk(const dsa_batch_t* batch, const float* scores, int64_t ld_scores, int32_t k_sel,
                      int32_t* idx, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Indexer scores and top-k in one call: `idx` as dsa_topk returns it for the
 * scores dsa_indexer_scores computes, bit for bit.  For decode batches (at
 * most 2 query tokens per sequence, rows of up to 16 x 16384 positions) one
 * fused kernel always does both (dsa_forward takes it only where it is the
 * faster path: one query token per sequence, enough sequences to fill the GPU) ("DeepSeek V3.2 稀疏注意力", what happens in prefill
 * and decode: score tile by tile, keep local candidates, merge, and hand the
 * selection to sparse MLA without writing the score matrix to HBM): a
 * cluster of CTAs per sequence scores one contiguous key chunk per CTA into
 * shared memory and selects with an exact radix select whose histograms are
 * reduced across the cluster.  Other batches run the two kernels with the
 * scores in `ws`.  Arguments as for dsa_indexer_scores and dsa_topk; ws of
 * dsa_workspace_size(DSA_OP_INDEXER_TOPK, ...) bytes. */
DSA_API dsa_status_t dsa_indexer_topk(const dsa_batch_t* batch, const void* q_fp8, const float* q_scale,
                                      const float* w, const void* k_fp8, const float* k_scale, int32_t k_sel,
                                      int32_t* idx, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Key-sharded selection ("DeepSeek V3.2 稀疏注意力", top-k section: with the
 * keys split across devices, select a local top k per shard, then merge the
 * shards' candidates).  Each of a row's top k lies in the top k of its own
 * shard, so the merge equals a selection over the whole row.
 *
 * dsa_topk_candidates: dsa_topk over one shard's scores (the batch describes
 * the shard: kv_len = the shard's positions, which start at global position
 * pos_offset[b] of sequence b), writing each selected position as a global one
 * and its score:
 *   cand_pos [total_q, k_sel] int32 out: pos_offset[b] + local position,
 *            ascending, -1 padding (pos_offset may be NULL: offsets 0)
 *   cand_val [total_q, k_sel] fp32 out: the scores; padding gets a NaN whose
 *            order key is below every score.
 *   ws as for dsa_topk. */
DSA_API dsa_status_t dsa_topk_candidates(const dsa_batch_t* batch, const float* scores, int64_t ld_scores,
                                         int32_t k_sel, const int32_t* pos_offset, int32_t* cand_pos,
                                         float* cand_val, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* dsa_topk_merge: per row, the k_sel highest-scoring of n_src candidate lists
 * of k_sel entries each (the shards' dsa_topk_candidates outputs, gathered in
 * shard order, shards covering ascending position ranges):
 *   cand_pos [n_rows, n_src, k_sel] int32, cand_val [n_rows, n_src, k_sel] fp32
 *   idx      [n_rows, k_sel] int32 out: positions ascending, -1 padding.
 * Ties as in dsa_topk (the lower position wins).  n_src * k_sel <= 32768 and a
 * multiple of 4 (else DSA_ERR_UNSUPPORTED).  No workspace. */
DSA_API dsa_status_t dsa_topk_merge(int32_t n_rows, int32_t n_src, int32_t k_sel, const int32_t* cand_pos,
                                    const float* cand_val, int32_t* idx, dsa_stream_t stream);

/* Sparse MLA (MQA mode).
 *   q    [total_q, n_heads, 576] bf16        kv [total_keys, 576] bf16 latent cache
 *   idx  [total_q, k_sel] int32 positions; entries < 0 or >= kv_len are skipped
 *   out  [total_q, n_heads, 512] bf16 (round to nearest even from fp32)
 *   lse  [total_q, n_heads] fp32 natural-log sum-exp of the scaled logits, or NULL.
 *   A row with no usable entry gives out = 0, lse = -inf.
 *   1 <= n_heads <= 128 (one 128-row MMA tile; fewer heads leave rows idle);
 *   k_sel as for dsa_topk.
 * Arithmetic: the logits q . c accumulate in fp32 on the tensor cores and the
 * softmax runs in fp32.  For P . V the probabilities are rounded to fp16 and
 * the value part of the gathered entries is converted to fp16, which holds
 * every bf16 value of magnitude 2^-17 .. 65280 exactly (smaller magnitudes
 * keep an absolute error below 2^-25; larger ones saturate at 65504).  The
 * logits use the bf16 values as given, except for batches whose selections
 * reuse each cache row many times (prefill-shaped), where the library first
 * makes an fp16 copy of the cache in `ws` and q and the whole entries go
 * through the same fp16 conversion.  A descriptor that addresses rows outside
 * the cache (q_len > kv_len, kv_start + kv_len > total_keys) records
 * DSA_ERR_DEVICE_BOUNDS and leaves that sequence's rows at out = 0, lse = -inf;
 * a row of q that lies in no sequence of cu_q (cu_q not covering 0..total_q)
 * records DSA_ERR_DEVICE_BOUNDS and gets out = 0, lse = -inf as well. */
DSA_API dsa_status_t dsa_sparse_mla(const dsa_batch_t* batch, const void* q, int32_t n_heads, const void* kv,
                            const int32_t* idx, int32_t k_sel, float sm_scale, void* out, float* lse, void* ws,
                            size_t ws_bytes, dsa_stream_t stream);

/* The whole hot path: indexer scores and top-k into `idx` (as
 * dsa_indexer_topk: fused on chip for decode batches, else with the scores
 * kept in ws), sparse MLA into `out`/`lse`.  Arguments as above. */
DSA_API dsa_status_t dsa_forward(const dsa_batch_t* batch, const void* q_fp8, const float* q_scale, const float* w,
                         const void* k_fp8, const float* k_scale, int32_t k_sel, const void* q, int32_t n_heads,
                         const void* kv, float sm_scale, int32_t* idx, void* out, float* lse, void* ws,
                         size_t ws_bytes, dsa_stream_t stream);

/* Sparse MLA without a caller workspace -- for callers that cannot allocate
 * device memory.  (The pages have no counterpart to this entry point; it is a
 * deployment convenience.)
 *
 * Who needs it: code that does not own an allocator, e.g. a plugin inside a
 * host engine that may only use the buffers the engine hands it, or a
 * latency-critical loop where cudaMalloc's implicit device synchronisation is
 * not acceptable.  Such callers still provide q, kv, idx, out and lse exactly
 * as for dsa_sparse_mla; the split-selection partial results that
 * dsa_sparse_mla keeps in `ws` live instead in a library-owned device array of
 * DSA_NO_ALLOC_SCRATCH_BYTES (32 MiB), which every GPU that loads the library
 * holds until the process exits.  The call itself performs no cudaMalloc,
 * cudaFree or other allocation.
 *
 *   - Batches whose partial results need more than the scratch array (more
 *     than 256 B + total_q * nsplit * 128 * 2056 B, rounded) return
 *     DSA_ERR_WORKSPACE before anything is launched; use dsa_sparse_mla then.
 *     (Selections are split only while total_q * nsplit fits 74 CTA pairs,
 *     into at most 4 parts, so valid batches need at most ~19 MiB.)
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array, which keeps the previous
 *     call's contents; each call clears the error word it needs at the start.
 *     Calls whose work overlaps on the GPU (different streams, no ordering)
 *     race on the array and must be serialised by the caller.
 *   - Device-side error statuses (bounded-wait timeouts, descriptors that
 *     address rows outside the cache) are recorded in the array and are not
 *     reported to the caller; use dsa_sparse_mla with a workspace and
 *     dsa_check_device_error when they are needed.  Rows of a sequence whose
 *     descriptors are out of range come out as out = 0, lse = -inf, never as
 *     another call's leftovers.
 *   - It always runs the bf16-cache kernel (bf16 Q . C^T on the gathered
 *     rows, no fp16 copy of the cache, which would need a workspace).  On the
 *     prefill-shaped batches where dsa_sparse_mla takes its fp16-copy path the
 *     two entry points therefore round q . c differently; both stay within the
 *     parity tolerances.  Arguments and results are otherwise those of
 *     dsa_sparse_mla. */
#define DSA_NO_ALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
DSA_API dsa_status_t dsa_sparse_mla_no_alloc(const dsa_batch_t* batch, const void* q, int32_t n_heads,
                                             const void* kv, const int32_t* idx, int32_t k_sel, float sm_scale,
                                             void* out, float* lse, dsa_stream_t stream);

/* Upstream preparation ("详解DSA", the indexer code: q and k pass through a
 * per-block activation quantiser with block = the indexer head dim, one fp32
 * scale per 128-element vector, and the new tokens' codes and scales are
 * stored in the key cache; "DeepSeek V3.2 稀疏注意力", data-flow section: the
 * latent rows go to the MLA cache).  Scale rule (open on the page; the plain
 * reading): scale = fp32(amax / 448) over the vector's values, 1 for an
 * all-zero vector; code = e4m3(fp32(x / scale)), round to nearest even,
 * saturating at +-448, sign of zero kept.  Inputs must be finite.
 *
 * dsa_quantize_fp8: n_vec vectors of 128 bf16 values.
 *   x      [n_vec, 128] bf16
 *   codes  [n_vec, 128] e4m3 out
 *   scales [n_vec] fp32 out
 *   n_vec >= 0 (0: nothing launched); e.g. q as [total_q * 64, 128] gives the
 *   q_fp8 / q_scale inputs of dsa_indexer_scores.  No workspace, no device
 *   error word (there is no index to check). */
DSA_API dsa_status_t dsa_quantize_fp8(const void* x, int64_t n_vec, void* codes, float* scales,
                                      dsa_stream_t stream);

/* dsa_indexer_prep: the whole input chain of the indexer's q or k vectors
 * ("详解DSA", indexer code: rotary embedding on the first 64 dims of each
 * 128-dim vector, then rotate_activation, then act_quant; "DeepSeek V3.2
 * 稀疏注意力": the indexer takes the non-interleaved RoPE layout).  Readings
 * (the pages define neither function): dims i and i + 32 (i < 32) rotate by
 * (rope_cos, rope_sin)[pos][i], out_i = x_i c - x_{i+32} s and out_{i+32} =
 * x_{i+32} c + x_i s in fp32 without fused multiply-adds, stored as bf16;
 * rotate_activation is the normalised Walsh-Hadamard transform over the 128
 * dims (Sylvester order, butterfly stages 1, 2, ..., 64 in fp32, times
 * fp32(128^-0.5)), stored as bf16; then the quantiser above.
 *   x        [n_vec, 128] bf16; vector v belongs to position pos[v / vecs_per_pos]
 *            (vecs_per_pos = 64 for q, the token's head vectors; 1 for k)
 *   pos      [n_vec / vecs_per_pos] int32 positions, 0 <= pos < n_pos
 *   rope_cos, rope_sin  [n_pos, 32] fp32 tables (the caller's frequencies)
 *   codes    [n_vec, 128] e4m3 out;  scales [n_vec] fp32 out
 *   ws       >= 256 bytes (device error word): a position outside the table is
 *            DSA_ERR_DEVICE_BOUNDS, its vector written as codes 0, scale 1. */
DSA_API dsa_status_t dsa_indexer_prep(const void* x, int64_t n_vec, int32_t vecs_per_pos, const int32_t* pos,
                                      const float* rope_cos, const float* rope_sin, int32_t n_pos, void* codes,
                                      float* scales, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* dsa_cache_write: the keys and latent rows of the batch's new tokens into the
 * flat caches.  Query row r (sequence b, position t, see "Ragged batches")
 * writes cache row kv_start[b] + t:
 *   k       [total_q, 128] bf16 new keys     -> k_cache [total_keys, 128] e4m3,
 *                                               k_scale [total_keys] fp32 (the rule above)
 *   latent  [total_q, 576] bf16 new entries  -> latent_cache [total_keys, 576] bf16 (copied)
 * Other cache rows are untouched.  ws: at least dsa_workspace_size(
 * DSA_OP_CACHE_WRITE, ...) bytes; a sequence whose cu_q / kv_len / kv_start
 * would address rows outside the caches is skipped and DSA_ERR_DEVICE_BOUNDS
 * recorded in the device error word. */
DSA_API dsa_status_t dsa_cache_write(const dsa_batch_t* batch, const void* k, const void* latent, void* k_cache,
                                     float* k_scale, void* latent_cache, void* ws, size_t ws_bytes,
                                     dsa_stream_t stream);

/* Synchronise `stream`, read the device error word of `ws`, clear it, and
 * return DSA_OK, DSA_ERR_DEVICE_TIMEOUT or DSA_ERR_DEVICE_BOUNDS (or
 * DSA_ERR_CUDA if the stream reports an error).  `site` / `info`, if not NULL,
 * receive the kernel site id and detail recorded with the error. */
DSA_API dsa_status_t dsa_check_device_error(void* ws, dsa_stream_t stream, uint32_t* site, uint32_t* info);

/* Kernel launches one dsa_forward call makes for this batch: the indexer and
 * the top-k (one fused launch for decode batches; otherwise one plus one, or
 * two for rows longer than 32768 positions with k_sel a multiple of 4),
 * the fp16 copy of the latent cache when the selections reuse its rows often,
 * the sparse MLA, and the merge of split selections.  0 when the arguments are
 * invalid.  Host-only; for accounting and profiling. */
DSA_API int32_t dsa_forward_launches(const dsa_batch_t* batch, int32_t k_sel, int32_t n_heads);

/* Static description of a status code. */
DSA_API const char* dsa_status_string(dsa_status_t status);

/* ABI version (major * 100 + minor); 200 added the paged-cache fields of
 * dsa_batch_t and dsa_indexer_topk. */
DSA_API int32_t dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
