// dsa_sparse_mla_no_alloc: the sparse MLA entry point for callers that cannot
// allocate device memory.
//
// Some callers own no allocator of their own: an engine plugin that may only
// touch the buffers its host framework hands it, or a latency-critical loop
// where cudaMalloc's implicit device synchronisation is not acceptable.  They
// can still pass inputs and outputs, but not the workspace dsa_sparse_mla
// needs for its split-selection partial results.  This entry point keeps that
// scratch in a fixed, library-owned device array instead, so it allocates
// nothing at call time.
//
// The array lives in this translation unit as a file-scope __device__ object.
// Host code cannot use its name as a device address, so each device's address
// is looked up once with cudaGetSymbolAddress (with that device current) and
// handed to the kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "../../include/dsa.h"
#include "kernels.cuh"

namespace {

constexpr size_t kHeader = 256;      // device error word, as in a caller workspace
constexpr int kMaxDevices = 64;

// Scratch shared by every call on a device; every GPU that loads the library
// holds it until the process exits.
static __device__ __align__(256) unsigned char g_mla_scratch[DSA_NO_ALLOC_SCRATCH_BYTES];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device address of g_mla_scratch on the current device (looked up on first use).
cudaError_t scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_mla_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" dsa_status_t dsa_sparse_mla_no_alloc(const dsa_batch_t* b, const void* q, int32_t n_heads, const void* kv,
                                                const int32_t* idx, int32_t k_sel, float sm_scale, void* out,
                                                float* lse, dsa_stream_t stream) {
  // ---- argument checks, the same rules as dsa_sparse_mla ----
  const dsa_status_t bs = dsa::validate_batch(b);
  if (bs != DSA_OK) return bs;
  auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (q == nullptr || kv == nullptr || out == nullptr || idx == nullptr) return DSA_ERR_INVALID_ARG;
  if (misaligned(q) || misaligned(kv) || misaligned(out)) return DSA_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return DSA_ERR_INVALID_ARG;
  if (n_heads < 1 || n_heads > 128 || k_sel < 1 || k_sel > DSA_MAX_K_SEL) return DSA_ERR_UNSUPPORTED;

  // ---- scratch size check, before touching the device ----
  const int nsplit = dsa::mla_num_splits(b->total_q, b->max_q_per_seq, b->num_seqs, k_sel);
  const size_t rows = static_cast<size_t>(b->total_q) * nsplit * 128;
  const size_t o_bytes = nsplit > 1 ? round_up(rows * 512 * sizeof(float), 256) : 0;
  const size_t lse_bytes = nsplit > 1 ? round_up(rows * 2 * sizeof(float), 256) : 0;
  if (kHeader + o_bytes + lse_bytes > DSA_NO_ALLOC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
  if (b->total_q == 0) return DSA_OK;

  void* base = nullptr;
  if (scratch_for_current_device(&base) != cudaSuccess) return DSA_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The previous call's contents stay in the array; only the error word must
  // start at zero.  Every partial result the merge reads is written by this
  // call first: a CTA pair that processes its split writes its partial output
  // and log-sum-exp, and a pair whose sequence descriptors are out of range
  // writes lse = -inf for its split, which the merge turns into out = 0,
  // lse = -inf for that row.
  if (cudaMemsetAsync(base, 0, 16, st) != cudaSuccess) return DSA_ERR_CUDA;

  dsa::MlaParams p;
  p.cu_q = b->cu_q;
  p.kv_len = b->kv_len;
  p.kv_start = b->kv_start;
  p.q = static_cast<const uint16_t*>(q);
  p.kv = static_cast<const uint16_t*>(kv);
  p.idx = idx;
  p.total_keys = b->total_keys;
  p.total_q = b->total_q;
  p.num_seqs = b->num_seqs;
  p.pt = dsa::batch_pages(b);
  p.k_sel = k_sel;
  p.n_heads = n_heads;
  p.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.nsplit = nsplit;
  p.keys_per_split = dsa::mla_keys_per_split(k_sel, nsplit);
  uint8_t* scratch = static_cast<uint8_t*>(base);
  p.part_o = nsplit > 1 ? reinterpret_cast<float*>(scratch + kHeader) : nullptr;
  p.part_lse = nsplit > 1 ? reinterpret_cast<float*>(scratch + kHeader + o_bytes) : nullptr;
  p.err = reinterpret_cast<uint32_t*>(scratch);
  p.budget = dsa::wait_budget();
  if (static_cast<int64_t>(b->total_q) * nsplit >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  dsa::MlaMaps maps;
  if (!dsa::make_mla_maps(&maps, q, b->total_q, n_heads)) return DSA_ERR_CUDA;
  if (dsa::launch_sparse_mla(p, maps, st) != cudaSuccess) return DSA_ERR_CUDA;
  if (nsplit > 1 && dsa::launch_mla_combine(b->total_q, p, st) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}
