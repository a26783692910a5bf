// noalloc.cu -- an indexer + top-k entry point that needs no caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the layer: code that
// runs inside another framework's memory pool without access to its allocator, plugins that are
// handed only the tensors they read and write, or latency-critical paths that must never call
// cudaMalloc. For them, csa_indexer_topk_noalloc keeps its scratch (the per-query score rows and
// the device status word) in one fixed array in device memory that the library defines at file
// scope. Every GPU that loads the library holds the array until the process exits.
//
// The array is shared by every call on a device and keeps the last call's contents: calls whose
// work overlaps on the GPU (different streams without ordering between them) race on it.

#include <cuda_runtime.h>

#include <mutex>

#include "csa.h"
#include "kernels.cuh"

namespace {

// Scratch bytes: the 256-byte status word, then the score rows (B*S*max_entries floats).
constexpr size_t kNoAllocScratchBytes = 256 + (size_t(4) << 20);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device (with that device current).
int scratch_address(void** out) {
  static void* addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return CSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return CSA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return CSA_OK;
}

}  // namespace

extern "C" {

int csa_indexer_topk_noalloc(int B, int S, int H_I, int d_I, int ratio, int topk, const int32_t* q_pos,
                             const uint16_t* q_idx, const float* w, const uint16_t* idx_cache, int64_t idx_bstride,
                             int max_entries, int32_t* topk_idx, void* stream) {
  // Every argument is checked before the fixed array is touched: a refused call writes nothing,
  // so it cannot clear the status word of another call still running on an unordered stream.
  if (int rc = csa::check_indexer_topk_args(B, S, H_I, d_I, ratio, topk, q_pos, q_idx, w, idx_cache, idx_bstride,
                                            max_entries, topk_idx))
    return rc;
  // The fixed array holds the status word and B*S*max_entries scores; rows longer than one top-k
  // chunk (16384 entries) would need the chunked selection's lists as well, so they are refused.
  const size_t rows = size_t(B) * size_t(S) * size_t(max_entries) * sizeof(float);
  const size_t need = 256 + (rows + 255) / 256 * 256;
  if (max_entries > 16384 || need > kNoAllocScratchBytes) return CSA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (int rc = scratch_address(&scratch)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The status word must start at zero; the score rows are written before they are read.
  if (cudaMemsetAsync(scratch, 0, 256, st) != cudaSuccess) return CSA_ERR_CUDA;
  return csa_indexer_topk(B, S, H_I, d_I, ratio, topk, q_pos, q_idx, w, idx_cache, idx_bstride, max_entries,
                          topk_idx, nullptr, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
