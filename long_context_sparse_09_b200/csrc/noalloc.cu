// noalloc.cu -- csa_index_topk_noalloc: the indexer + top-k entry point for
// callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: host
// frameworks that own every byte of device memory and give their plugins no
// workspace hook, and latency-critical loops where an allocation would
// synchronise the device or fail against a pool that is already reserved.
// For them this entry point takes its scratch (the fp32 score buffer of the
// indexer) from a fixed array compiled into the library instead of a
// caller-provided workspace.  The array lives in device memory on every GPU
// that loads the library, from the first call until the process exits.
#include <atomic>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace csa {

// 16 MiB.  A request fits when csa_index_topk_workspace_bytes(p, B, Q, N),
// the workspace the allocating entry point would take, is at most this: the
// fp32 scores (4 B*Q*N bytes) plus the tile plan and, for a few long
// queries, the multi-CTA top-k lists.  The 1M-context decode of 4 sequences
// needs about 6.6 MiB.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// In host code g_noalloc_scratch names a host-side stand-in, not device
// memory: its device address is looked up once per device, with that device
// current, and cached here.  Host threads may make their first calls on a
// device at the same time: each slot is an atomic, and a thread that finds
// it empty looks the address up itself (the lookups agree).
static void* noalloc_scratch_ptr() {
  static std::atomic<void*> addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  void* p = addr[dev].load(std::memory_order_relaxed);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev].store(p, std::memory_order_relaxed);
  }
  return p;
}

}  // namespace csa

extern "C" csa_status csa_index_topk_noalloc(const csa_params* p, int B, int Q,
                                             const int32_t* q_pos, const void* qI,
                                             const float* w, const void* kI, int N,
                                             int32_t* idx_out, float* score_out,
                                             csa_stream_t stream) {
  using namespace csa;
  if (p == nullptr) return CSA_ERR_ARG;
  if (B <= 0 || Q <= 0 || N < 0) return CSA_ERR_SHAPE;
  // the same workspace the allocating entry point would need must fit
  const size_t need = csa_index_topk_workspace_bytes(p, B, Q, N);
  if (need > kNoAllocScratchBytes) return CSA_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_ptr();
  if (scratch == nullptr) return CSA_ERR_CUDA;
  // Nothing in the scratch has to start at zero: the scorer writes every
  // score that the selection reads.  Argument checks are those of
  // csa_index_topk, which this forwards to with the fixed scratch.
  return csa_index_topk(p, B, Q, q_pos, qI, w, kI, N, idx_out, score_out, scratch,
                        kNoAllocScratchBytes, stream);
}
