// dsa_noalloc.cu -- top-k select for callers that cannot allocate device memory.
//
// Some callers of this library may not allocate GPU memory at the point where they run
// the select: a plugin inside an inference engine whose enqueue step must not allocate
// (the engine owns every buffer), a serving loop that works inside a fixed, pre-planned
// memory budget, or a latency-critical host thread that must not call cudaMalloc, which
// can synchronise the whole device.  dsa_topk_noalloc serves them: its scratch memory is
// a fixed array compiled into the library (below), so the caller passes only the scores
// and the output buffer.  Shapes whose rows each fit one cluster of CTAs on chip use no
// scratch at all; the others (many rows, or rows longer than a cluster holds) take the
// scan kernels, whose scratch must fit the array.
//
// The array lives in every GPU that loads the library until the process exits.  All
// calls share it and it keeps the last call's contents; the parts that must start at
// zero are cleared on the stream at the start of every call.  Two calls that overlap on
// the GPU (different streams, no ordering between them) race on it.
#include "dsa.h"
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)DSA_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_topk_scratch[kScratchBytes];

// device address of g_topk_scratch, looked up once per device with that device current
struct ScratchAddress {
  std::atomic<void*> ptr[64] = {};

  cudaError_t get(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    void* p = ptr[dev].load(std::memory_order_acquire);
    if (!p) {
      e = cudaGetSymbolAddress(&p, g_topk_scratch);
      if (e != cudaSuccess) return e;
      ptr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
  }
};

ScratchAddress g_scratch_address;

}  // namespace

extern "C" dsa_status dsa_topk_noalloc(const float* scores, int B, int T, int N, long long q_pos0, int k,
                                       int32_t* idx, cudaStream_t stream) {
  if (!scores || !idx || B <= 0 || T <= 0 || N <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if ((long long)B * T > 65535) return DSA_ERR_INVALID_ARG;
  if (k > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(scores) | reinterpret_cast<uintptr_t>(idx)) % 4) return DSA_ERR_INVALID_ARG;
  const long long rows = (long long)B * T;
  const long long vmax = dsa::visible_count(N, q_pos0, T - 1);
  if (dsa::topk_uses_workspace(rows, vmax) && dsa::topk_workspace_bytes(rows, N) > kScratchBytes)
    return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const cudaError_t ea = g_scratch_address.get(&scratch);
  if (ea != cudaSuccess) return dsa::cuda_status(ea);
  dsa::TopkWorkspace ws = dsa::topk_workspace(scratch, rows, N);
  const cudaError_t e = dsa::launch_topk(scores, B, T, N, q_pos0, k, idx, ws, false, 0, stream);
  return dsa::cuda_status(e);
}
