// dsa_api.cu -- the C ABI of libdsa: argument checks, workspace layout, launch order.
//
// The IndexShare group driver follows "GLM-5.2 1M architecture teardown", Cut 2:
// IndexShare (the indexer runs in the first of every 4 layers and its top-k list is used
// by all 4) and "GLM-5.2 MTP IndexShare inference", Indexer Share in the MTP layer (draft
// steps 2.. reuse the step-1 index list, so draft-token rows are never attended; the MTP
// layer reads the target cache -- KV Share).
#include <cstdio>

#include "dsa.h"
#include "dsa_common.cuh"
#include "dsa_internal.h"

using namespace dsa;

namespace dsa {
std::atomic<int> g_last_cuda_error{0};
dsa_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return DSA_OK;
  g_last_cuda_error.store((int)e, std::memory_order_relaxed);
  return DSA_ERR_CUDA;
}

int device_sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 0;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}
}  // namespace dsa

namespace {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

bool sizes_ok(int B, int T, int N) {
  if (B <= 0 || T <= 0 || N <= 0) return false;
  const long long rows = (long long)B * T;
  if (rows > 65535) return false;                        // grid y/z limits
  if ((long long)N > 0x7FFFFFFFLL / 1) return false;
  return true;
}

struct GroupLayout {
  size_t topk_off, topk_bytes, scores_off, scores_bytes, attn_off, attn_bytes, total;
};

GroupLayout group_layout(int B, int T, int N, int k, int H, int L) {
  const long long rows = (long long)B * T;
  GroupLayout g;
  g.topk_off = 0;
  g.topk_bytes = round256(topk_workspace_bytes(rows, N));
  g.scores_off = g.topk_off + g.topk_bytes;
  g.scores_bytes = round256((size_t)rows * N * sizeof(float));
  g.attn_off = g.scores_off + g.scores_bytes;
  g.attn_bytes = round256(attn_workspace_bytes(rows, L, H, k));
  g.total = g.attn_off + g.attn_bytes;
  return g;
}

bool heads_supported(int H) { return H == 16 || H == 32 || H == 48 || H == 64; }

// The error words of the indexer, the attention and the top-k, in that order.
struct ErrorWords {
  int code[3] = {0, 0, 0};
  int first() const { return code[0] ? code[0] : code[1] ? code[1] : code[2]; }
  // a wait that ran out (indexer, attention) is a timeout; a broken top-k invariant a
  // device error
  dsa_status status() const { return (code[0] || code[1]) ? DSA_ERR_TIMEOUT : code[2] ? DSA_ERR_DEVICE : DSA_OK; }
};

// Reads the error words on `stream` (the caller has synchronised whatever it wants
// covered) and, with `clear`, resets the ones that are set.
cudaError_t read_error_words(cudaStream_t stream, bool clear, ErrorWords* w) {
  int* p[3] = {nullptr, nullptr, nullptr};
  cudaError_t e;
  if ((e = indexer_error_word(&p[0])) != cudaSuccess) return e;
  if ((e = attn_error_word(&p[1])) != cudaSuccess) return e;
  if ((e = topk_error_word(&p[2])) != cudaSuccess) return e;
  for (int i = 0; i < 3; ++i)
    if ((e = cudaMemcpyAsync(&w->code[i], p[i], sizeof(int), cudaMemcpyDeviceToHost, stream)) != cudaSuccess) return e;
  if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return e;
  if (clear) {
    for (int i = 0; i < 3; ++i)
      if (w->code[i] && (e = cudaMemsetAsync(p[i], 0, sizeof(int), stream)) != cudaSuccess) return e;
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

extern "C" {

int dsa_last_cuda_error(void) { return g_last_cuda_error.load(std::memory_order_relaxed); }

const char* dsa_cuda_error_string(int code) { return cudaGetErrorString((cudaError_t)code); }

const char* dsa_status_string(int status) {
  switch (status) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    case DSA_ERR_DEVICE: return "DSA_ERR_DEVICE";
    default: return "DSA_ERR_UNKNOWN";
  }
}

int dsa_version(void) { return 10000; }

dsa_status dsa_device_error(int* code, int clear) {
  if (!code) return DSA_ERR_INVALID_ARG;
  *code = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e);
  ErrorWords w;
  if ((e = read_error_words(0, clear != 0, &w)) != cudaSuccess) return cuda_status(e);
  *code = w.first();
  return w.status();
}

dsa_status dsa_check_device_status(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_status(e);
  ErrorWords w;
  if ((e = read_error_words(stream, true, &w)) != cudaSuccess) return cuda_status(e);
  return w.status();
}

size_t dsa_workspace_size(int B, int T, int N, int k, int H, int L) {
  if (!sizes_ok(B, T, N) || k <= 0 || k > DSA_MAX_TOPK || H <= 0 || L <= 0 || L > DSA_MAX_LAYERS) return 0;
  return group_layout(B, T, N, k, H, L).total;
}

dsa_status dsa_index_score(const uint16_t* q, const float* w, const uint16_t* k, int B, int T, int N,
                           long long q_pos0, float* scores, cudaStream_t stream) {
  if (!q || !w || !k || !scores || !sizes_ok(B, T, N)) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(w, 16) || !aligned(scores, 4)) return DSA_ERR_INVALID_ARG;
  return cuda_status(launch_index_score_tc(q, w, k, B, T, N, q_pos0, scores, nullptr, stream));
}

dsa_status dsa_topk(const float* scores, int B, int T, int N, long long q_pos0, int k, int32_t* idx, void* workspace,
                    size_t workspace_bytes, cudaStream_t stream) {
  if (!scores || !idx || !sizes_ok(B, T, N) || k <= 0) return DSA_ERR_INVALID_ARG;
  if (k > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if (!aligned(scores, 4) || !aligned(idx, 4)) return DSA_ERR_INVALID_ARG;
  const long long rows = (long long)B * T;
  const size_t need = topk_workspace_bytes(rows, N);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return DSA_ERR_WORKSPACE;
  TopkWorkspace ws = topk_workspace(workspace, rows, N);
  return cuda_status(launch_topk(scores, B, T, N, q_pos0, k, idx, ws, false, stream));
}

dsa_status dsa_sparse_attn(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T, int N, int H,
                           int k, float scale, float* out, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
  if (!q || !kv || !idx || !out || !sizes_ok(B, T, N) || k <= 0 || H <= 0) return DSA_ERR_INVALID_ARG;
  if (k > DSA_MAX_TOPK || !heads_supported(H)) return DSA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(idx, 4) || !aligned(out, 16)) return DSA_ERR_INVALID_ARG;
  (void)workspace_bytes;
  AttnLayers layers{};
  layers.q[0] = q;
  layers.kv[0] = kv;
  layers.out[0] = out;
  return cuda_status(launch_sparse_attn_tc(layers, 1, idx, B, T, N, H, k, scale, workspace, false, stream));
}

dsa_status dsa_group_forward(const uint16_t* iq, const float* w, const uint16_t* ik, const uint16_t* const* q,
                             const uint16_t* const* kv, int L, int B, int T, int N, long long q_pos0, int H, int k,
                             float scale, int compute_indices, int32_t* idx_shared, float* const* out, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !kv || !out || !idx_shared || !sizes_ok(B, T, N) || k <= 0 || H <= 0 || L <= 0)
    return DSA_ERR_INVALID_ARG;
  if (L > DSA_MAX_LAYERS || k > DSA_MAX_TOPK || !heads_supported(H)) return DSA_ERR_UNSUPPORTED;
  if (compute_indices && (!iq || !w || !ik)) return DSA_ERR_INVALID_ARG;
  if (compute_indices && (!aligned(iq, 16) || !aligned(ik, 16) || !aligned(w, 16))) return DSA_ERR_INVALID_ARG;
  if (!aligned(idx_shared, 4)) return DSA_ERR_INVALID_ARG;
  AttnLayers layers{};
  for (int l = 0; l < L; ++l) {
    if (!q[l] || !kv[l] || !out[l]) return DSA_ERR_INVALID_ARG;
    if (!aligned(q[l], 16) || !aligned(kv[l], 16) || !aligned(out[l], 16)) return DSA_ERR_INVALID_ARG;
    layers.q[l] = q[l];
    layers.kv[l] = kv[l];
    layers.out[l] = out[l];
  }
  const GroupLayout g = group_layout(B, T, N, k, H, L);
  if (!workspace || workspace_bytes < g.total || !aligned(workspace, 256)) return DSA_ERR_WORKSPACE;
  unsigned char* base = static_cast<unsigned char*>(workspace);
  const long long rows = (long long)B * T;
  cudaError_t e;
  if (compute_indices) {
    TopkWorkspace tws = topk_workspace(base + g.topk_off, rows, N);
    float* scores = reinterpret_cast<float*>(base + g.scores_off);
    // in decode the indexer folds the first radix digit of the select into its epilogue
    const int sms = device_sm_count();
    if (sms <= 0) return cuda_status(cudaErrorInvalidDevice);
    const bool fused_hist = T == 1 && B <= sms;
    if (fused_hist && (e = cudaMemsetAsync(tws.hist, 0, tws.zero_bytes, stream)) != cudaSuccess)
      return cuda_status(e);
    if ((e = launch_index_score_tc(iq, w, ik, B, T, N, q_pos0, scores, fused_hist ? tws.hist : nullptr, stream)) !=
        cudaSuccess)
      return cuda_status(e);
    if ((e = launch_topk(scores, B, T, N, q_pos0, k, idx_shared, tws, fused_hist, stream)) != cudaSuccess)
      return cuda_status(e);
  }
  e = launch_sparse_attn_tc(layers, L, idx_shared, B, T, N, H, k, scale, base + g.attn_off,
                            /*q_early=*/compute_indices != 0, stream);
  return cuda_status(e);
}

}  // extern "C"
