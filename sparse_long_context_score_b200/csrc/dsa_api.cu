// dsa_api.cu -- the C ABI of libdsa: argument checks, workspace layout, launch order.
//
// The IndexShare group driver follows "GLM-5.2 1M architecture teardown", Cut 2:
// IndexShare (the indexer runs in the first of every 4 layers and its top-k list is used
// by all 4) and "GLM-5.2 MTP IndexShare inference", Indexer Share in the MTP layer (draft
// steps 2.. reuse the step-1 index list, so draft-token rows are never attended; the MTP
// layer reads the target cache -- KV Share).
#include <cstdio>
#include <vector>

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
  int chunk;  // query rows (of one sequence) per indexer + select pass; T: the whole plane at once
};

// Workspace of a group call: the select's workspace and the score plane for `chunk` query
// rows of one sequence at a time (chunk == T: all B x T rows in one pass), and the
// attention's split partials for all rows.
GroupLayout group_layout(int B, int T, int N, int k, int H, int L, int chunk) {
  const long long rows = chunk >= T ? (long long)B * T : (long long)chunk;
  GroupLayout g;
  g.chunk = chunk >= T ? T : chunk;
  g.topk_off = 0;
  g.topk_bytes = round256(topk_workspace_bytes(rows, N));
  g.scores_off = g.topk_off + g.topk_bytes;
  g.scores_bytes = round256((size_t)rows * N * sizeof(float));
  g.attn_off = g.scores_off + g.scores_bytes;
  g.attn_bytes = round256(attn_workspace_bytes((long long)B * T, L, H, k));
  g.total = g.attn_off + g.attn_bytes;
  return g;
}
GroupLayout group_layout(int B, int T, int N, int k, int H, int L) { return group_layout(B, T, N, k, H, L, T); }

// Query rows per pass when the score plane is processed in chunks: a multiple of 8 (the
// prefill indexer's query group), and no fewer than 8 unless T is.
constexpr int kChunkQuantum = 8;
int min_chunk(int T) { return T < kChunkQuantum ? T : kChunkQuantum; }

// The layout a workspace of `bytes` allows: the whole plane when it fits, else the largest
// chunk that does (chunk == 0: not even the smallest).  Decode (T == 1) never chunks.
GroupLayout layout_for(int B, int T, int N, int k, int H, int L, size_t bytes) {
  GroupLayout g = group_layout(B, T, N, k, H, L);
  if (bytes >= g.total || T == 1) return g;
  int lo = min_chunk(T), hi = T - 1;
  GroupLayout best = group_layout(B, T, N, k, H, L, lo);
  if (best.total > bytes) {
    best.chunk = 0;
    return best;
  }
  while (lo < hi) {  // the largest multiple of 8 below T that fits (the total grows with the chunk)
    const int mid = ((lo + hi + 1) / 2) / kChunkQuantum * kChunkQuantum;
    if (mid <= lo) break;
    const GroupLayout m = group_layout(B, T, N, k, H, L, mid);
    if (m.total <= bytes) {
      lo = mid;
      best = m;
    } else {
      hi = mid - 1;
    }
  }
  return best;
}

bool heads_supported(int H) { return H == 16 || H == 32 || H == 48 || H == 64; }

// One group call, checked.
struct GroupCall {
  const void* iq;  // bf16 or (f8) E4M3 elements
  const float* w;
  const void* ik;
  bool f8;
  AttnLayers layers;
  int L, B, T, N, H, k, compute_indices;
  long long q_pos0;
  float scale;
  int32_t* idx;
  bool rows_once = false;  // the attention's rows are read once (a decode step)
};

dsa_status check_group(const void* iq, const float* w, const void* ik, bool f8, const uint16_t* const* q,
                       const uint16_t* const* kv, int L, int B, int T, int N, int H, int k, int compute_indices,
                       int32_t* idx_shared, float* const* out, GroupCall* c) {
  if (!q || !kv || !out || !idx_shared || !sizes_ok(B, T, N) || k <= 0 || H <= 0 || L <= 0)
    return DSA_ERR_INVALID_ARG;
  if (L > DSA_MAX_LAYERS || k > DSA_MAX_TOPK || !heads_supported(H)) return DSA_ERR_UNSUPPORTED;
  if (compute_indices && (!iq || !w || !ik)) return DSA_ERR_INVALID_ARG;
  if (compute_indices && (!aligned(iq, 16) || !aligned(ik, 16) || !aligned(w, 16))) return DSA_ERR_INVALID_ARG;
  if (!aligned(idx_shared, 4)) return DSA_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l) {
    if (!q[l] || !kv[l] || !out[l]) return DSA_ERR_INVALID_ARG;
    if (!aligned(q[l], 16) || !aligned(kv[l], 16) || !aligned(out[l], 16)) return DSA_ERR_INVALID_ARG;
    c->layers.q[l] = q[l];
    c->layers.kv[l] = kv[l];
    c->layers.out[l] = out[l];
  }
  c->iq = iq;
  c->w = w;
  c->ik = ik;
  c->f8 = f8;
  c->L = L;
  c->B = B;
  c->T = T;
  c->N = N;
  c->H = H;
  c->k = k;
  c->compute_indices = compute_indices;
  c->idx = idx_shared;
  return DSA_OK;
}

// Enqueues one group on `stream`: the indexer (after `before`, if given; on at most idx_sms
// SMs; `after_idx` recorded behind it, if given), then the top-k and the attention (on at
// most tail_sms SMs).  A budget of 0 means all SMs.
cudaError_t enqueue_group(const GroupCall& c, unsigned char* base, const GroupLayout& g, int idx_sms, int tail_sms,
                          cudaEvent_t before, cudaEvent_t after_idx, cudaStream_t stream) {
  const long long rows = (long long)c.B * c.T;
  cudaError_t e;
  if (before && (e = cudaStreamWaitEvent(stream, before, 0)) != cudaSuccess) return e;
  if (c.compute_indices && g.chunk < c.T) {
    // the score plane in chunks of query rows of one sequence, each scored and selected
    // before the next (the chunk's plane is reused, and stays in L2 when it fits)
    float* scores = reinterpret_cast<float*>(base + g.scores_off);
    const size_t esz = c.f8 ? 1 : 2;
    for (int b = 0; b < c.B; ++b)
      for (int t0 = 0; t0 < c.T; t0 += g.chunk) {
        const int tn = c.T - t0 < g.chunk ? c.T - t0 : g.chunk;
        const size_t r0 = (size_t)b * c.T + t0;
        TopkWorkspace tws = topk_workspace(base + g.topk_off, tn, c.N);
        if ((e = launch_index_score_tc(static_cast<const unsigned char*>(c.iq) + r0 * kIndexHeads * kIndexDim * esz,
                                       c.w + r0 * kIndexHeads,
                                       static_cast<const unsigned char*>(c.ik) + (size_t)b * c.N * kIndexDim * esz, 1,
                                       tn, c.N, c.q_pos0 + t0, scores, nullptr, idx_sms, c.f8, stream)) != cudaSuccess)
          return e;
        if ((e = launch_topk(scores, 1, tn, c.N, c.q_pos0 + t0, c.k, c.idx + r0 * c.k, tws, false, tail_sms, stream)) !=
            cudaSuccess)
          return e;
      }
    if (after_idx && (e = cudaEventRecord(after_idx, stream)) != cudaSuccess) return e;
  } else if (c.compute_indices) {
    TopkWorkspace tws = topk_workspace(base + g.topk_off, rows, c.N);
    float* scores = reinterpret_cast<float*>(base + g.scores_off);
    // in decode the indexer folds the first radix digit of the select into its epilogue
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const int cap = idx_sms > 0 && idx_sms < sms ? idx_sms : sms;
    const bool fused_hist = c.T == 1 && c.B <= cap;
    if (fused_hist && (e = cudaMemsetAsync(tws.hist, 0, tws.zero_bytes, stream)) != cudaSuccess) return e;
    if ((e = launch_index_score_tc(c.iq, c.w, c.ik, c.B, c.T, c.N, c.q_pos0, scores, fused_hist ? tws.hist : nullptr,
                                   idx_sms, c.f8, stream)) != cudaSuccess)
      return e;
    if (after_idx && (e = cudaEventRecord(after_idx, stream)) != cudaSuccess) return e;
    if ((e = launch_topk(scores, c.B, c.T, c.N, c.q_pos0, c.k, c.idx, tws, fused_hist, tail_sms, stream)) != cudaSuccess)
      return e;
  }
  return launch_sparse_attn_tc(c.layers, c.L, c.idx, c.B, c.T, c.N, c.H, c.k, c.scale, 0, base + g.attn_off, g.attn_bytes,
                               /*q_early=*/c.compute_indices != 0, c.rows_once, tail_sms, stream);
}

// Events of dsa_decode_step, created once per device and host thread.
struct DecodeEvents {
  cudaEvent_t fork = nullptr, join = nullptr, idx[2] = {nullptr, nullptr};
};

DecodeEvents* decode_events() {
  thread_local DecodeEvents ev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  DecodeEvents& d = ev[dev];
  if (!d.fork) {
    cudaEvent_t* all[4] = {&d.fork, &d.join, &d.idx[0], &d.idx[1]};
    for (cudaEvent_t* x : all)
      if (cudaEventCreateWithFlags(x, cudaEventDisableTiming) != cudaSuccess) return nullptr;
  }
  return &d;
}

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

size_t dsa_workspace_size_min(int B, int T, int N, int k, int H, int L) {
  if (!sizes_ok(B, T, N) || k <= 0 || k > DSA_MAX_TOPK || H <= 0 || L <= 0 || L > DSA_MAX_LAYERS) return 0;
  if (T == 1) return group_layout(B, T, N, k, H, L).total;
  const size_t whole = group_layout(B, T, N, k, H, L).total, chunked = group_layout(B, T, N, k, H, L, min_chunk(T)).total;
  return chunked < whole ? chunked : whole;
}

dsa_status dsa_index_score(const uint16_t* q, const float* w, const uint16_t* k, int B, int T, int N,
                           long long q_pos0, float* scores, cudaStream_t stream) {
  if (!q || !w || !k || !scores || !sizes_ok(B, T, N)) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(w, 16) || !aligned(scores, 4)) return DSA_ERR_INVALID_ARG;
  return cuda_status(launch_index_score_tc(q, w, k, B, T, N, q_pos0, scores, nullptr, 0, false, stream));
}

dsa_status dsa_index_score_e4m3(const uint8_t* q, const float* w, const uint8_t* k, int B, int T, int N,
                                long long q_pos0, float* scores, cudaStream_t stream) {
  if (!q || !w || !k || !scores || !sizes_ok(B, T, N)) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(w, 16) || !aligned(scores, 4)) return DSA_ERR_INVALID_ARG;
  return cuda_status(launch_index_score_tc(q, w, k, B, T, N, q_pos0, scores, nullptr, 0, true, stream));
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
  return cuda_status(launch_topk(scores, B, T, N, q_pos0, k, idx, ws, false, 0, stream));
}

dsa_status dsa_sparse_attn(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T, int N, int H,
                           int k, float scale, float* out, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
  if (!q || !kv || !idx || !out || !sizes_ok(B, T, N) || k <= 0 || H <= 0) return DSA_ERR_INVALID_ARG;
  if (k > DSA_MAX_TOPK || !heads_supported(H)) return DSA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(idx, 4) || !aligned(out, 16)) return DSA_ERR_INVALID_ARG;
  const size_t need = attn_workspace_bytes((long long)B * T, 1, H, k);
  if (need && (!workspace || workspace_bytes < need || !aligned(workspace, 256))) return DSA_ERR_WORKSPACE;
  AttnLayers layers{};
  layers.q[0] = q;
  layers.kv[0] = kv;
  layers.out[0] = out;
  return cuda_status(
      launch_sparse_attn_tc(layers, 1, idx, B, T, N, H, k, scale, 0, workspace, workspace_bytes, false, false, 0, stream));
}

dsa_status dsa_group_forward(const uint16_t* iq, const float* w, const uint16_t* ik, const uint16_t* const* q,
                             const uint16_t* const* kv, int L, int B, int T, int N, long long q_pos0, int H, int k,
                             float scale, int compute_indices, int32_t* idx_shared, float* const* out, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  GroupCall c{};
  const dsa_status st = check_group(iq, w, ik, false, q, kv, L, B, T, N, H, k, compute_indices, idx_shared, out, &c);
  if (st != DSA_OK) return st;
  c.q_pos0 = q_pos0;
  c.scale = scale;
  // a workspace smaller than dsa_workspace_size (down to dsa_workspace_size_min) scores and
  // selects the query rows in chunks
  const GroupLayout g = layout_for(B, T, N, k, H, L, workspace_bytes);
  if (!workspace || g.chunk == 0 || workspace_bytes < g.total || !aligned(workspace, 256)) return DSA_ERR_WORKSPACE;
  return cuda_status(enqueue_group(c, static_cast<unsigned char*>(workspace), g, 0, 0, nullptr, nullptr, stream));
}

size_t dsa_decode_workspace_size(int B, int N, int k, int H, int L) {
  if (!sizes_ok(B, 1, N) || k <= 0 || k > DSA_MAX_TOPK || H <= 0 || L <= 0 || L > DSA_MAX_LAYERS) return 0;
  const int B0 = (B + 1) / 2, B1 = B - B0;
  size_t n = round256(group_layout(B0, 1, N, k, H, L).total);
  if (B1 > 0) n += group_layout(B1, 1, N, k, H, L).total;
  const size_t whole = group_layout(B, 1, N, k, H, L).total;  // the in-order step (side == stream)
  return n > whole ? n : whole;
}

dsa_status dsa_decode_step(const dsa_group_io* groups, int G, int L, int B, int N, int H, int k, float scale,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream, cudaStream_t side) {
  if (!groups || G <= 0 || !sizes_ok(B, 1, N)) return DSA_ERR_INVALID_ARG;
  // side == stream: the whole batch runs its groups in order on `stream`
  const int B0 = side == stream ? B : (B + 1) / 2, B1 = B - B0;
  const GroupLayout g0 = group_layout(B0, 1, N, k, H, L);
  const GroupLayout g1 = group_layout(B1 > 0 ? B1 : 1, 1, N, k, H, L);
  const size_t off1 = round256(g0.total);
  const size_t need = B1 > 0 ? off1 + g1.total : g0.total;
  // every group's arguments are checked before anything is enqueued
  std::vector<GroupCall> calls((size_t)G * 2);
  for (int gi = 0; gi < G; ++gi) {
    const dsa_group_io& io = groups[gi];
    for (int mb = 0; mb < 2; ++mb) {
      const int b0 = mb ? B0 : 0, bn = mb ? B1 : B0;
      GroupCall& c = calls[(size_t)gi * 2 + mb];
      if (bn == 0) continue;
      const uint16_t* qs[DSA_MAX_LAYERS];
      const uint16_t* kvs[DSA_MAX_LAYERS];
      float* outs[DSA_MAX_LAYERS];
      if (L <= 0 || L > DSA_MAX_LAYERS) return L <= 0 ? DSA_ERR_INVALID_ARG : DSA_ERR_UNSUPPORTED;
      for (int l = 0; l < L; ++l) {
        if (!io.q[l] || !io.kv[l] || !io.out[l]) return DSA_ERR_INVALID_ARG;
        qs[l] = io.q[l] + (size_t)b0 * H * kDqk;
        kvs[l] = io.kv[l] + (size_t)b0 * N * kDqk;
        outs[l] = io.out[l] + (size_t)b0 * H * kDv;
      }
      if (!io.iq || !io.w || !io.ik || !io.idx) return DSA_ERR_INVALID_ARG;
      if (io.index_format != DSA_INDEX_BF16 && io.index_format != DSA_INDEX_E4M3) return DSA_ERR_UNSUPPORTED;
      const bool f8 = io.index_format == DSA_INDEX_E4M3;
      const size_t esz = f8 ? 1 : 2;
      const dsa_status st =
          check_group(static_cast<const unsigned char*>(io.iq) + (size_t)b0 * kIndexHeads * kIndexDim * esz,
                      io.w + (size_t)b0 * kIndexHeads,
                      static_cast<const unsigned char*>(io.ik) + (size_t)b0 * N * kIndexDim * esz, f8, qs, kvs, L, bn,
                      1, N, H, k, 1, io.idx + (size_t)b0 * k, outs, &c);
      if (st != DSA_OK) return st;
      c.q_pos0 = N - 1;
      c.scale = scale;
      c.rows_once = true;
    }
  }
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return DSA_ERR_WORKSPACE;
  unsigned char* base = static_cast<unsigned char*>(workspace);
  cudaError_t e;
  if (B1 == 0) {  // one sequence: nothing to overlap
    for (int gi = 0; gi < G; ++gi)
      if ((e = enqueue_group(calls[(size_t)gi * 2], base, g0, 0, 0, nullptr, nullptr, stream)) != cudaSuccess)
        return cuda_status(e);
    return DSA_OK;
  }
  const int sms = device_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorInvalidDevice);
  // The indexer keeps HBM near its peak on three quarters of the SMs; the other
  // micro-batch's top-k and attention run beside it on the rest (measured on B200 at 1M
  // contexts: a quarter of the SMs for them 871 us per step, a third 893, a fifth 886-893,
  // two fifths 934).
  const int tail_sms = sms / 4, idx_sms = sms - tail_sms;
  DecodeEvents* ev = decode_events();
  if (!ev) return cuda_status(cudaErrorInvalidDevice);
  if ((e = cudaEventRecord(ev->fork, stream)) != cudaSuccess || (e = cudaStreamWaitEvent(side, ev->fork, 0)) != cudaSuccess)
    return cuda_status(e);
  for (int gi = 0; gi < G; ++gi) {
    for (int mb = 0; mb < 2; ++mb) {
      const bool first = gi == 0 && mb == 0, last = gi == G - 1 && mb == 1;
      // indexers alternate (each waits for the previous one); the first runs alone, and
      // the last micro-batch's last top-k and attention run alone
      e = enqueue_group(calls[(size_t)gi * 2 + mb], base + (mb ? off1 : 0), mb ? g1 : g0, first ? sms : idx_sms,
                        last ? sms : tail_sms, first ? nullptr : ev->idx[1 - mb], ev->idx[mb], mb ? side : stream);
      if (e != cudaSuccess) return cuda_status(e);
    }
  }
  if ((e = cudaEventRecord(ev->join, side)) != cudaSuccess || (e = cudaStreamWaitEvent(stream, ev->join, 0)) != cudaSuccess)
    return cuda_status(e);
  return DSA_OK;
}

dsa_status dsa_sparse_attn_shard(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T, int N,
                                 long long offset, int H, int k, float scale, float* out, float* lse, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !kv || !idx || !out || !lse || !sizes_ok(B, T, N) || k <= 0 || H <= 0 || offset < 0)
    return DSA_ERR_INVALID_ARG;
  if (k > DSA_MAX_TOPK || !heads_supported(H)) return DSA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(idx, 4) || !aligned(out, 16) || !aligned(lse, 4))
    return DSA_ERR_INVALID_ARG;
  const size_t need = attn_workspace_bytes((long long)B * T, 1, H, k);
  if (need && (!workspace || workspace_bytes < need || !aligned(workspace, 256))) return DSA_ERR_WORKSPACE;
  AttnLayers layers{};
  layers.q[0] = q;
  layers.kv[0] = kv;
  layers.out[0] = out;
  layers.lse[0] = lse;
  return cuda_status(
      launch_sparse_attn_tc(layers, 1, idx, B, T, N, H, k, scale, offset, workspace, workspace_bytes, false, false, 0, stream));
}

dsa_status dsa_shard_candidates(const float* scores, const int32_t* idx, int B, int T, int N, int k, long long offset,
                                float* cand_score, int32_t* cand_pos, cudaStream_t stream) {
  if (!scores || !idx || !cand_score || !cand_pos || !sizes_ok(B, T, N) || k <= 0 || offset < 0 ||
      offset + N > 0x7FFFFFFFLL)
    return DSA_ERR_INVALID_ARG;
  return cuda_status(launch_shard_candidates(scores, idx, (long long)B * T, N, k, offset, cand_score, cand_pos, stream));
}

dsa_status dsa_merge_candidates(const float* cand_score, const int32_t* cand_pos, int W, int B, int T, int kc, int k,
                                int32_t* idx, cudaStream_t stream) {
  if (!cand_score || !cand_pos || !idx || W <= 0 || B < 0 || T < 0 || kc <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (k > DSA_MAX_TOPK || (long long)W * kc > 8 * DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if ((long long)B * T == 0) return DSA_OK;
  return cuda_status(launch_merge_candidates(cand_score, cand_pos, W, (long long)B * T, kc, k, idx, stream));
}

dsa_status dsa_merge_partials(const float* outs, const float* lses, int W, int B, int T, int H, float* out,
                              cudaStream_t stream) {
  if (!outs || !lses || !out || W <= 0 || B < 0 || T < 0 || H <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned(outs, 16) || !aligned(out, 16) || !aligned(lses, 4)) return DSA_ERR_INVALID_ARG;
  const long long R = (long long)B * T * H;
  if (R == 0) return DSA_OK;
  return cuda_status(launch_merge_partials(outs, lses, W, R, out, stream));
}

dsa_status dsa_verify(const float* p, const float* q, const int32_t* draft, const float* u, const float* u2, int B,
                      int S, int V, float* alpha, int32_t* accept, int32_t* token, int32_t* accepted_len,
                      cudaStream_t stream) {
  if (!p || !q || !draft || !u || !u2 || !alpha || !accept || !token || !accepted_len) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || S <= 0 || V <= 0 || V >= (1 << 24) || (long long)B * S > 0x7FFFFFFFLL) return DSA_ERR_INVALID_ARG;
  if (!aligned(p, 4) || !aligned(q, 4) || !aligned(alpha, 4) || !aligned(draft, 4) || !aligned(u, 4) ||
      !aligned(u2, 4) || !aligned(accept, 4) || !aligned(token, 4) || !aligned(accepted_len, 4))
    return DSA_ERR_INVALID_ARG;
  return cuda_status(launch_verify(p, q, draft, u, u2, B, S, V, alpha, accept, token, accepted_len, stream));
}

}  // extern "C"
