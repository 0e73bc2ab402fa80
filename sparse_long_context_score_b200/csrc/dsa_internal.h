// dsa_internal.h -- constants and launch entry points shared by the libdsa sources.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include <atomic>

#include "dsa.h"

namespace dsa {

// Runs a set-up call (a kernel attribute) once per device, outside any stream capture
// that follows the first call on that device.
struct DeviceOnce {
  std::atomic<int> done[64] = {};
  template <class F>
  cudaError_t run(F f) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return f();
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = f();
    if (e == cudaSuccess) done[dev].store(1, std::memory_order_release);
    return e;
  }
};

// Device address of a file-scope __device__ int (an error word), looked up once per device
// with that device current.  Instantiate it in the file that defines the variable.
struct SymbolAddress {
  std::atomic<int*> ptr[64] = {};
  template <class Sym>
  cudaError_t get(const Sym& symbol, int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int* p = ptr[dev].load(std::memory_order_acquire);
    if (!p) {
      void* v = nullptr;
      if ((e = cudaGetSymbolAddress(&v, symbol)) != cudaSuccess) return e;
      p = static_cast<int*>(v);
      ptr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
  }
};

// SM count of the current device, read once per device (0 if it cannot be read)
int device_sm_count();

// DSA_OK for cudaSuccess; otherwise records `e` as the last CUDA error (dsa_last_cuda_error)
// and returns DSA_ERR_CUDA
dsa_status cuda_status(cudaError_t e);

constexpr int kIndexHeads = 32;   // index_n_heads
constexpr int kIndexDim = 128;    // index_head_dim
constexpr int kDqk = 576;         // compressed row: 512 latent + 64 rope
constexpr int kDv = 512;          // value = first 512 entries
constexpr int kMaxTopk = 2048;    // index_topk
constexpr int kMaxLayers = 8;

// top-k: first radix digit = the top 12 bits of the order key
constexpr int kHistBits = 12;
constexpr int kHistBins = 1 << kHistBits;
constexpr int kHistShift = 32 - kHistBits;
constexpr int kTopkChunk = 8192;       // scores per CTA in the scan kernels
constexpr int kCandCap = 8192;         // candidates kept per row for the resolve
constexpr int kHist2Bins = 1024;       // second radix digit: key bits 19..10
constexpr int kRowStateWords = 16;

struct TopkWorkspace {
  uint32_t* hist;        // [rows][kHistBins]
  uint32_t* row_state;   // [rows][kRowStateWords]
  uint32_t* chunk_sel;   // [rows][nchunks]  selected threshold-bin candidates per chunk
  uint32_t* hist2;       // [rows][kHist2Bins] next 10 key bits of the threshold-bin elements
  uint32_t* lvl;         // [rows][2][kHist2Bins] more digit histograms (one-launch select of long rows)
  uint32_t* chunk_above; // [rows][nchunks]  elements above the threshold bin per chunk
  uint32_t* chunk_off;   // [rows][nchunks]  output offset of each chunk
  uint64_t* cand;        // [rows][kCandCap] composite keys of threshold-bin elements
  size_t zero_bytes;     // bytes from hist that must be zero before a select
};

size_t topk_workspace_bytes(long long rows, int N);
TopkWorkspace topk_workspace(void* base, long long rows, int N);

struct AttnLayers {
  const uint16_t* q[kMaxLayers];
  const uint16_t* kv[kMaxLayers];
  float* out[kMaxLayers];
  float* lse[kMaxLayers];  // optional [rows][H] natural log-sum-exp of the logits (nullptr: none)
};

constexpr int kAttnTile = 64;  // selected rows per tile of the tensor-core attention (a split's granularity)

int attn_num_splits(long long rows, int L, int k, int sm_budget);
int attn_split_chunk(int k, int nsplit);
size_t attn_workspace_bytes(long long rows, int L, int H, int k, int sm_budget = 0);

// tcgen05 indexer (T == 1: decode, one query per MMA; T > 1: 8 queries per MMA).  With a
// histogram pointer (decode only, B no more than the SMs of the budget; zeroed by the
// caller) the first radix digit of the select is counted.
// f8: q and k hold E4M3 bytes instead of bf16 (the same layouts, one byte per element).
cudaError_t launch_index_score_tc(const void* q, const float* w, const void* k, int B, int T, int N, long long q_pos0,
                                  float* scores, uint32_t* hist, int sm_budget, bool f8, cudaStream_t stream);
// Device addresses of the error words: the indexer's and the attention's bounded waits
// record a code when they run out; the top-k records one when a selection invariant
// fails (the selected count is not k).  0 = none.
cudaError_t indexer_error_word(int** p);
cudaError_t attn_error_word(int** p);

// MTP verify step (verify.cu)
cudaError_t launch_verify(const float* p, const float* q, const int32_t* draft, const float* u, const float* u2, int B,
                          int S, int V, float* alpha, int32_t* accept, int32_t* token, int32_t* accepted_len,
                          cudaStream_t stream);
cudaError_t topk_error_word(int** p);

// Whether launch_topk takes the scan kernels for this shape (and so reads and writes the
// workspace): false when every row fits one cluster of CTAs on chip.
bool topk_uses_workspace(long long rows, long long vmax);

cudaError_t launch_topk(const float* scores, int B, int T, int N, long long q_pos0, int k, int32_t* idx,
                        const TopkWorkspace& ws, bool hist_ready, int sm_budget, cudaStream_t stream);
// top-k of rows short enough for one cluster of CTAs (topk_cluster.cu); launch_topk
// chooses it when topk_cluster_plan accepts the shape.  `hist` (nullable) holds the
// first digit's histogram per row, counted by the indexer.
bool topk_cluster_plan(long long rows, long long vmax, int sms, int* C, int* kpt);
cudaError_t launch_topk_cluster(const float* scores, int B, int T, int N, long long q_pos0, int k, int C, int kpt,
                                const uint32_t* hist, int32_t* idx, int* err, cudaStream_t stream);

// q_early: the kernel before it in the stream does not write the queries (it is the
// group's own top-k), so they are loaded before that kernel completes
// idx_offset: the cache holds global positions [idx_offset, idx_offset + N); selected
// positions outside it are skipped (a context shard)
// rows_once: the caller reads the selected rows once (a decode step), so they are gathered
// under an L2 evict-first policy; otherwise (MTP draft steps, prefill) they may stay in L2
// for the next call or the next query
cudaError_t launch_sparse_attn_tc(const AttnLayers& layers, int L, const int32_t* idx, int B, int T, int N, int H,
                                  int k, float scale, long long idx_offset, void* ws, size_t ws_bytes, bool q_early,
                                  bool rows_once, int sm_budget, cudaStream_t stream);

// context-sharded decode (shard.cu)
cudaError_t launch_shard_candidates(const float* scores, const int32_t* idx, long long rows, int Ns, int k,
                                    long long offset, float* cand_score, int32_t* cand_pos, cudaStream_t stream);
cudaError_t launch_merge_candidates(const float* cand_score, const int32_t* cand_pos, int W, long long rows, int kc,
                                    int k, int32_t* idx, cudaStream_t stream);
cudaError_t launch_merge_partials(const float* outs, const float* lses, int W, long long R, float* out,
                                  cudaStream_t stream);

}  // namespace dsa
