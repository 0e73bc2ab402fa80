// indexer.cu -- lightweight indexer score I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s]).
//
// "GLM-5.2 1M architecture teardown", Cut 1: DSA -- before attention, a small indexer
// scores every history token (index_n_heads 32, index_head_dim 128) so that only the
// best index_topk of them are attended.
//
// Streaming design (decode, and the generic path for any T): every key is read from HBM
// exactly once per query, with 16-byte vector loads, and multiplied against the 32
// query heads on the tensor cores (m16n8k16, bf16 x bf16 -> f32).  A warp handles 16
// keys per step: M = 16 keys, N = 4 x 8 heads, K = 8 x 16 dims.  The head dimension is
// permuted identically in q and k (a dot product does not depend on the order of its
// terms) so that each lane's A fragments are four whole 16-byte chunks of a key row,
// loaded fully coalesced: lane (g, t) reads chunks 4j + t (j = 0..3) of rows g and g+8.
// The query fragments stay in registers for the whole kernel.  The epilogue applies
// ReLU and the head weights and reduces over the heads inside each 4-lane quad.
//
// The same kernel can fold the first radix digit of the top-k key into a per-row
// histogram (see topk.cu), so the select step need not re-read the scores to build it.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTileKeys = 16;

template <bool kHist>
__global__ void __launch_bounds__(kThreads, 2)
indexer_stream_kernel(const uint16_t* __restrict__ q, const float* __restrict__ w,
                      const uint16_t* __restrict__ k, int T, int N, long long q_pos0,
                      float* __restrict__ scores, uint32_t* __restrict__ hist) {
  const int row = blockIdx.x;  // b * T + t
  const int b = row / T;
  const int t = row - b * T;
  const long long vis = visible_count(N, q_pos0, t);
  const long long ntiles = (vis + kTileKeys - 1) / kTileKeys;

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;
  const int tq = lane & 3;

  __shared__ uint32_t s_hist[kHist ? kHistBins : 1];
  if (kHist) {
    for (int i = threadIdx.x; i < kHistBins; i += kThreads) s_hist[i] = 0;
    __syncthreads();
  }

  // Query fragments: head 8*nt + g, chunk 4*j + tq (8 dims = 16 bytes).
  const uint16_t* qrow = q + (size_t)row * kIndexHeads * kIndexDim;
  uint4 qf[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      qf[nt][j] = ld_nc_v4(qrow + (8 * nt + g) * kIndexDim + 8 * (4 * j + tq));
  float wv[4][2];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    wv[nt][0] = w[(size_t)row * kIndexHeads + 8 * nt + 2 * tq];
    wv[nt][1] = w[(size_t)row * kIndexHeads + 8 * nt + 2 * tq + 1];
  }

  const uint16_t* kb = k + (size_t)b * N * kIndexDim;
  float* srow = scores + (size_t)row * N;

  for (long long tile = (long long)blockIdx.y * kWarps + warp; tile < ntiles;
       tile += (long long)gridDim.y * kWarps) {
    const long long r0 = tile * kTileKeys + g;
    const long long r1 = r0 + 8;
    uint4 ka[4], kc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ka[j] = r0 < vis ? ld_stream_v4(kb + r0 * kIndexDim + 8 * (4 * j + tq)) : make_uint4(0, 0, 0, 0);
      kc[j] = r1 < vis ? ld_stream_v4(kb + r1 * kIndexDim + 8 * (4 * j + tq)) : make_uint4(0, 0, 0, 0);
    }
    float acc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t a0 = u ? ka[j].z : ka[j].x;
        const uint32_t a2 = u ? ka[j].w : ka[j].y;
        const uint32_t a1 = u ? kc[j].z : kc[j].x;
        const uint32_t a3 = u ? kc[j].w : kc[j].y;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const uint32_t b0 = u ? qf[nt][j].z : qf[nt][j].x;
          const uint32_t b1 = u ? qf[nt][j].w : qf[nt][j].y;
          mma_bf16_16816(acc[nt], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    float s_lo = 0.f, s_hi = 0.f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      s_lo = fmaf(wv[nt][0], fmaxf(acc[nt][0], 0.f), s_lo);
      s_lo = fmaf(wv[nt][1], fmaxf(acc[nt][1], 0.f), s_lo);
      s_hi = fmaf(wv[nt][0], fmaxf(acc[nt][2], 0.f), s_hi);
      s_hi = fmaf(wv[nt][1], fmaxf(acc[nt][3], 0.f), s_hi);
    }
    s_lo += __shfl_xor_sync(0xFFFFFFFFu, s_lo, 1);
    s_lo += __shfl_xor_sync(0xFFFFFFFFu, s_lo, 2);
    s_hi += __shfl_xor_sync(0xFFFFFFFFu, s_hi, 1);
    s_hi += __shfl_xor_sync(0xFFFFFFFFu, s_hi, 2);
    if (tq == 0 && r0 < vis) {
      srow[r0] = s_lo;
      if (kHist) atomicAdd(&s_hist[order_key(s_lo) >> kHistShift], 1u);
    }
    if (tq == 1 && r1 < vis) {
      srow[r1] = s_hi;
      if (kHist) atomicAdd(&s_hist[order_key(s_hi) >> kHistShift], 1u);
    }
  }

  if (kHist) {
    __syncthreads();
    uint32_t* grow = hist + (size_t)row * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += kThreads)
      if (s_hist[i]) atomicAdd(&grow[i], s_hist[i]);
  }
}

}  // namespace

cudaError_t launch_index_score(const uint16_t* q, const float* w, const uint16_t* k, int B, int T, int N,
                               long long q_pos0, float* scores, uint32_t* hist, cudaStream_t stream) {
  const long long rows = (long long)B * T;
  const long long vmax = visible_count(N, q_pos0, T - 1);
  const long long tiles = (vmax + kTileKeys - 1) / kTileKeys;
  long long per_row = (2LL * kNumSMs + rows - 1) / rows;  // about two CTAs per SM in total
  const long long need = (tiles + kWarps - 1) / kWarps;
  if (per_row > need) per_row = need;
  if (per_row < 1) per_row = 1;
  if (per_row > 65535) per_row = 65535;
  dim3 grid((unsigned)rows, (unsigned)per_row);
  if (hist)
    indexer_stream_kernel<true><<<grid, kThreads, 0, stream>>>(q, w, k, T, N, q_pos0, scores, hist);
  else
    indexer_stream_kernel<false><<<grid, kThreads, 0, stream>>>(q, w, k, T, N, q_pos0, scores, nullptr);
  return cudaGetLastError();
}

}  // namespace dsa
