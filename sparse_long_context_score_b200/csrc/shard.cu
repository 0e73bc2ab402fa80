// shard.cu -- the exchange steps of the context-sharded decode step.
//
// "Le contexte d'un million de tokens", Service efficace pour un million de contextes: a
// long context is spread over several GPUs.  Each GPU holds a contiguous range of the
// cached tokens, scores them and keeps its own top-k (a token in the row's top-k is in its
// shard's top-k); the candidates of all GPUs are exchanged and the k best of them are the
// row's index list; each GPU attends over the selected rows it holds, and the partial
// outputs combine exactly by their log-sum-exp:
//     out = sum_w exp(lse_w - LSE) out_w,   LSE = ln sum_w exp(lse_w).
// This file holds the three steps around the exchange:
//   candidates        a shard's top-k list -> (score, global position) pairs (a gather);
//   merge_candidates  the k best of the exchanged candidates of a row: radix select over
//                     the 64-bit composite (order key of the score, inverted position) in
//                     shared memory, one CTA per row; ties go to the lower position;
//   merge_partials    the log-sum-exp combination of the shards' partial outputs.
#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

__global__ void candidates_kernel(const float* __restrict__ scores, const int32_t* __restrict__ idx, long long rows,
                                  int Ns, int k, long long offset, float* __restrict__ cand_score,
                                  int32_t* __restrict__ cand_pos) {
  grid_dep_wait();
  const long long n = rows * k;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / k;
    const int j = idx[i];
    const bool v = j >= 0 && j < Ns;
    cand_score[i] = v ? scores[r * Ns + j] : -INFINITY;
    cand_pos[i] = v ? (int32_t)(j + offset) : -1;
  }
}

constexpr int kMT = 1024;                  // threads of the candidate merge
constexpr int kMaxCand = 8 * kMaxTopk;     // candidates of a row: up to 8 shards x 2048
constexpr int kMBits = 11;                 // radix digit width
constexpr int kMBins = 1 << kMBits;

struct MergeSmem {
  unsigned long long c[kMaxCand];  // composites; 0 = no candidate
  uint32_t hist[kMBins];
  uint32_t warp_tmp[32];
  uint32_t res[3];
};

// k best composites of a row (all > 0 when valid), output in candidate order (the valid
// positions increase along a row), then -1.  Candidate j of row r is entry (j / kc, r,
// j % kc) of the gathered [W][rows][kc] arrays (shard-major, as an all-gather leaves them).
__global__ void __launch_bounds__(kMT, 1)
merge_candidates_kernel(const float* __restrict__ cand_score, const int32_t* __restrict__ cand_pos, long long rows,
                        int kc, int M, int k, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  MergeSmem& sm = *reinterpret_cast<MergeSmem*>(smem_raw);
  grid_dep_wait();
  const long long row = blockIdx.x;
  auto at = [&](int j) { return ((long long)(j / kc) * rows + row) * kc + j % kc; };
  int32_t* out = idx + row * k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t nvalid = 0;
  for (int j = threadIdx.x; j < M; j += kMT) {
    const int32_t p = cand_pos[at(j)];
    const unsigned long long c = p >= 0 ? ((unsigned long long)order_key(cand_score[at(j)]) << 32) |
                                              (unsigned long long)(0xFFFFFFFFu - (uint32_t)p)
                                        : 0ull;
    sm.c[j] = c;
    nvalid += p >= 0 ? 1u : 0u;
  }
  // the threshold: the k-th largest composite (0 when there are no more than k candidates)
  unsigned long long thr = 0ull;
  {
    uint32_t x = nvalid;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    if (lane == 0) sm.warp_tmp[warp] = x;
    __syncthreads();
    uint32_t total = 0;
    for (int i = 0; i < kMT / 32; ++i) total += sm.warp_tmp[i];
    __syncthreads();
    if (total > (uint32_t)k) {
      unsigned long long prefix = 0ull;
      int pos = 64;
      uint32_t r = (uint32_t)k;  // rank still needed among the composites matching the prefix
      while (pos > 0) {
        const int width = pos >= kMBits ? kMBits : pos;
        const int shift = pos - width;
        const uint32_t mask = (1u << width) - 1u;
        for (int b = threadIdx.x; b < kMBins; b += kMT) sm.hist[b] = 0u;
        __syncthreads();
        for (int j = threadIdx.x; j < M; j += kMT) {
          const unsigned long long c = sm.c[j];
          if (c != 0ull && (pos == 64 || (c >> pos) == (prefix >> pos)))
            atomicAdd(&sm.hist[(uint32_t)(c >> shift) & mask], 1u);
        }
        __syncthreads();
        // bins from the top: this thread's two bins, then a CTA scan to the bin holding rank r
        const int nb = 1 << width;
        const int b0 = nb - 1 - 2 * (int)threadIdx.x;
        const uint32_t v0 = b0 >= 0 ? sm.hist[b0] : 0u, v1 = b0 - 1 >= 0 ? sm.hist[b0 - 1] : 0u;
        uint32_t s = v0 + v1, incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane == 31) sm.warp_tmp[warp] = incl;
        __syncthreads();
        uint32_t wbase = 0;
        for (int i = 0; i < warp; ++i) wbase += sm.warp_tmp[i];
        const uint32_t before = wbase + incl - s;  // composites in higher bins
        if (b0 >= 0 && before < r && before + v0 >= r) {
          sm.res[0] = (uint32_t)b0;
          sm.res[1] = before;
          sm.res[2] = v0;
        } else if (b0 - 1 >= 0 && before + v0 < r && before + v0 + v1 >= r) {
          sm.res[0] = (uint32_t)(b0 - 1);
          sm.res[1] = before + v0;
          sm.res[2] = v1;
        }
        __syncthreads();
        const uint32_t d = sm.res[0], above = sm.res[1], cnt = sm.res[2];
        __syncthreads();
        r -= above;
        prefix |= (unsigned long long)d << shift;
        pos = shift;
        if (cnt == r) break;  // every composite of this digit is selected
      }
      thr = prefix;  // the selected composites are exactly those >= prefix
    } else {
      thr = 1ull;    // every candidate
    }
  }
  // ordered compaction of the selected composites (positions increase along the row)
  uint32_t base = 0;
  for (int j0 = 0; j0 < M; j0 += kMT) {
    const int j = j0 + (int)threadIdx.x;
    const bool s = j < M && sm.c[j] >= thr;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, s);
    if (lane == 0) sm.warp_tmp[warp] = __popc(m);
    __syncthreads();
    uint32_t wbase = 0, tot = 0;
    for (int i = 0; i < kMT / 32; ++i) {
      if (i < warp) wbase += sm.warp_tmp[i];
      tot += sm.warp_tmp[i];
    }
    if (s) {
      const uint32_t o = base + wbase + __popc(m & ((1u << lane) - 1u));
      if (o < (uint32_t)k) out[o] = (int32_t)(0xFFFFFFFFu - (uint32_t)(sm.c[j] & 0xFFFFFFFFull));
    }
    base += tot;
    __syncthreads();
  }
  for (uint32_t j = base + threadIdx.x; j < (uint32_t)k; j += kMT) out[j] = -1;
}

// out = sum_w exp(lse_w - LSE) out_w over W shards; one thread per 4 value dims of a row
__global__ void merge_partials_kernel(const float* __restrict__ outs, const float* __restrict__ lses, int W,
                                      long long R, float* __restrict__ out) {
  grid_dep_wait();
  const long long n4 = R * (kDv / 4);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / (kDv / 4);
    float m = -INFINITY;
    for (int w = 0; w < W; ++w) m = fmaxf(m, lses[(long long)w * R + r]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m != -INFINITY) {
      float s = 0.f;
      for (int w = 0; w < W; ++w) s += expf(lses[(long long)w * R + r] - m);
      for (int w = 0; w < W; ++w) {
        const float c = expf(lses[(long long)w * R + r] - m) / s;
        const float4 v = reinterpret_cast<const float4*>(outs + (long long)w * R * kDv)[i];
        acc.x += c * v.x;
        acc.y += c * v.y;
        acc.z += c * v.z;
        acc.w += c * v.w;
      }
    }
    reinterpret_cast<float4*>(out)[i] = acc;
  }
}

int grid_of(long long n, int threads) {
  const int sms = device_sm_count();
  const long long want = (n + threads - 1) / threads;
  const long long cap = (long long)(sms > 0 ? sms : 148) * 8;
  return (int)(want < 1 ? 1 : want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_shard_candidates(const float* scores, const int32_t* idx, long long rows, int Ns, int k,
                                    long long offset, float* cand_score, int32_t* cand_pos, cudaStream_t stream) {
  candidates_kernel<<<grid_of(rows * k, 256), 256, 0, stream>>>(scores, idx, rows, Ns, k, offset, cand_score, cand_pos);
  return cudaGetLastError();
}

cudaError_t launch_merge_candidates(const float* cand_score, const int32_t* cand_pos, int W, long long rows, int kc,
                                    int k, int32_t* idx, cudaStream_t stream) {
  const int M = W * kc;
  if (M > kMaxCand || kc <= 0) return cudaErrorInvalidValue;
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    return cudaFuncSetAttribute(merge_candidates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(MergeSmem));
  });
  if (e != cudaSuccess) return e;
  merge_candidates_kernel<<<(unsigned)rows, kMT, sizeof(MergeSmem), stream>>>(cand_score, cand_pos, rows, kc, M, k, idx);
  return cudaGetLastError();
}

cudaError_t launch_merge_partials(const float* outs, const float* lses, int W, long long R, float* out,
                                  cudaStream_t stream) {
  merge_partials_kernel<<<grid_of(R * (kDv / 4), 256), 256, 0, stream>>>(outs, lses, W, R, out);
  return cudaGetLastError();
}

}  // namespace dsa
