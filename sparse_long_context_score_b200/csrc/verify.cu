// verify.cu -- the MTP verify step: rejection sampling of the draft tokens.
//
// "GLM-5.2 MTP IndexShare inference", Rejection Sampling: the acceptance rate of a draft
// token is the sum over the vocabulary of the smaller of the target and draft
// probabilities, sum_v min(p_v, q_v).  The accept / resample rule that has exactly that
// acceptance rate is standard speculative sampling: keep the draft token x iff
// u * q[x] < p[x] (u uniform in [0, 1)), else draw from the residual max(0, p - q).  The
// MTP pages verify the draft tokens in order and cut the sequence at the first rejection.
//
// Both decisions are integers and are taken exactly: the accept test is one float32
// product and comparison; the residual draw uses integer weights floor(max(0, p - q) *
// 2^40), their exact 64-bit sum S and target floor(floor(u2 * 2^24) * S / 2^24), and picks
// the first token whose inclusive prefix sum exceeds the target.
//
// One CTA per draft position (16 warps).  Warp w streams its contiguous segment of the
// vocabulary once (coalesced 16-byte loads of p and q), accumulating the acceptance rate
// and its residual weight; the CTA then knows the totals, and only on a rejection does the
// warp whose segment holds the target re-read that segment to find the token.  A second,
// one-thread-per-sequence kernel counts the leading accepted positions.  HBM-bound: 8 B
// read per vocabulary entry and draft position.
#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kVThreads = 512;
constexpr int kVWarps = kVThreads / 32;

__device__ __forceinline__ uint64_t residual_weight(float p, float q) {
  const float r = p - q;
  return r > 0.f ? (uint64_t)(r * 1099511627776.0f) : 0ull;  // 2^40, truncated
}

__global__ void __launch_bounds__(kVThreads)
verify_kernel(const float* __restrict__ p, const float* __restrict__ q, const int32_t* __restrict__ draft,
              const float* __restrict__ u, const float* __restrict__ u2, int V, int vec, float* __restrict__ alpha,
              int32_t* __restrict__ accept, int32_t* __restrict__ token) {
  __shared__ float s_alpha[kVWarps];
  __shared__ unsigned long long s_w[kVWarps];
  __shared__ int s_token;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = blockIdx.x;
  const float* pr = p + r * V;
  const float* qr = q + r * V;
  // contiguous segment of this warp, a multiple of 4 entries long
  const int seg = ((V + kVWarps - 1) / kVWarps + 3) & ~3;
  const int s0 = min(V, warp * seg), s1 = min(V, s0 + seg);
  grid_dep_wait();
  float a = 0.f;
  unsigned long long w = 0ull;
  if (vec) {
#pragma unroll 4
    for (int i = s0 + 4 * lane; i < s1; i += 128) {
      const float4 pv = __ldcs(reinterpret_cast<const float4*>(pr + i));
      const float4 qv = __ldcs(reinterpret_cast<const float4*>(qr + i));
      a += fminf(pv.x, qv.x) + fminf(pv.y, qv.y) + fminf(pv.z, qv.z) + fminf(pv.w, qv.w);
      w += residual_weight(pv.x, qv.x) + residual_weight(pv.y, qv.y) + residual_weight(pv.z, qv.z) +
           residual_weight(pv.w, qv.w);
    }
  } else {
    for (int i = s0 + lane; i < s1; i += 32) {
      const float pv = __ldcs(pr + i), qv = __ldcs(qr + i);
      a += fminf(pv, qv);
      w += residual_weight(pv, qv);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
    w += __shfl_xor_sync(0xFFFFFFFFu, w, o);
  }
  if (lane == 0) {
    s_alpha[warp] = a;
    s_w[warp] = w;
  }
  if (threadIdx.x == 0) s_token = -1;
  __syncthreads();
  const int x = draft[r];
  const bool x_ok = x >= 0 && x < V;  // an out-of-range draft token is rejected and not replaced
  // the decisions, taken by every thread from the same shared values
  float at = 0.f;
  unsigned long long S = 0ull;
#pragma unroll
  for (int i = 0; i < kVWarps; ++i) {
    at += s_alpha[i];
    S += s_w[i];
  }
  const bool acc = x_ok && u[r] * qr[x] < pr[x];
  if (x_ok && !acc && S > 0ull) {
    const unsigned long long u24 = (unsigned long long)(u2[r] * 16777216.0f);  // 2^24
    const unsigned long long hi = __umul64hi(u24, S), lo = u24 * S;
    const unsigned long long T = (hi << 40) | (lo >> 24);                   // floor(u24 * S / 2^24)
    unsigned long long base = 0ull;
    int ws = kVWarps - 1;
    for (int i = 0; i < kVWarps; ++i) {
      if (base + s_w[i] > T) {
        ws = i;
        break;
      }
      base += s_w[i];
    }
    if (warp == ws) {
      // this warp's segment holds the target: find the entry, 128 at a time
      for (int i0 = s0; i0 < s1; i0 += 128) {
        const int i = i0 + 4 * lane;
        unsigned long long w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w4[e] = i + e < s1 ? residual_weight(pr[i + e], qr[i + e]) : 0ull;
        const unsigned long long lsum = w4[0] + w4[1] + w4[2] + w4[3];
        unsigned long long incl = lsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned int hit = __ballot_sync(0xFFFFFFFFu, base + incl > T);
        if (hit) {
          if (lane == __ffs(hit) - 1) {
            unsigned long long run = base + incl - lsum;
            int t = i + 3;
            for (int e = 0; e < 4; ++e) {
              run += w4[e];
              if (run > T) {
                t = i + e;
                break;
              }
            }
            s_token = t;
          }
          break;
        }
        base += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    alpha[r] = at;
    accept[r] = acc ? 1 : 0;
    token[r] = !x_ok ? -1 : (acc || s_token < 0) ? x : s_token;
  }
}

// accepted_len[b]: the leading accepted positions of sequence b
__global__ void verify_len_kernel(const int32_t* __restrict__ accept, int B, int S, int32_t* __restrict__ accepted_len) {
  grid_dep_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int n = 0;
  while (n < S && accept[(long long)b * S + n]) ++n;
  accepted_len[b] = n;
}

}  // namespace

cudaError_t launch_verify(const float* p, const float* q, const int32_t* draft, const float* u, const float* u2, int B,
                          int S, int V, float* alpha, int32_t* accept, int32_t* token, int32_t* accepted_len,
                          cudaStream_t stream) {
  const long long rows = (long long)B * S;
  const int vec = (V % 4 == 0) && ((reinterpret_cast<uintptr_t>(p) | reinterpret_cast<uintptr_t>(q)) % 16 == 0);
  verify_kernel<<<(unsigned)rows, kVThreads, 0, stream>>>(p, q, draft, u, u2, V, vec, alpha, accept, token);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((B + 127) / 128));
  cfg.blockDim = dim3(128);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // waits in-kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, verify_len_kernel, (const int32_t*)accept, B, S, accepted_len);
}

}  // namespace dsa
