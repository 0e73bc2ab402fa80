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
// One CTA per draft position (32 warps).  Warp w streams its contiguous segment of the
// vocabulary once (coalesced 16-byte loads of p and q, four steps' loads in flight per
// thread), accumulating the acceptance rate and its residual weight, and keeps the
// residual weight of every chunk it reads (128 entries per warp step) in shared memory.  On a rejection the chunk sums locate the
// target to one chunk, and only that chunk is read again: the token is found a memory round
// trip after the stream, not a whole segment later.  A second, one-thread-per-sequence
// kernel counts the leading accepted positions.  HBM-bound: 8 B read per vocabulary entry
// and draft position.
#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kVThreads = 1024;
constexpr int kVWarps = kVThreads / 32;
// the chunk sums' shared memory: 8 B per chunk and warp, at most kVMaxChunks chunks per
// warp (192 KB in all); a chunk is one warp step of 128 entries (16-byte loads) or 32, or
// several steps for the largest vocabularies
constexpr int kVerifyMaxSmem = 196608;
constexpr int kVMaxChunks = kVerifyMaxSmem / (kVWarps * 8);

__device__ __forceinline__ uint64_t residual_weight(float p, float q) {
  const float r = p - q;
  return r > 0.f ? (uint64_t)(r * 1099511627776.0f) : 0ull;  // 2^40, truncated
}

// sum over the warp of v < 2^42 (four residual weights of a lane): two 32-bit warp
// reductions of its 24-bit halves, each sum below 2^29
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
  const uint32_t lo = __reduce_add_sync(0xFFFFFFFFu, (uint32_t)(v & 0xFFFFFFull));
  const uint32_t hi = __reduce_add_sync(0xFFFFFFFFu, (uint32_t)(v >> 24));
  return ((unsigned long long)hi << 24) + lo;
}

// A warp's segment (a multiple of 4 entries), its steps (128 entries with 16-byte loads,
// else 32), the steps per chunk and the chunks (the shared memory holds one weight per chunk
// and warp).
__host__ __device__ inline int verify_seg(int V) { return ((V + kVWarps - 1) / kVWarps + 3) & ~3; }
__host__ __device__ inline int verify_steps(int V, int vec) {
  const int cw = vec ? 128 : 32;
  return (verify_seg(V) + cw - 1) / cw;
}
__host__ __device__ inline int verify_spc(int V, int vec) {
  return (verify_steps(V, vec) + kVMaxChunks - 1) / kVMaxChunks;
}
__host__ __device__ inline int verify_chunks(int V, int vec) {
  const int spc = verify_spc(V, vec);
  return (verify_steps(V, vec) + spc - 1) / spc;
}

__global__ void __launch_bounds__(kVThreads)
verify_kernel(const float* __restrict__ p, const float* __restrict__ q, const int32_t* __restrict__ draft,
              const float* __restrict__ u, const float* __restrict__ u2, int V, int vec, float* __restrict__ alpha,
              int32_t* __restrict__ accept, int32_t* __restrict__ token) {
  __shared__ float s_alpha[kVWarps];
  __shared__ unsigned long long s_w[kVWarps];
  __shared__ int s_token;
  extern __shared__ unsigned long long s_cw[];  // [kVWarps][nchunk]: residual weight per chunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = blockIdx.x;
  const float* pr = p + r * V;
  const float* qr = q + r * V;
  // contiguous segment of this warp, a multiple of 4 entries long, read in chunks of cw
  // entries (one per warp step)
  const int seg = verify_seg(V);
  const int s0 = min(V, warp * seg), s1 = min(V, s0 + seg);
  const int cw = vec ? 128 : 32, nsteps = verify_steps(V, vec), spc = verify_spc(V, vec);
  const int nchunk = verify_chunks(V, vec);
  unsigned long long* cwarp = s_cw + (size_t)warp * nchunk;
  grid_dep_wait();
  float a = 0.f;
  unsigned long long w = 0ull;
  unsigned long long wc = 0ull;  // the current chunk's weight (lane 0)
  if (vec) {
    // four steps' loads issued together, then their arithmetic
    for (int c0 = 0; c0 < nsteps; c0 += 4) {
      float4 pv[4], qv[4];
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        const int i = s0 + (c0 + u4) * 128 + 4 * lane;
        if (c0 + u4 < nsteps && i < s1) {
          pv[u4] = __ldcs(reinterpret_cast<const float4*>(pr + i));
          qv[u4] = __ldcs(reinterpret_cast<const float4*>(qr + i));
        } else {
          pv[u4] = qv[u4] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        const int c = c0 + u4;
        if (c >= nsteps) break;
        a += fminf(pv[u4].x, qv[u4].x) + fminf(pv[u4].y, qv[u4].y) + fminf(pv[u4].z, qv[u4].z) +
             fminf(pv[u4].w, qv[u4].w);
        const unsigned long long wl = residual_weight(pv[u4].x, qv[u4].x) + residual_weight(pv[u4].y, qv[u4].y) +
                                      residual_weight(pv[u4].z, qv[u4].z) + residual_weight(pv[u4].w, qv[u4].w);
        w += wl;
        wc += warp_sum_u64(wl);
        if ((c + 1) % spc == 0 || c + 1 == nsteps) {
          if (lane == 0) cwarp[c / spc] = wc;
          wc = 0ull;
        }
      }
    }
  } else {
    for (int c = 0; c < nsteps; ++c) {
      const int i = s0 + c * 32 + lane;
      unsigned long long wl = 0ull;
      if (i < s1) {
        const float pv = __ldcs(pr + i), qv = __ldcs(qr + i);
        a += fminf(pv, qv);
        wl = residual_weight(pv, qv);
      }
      w += wl;
      wc += warp_sum_u64(wl);
      if ((c + 1) % spc == 0 || c + 1 == nsteps) {
        if (lane == 0) cwarp[c / spc] = wc;
        wc = 0ull;
      }
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
      // this warp's segment holds the target: its chunk from the chunk sums (32 at a time),
      // then the entry from that chunk, read again
      const unsigned long long* cs = s_cw + (size_t)ws * nchunk;
      int chunk = -1;
      for (int c0 = 0; c0 < nchunk && chunk < 0; c0 += 32) {
        const unsigned long long v = c0 + lane < nchunk ? cs[c0 + lane] : 0ull;
        unsigned long long incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned int hit = __ballot_sync(0xFFFFFFFFu, c0 + lane < nchunk && base + incl > T);
        if (hit) {
          const int h = __ffs(hit) - 1;
          chunk = c0 + h;
          base += __shfl_sync(0xFFFFFFFFu, incl - v, h);  // weight before the chunk
        } else {
          base += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
      }
      if (chunk >= 0) {
        // the chunk's steps, read again in order until the target is passed
        const int per = cw / 32;  // entries per lane and step: 4 (vec) or 1
        for (int c = chunk * spc; c < min(nsteps, (chunk + 1) * spc); ++c) {
          const int i = s0 + c * cw + per * lane;
          unsigned long long w4[4] = {0ull, 0ull, 0ull, 0ull};
          for (int e = 0; e < per; ++e) w4[e] = i + e < s1 ? residual_weight(pr[i + e], qr[i + e]) : 0ull;
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
              int t = i + per - 1;
              for (int e = 0; e < per; ++e) {
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
  const size_t smem = (size_t)kVWarps * verify_chunks(V, vec) * sizeof(unsigned long long);  // <= kVerifyMaxSmem
  static DeviceOnce once;
  cudaError_t e = once.run(
      [] { return cudaFuncSetAttribute(verify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kVerifyMaxSmem); });
  if (e != cudaSuccess) return e;
  verify_kernel<<<(unsigned)rows, kVThreads, smem, stream>>>(p, q, draft, u, u2, V, vec, alpha, accept, token);
  e = cudaGetLastError();
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
