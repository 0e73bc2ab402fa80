// attn.cu -- sparse MLA attention over the top-k selected compressed rows.
//
// "GLM-5.2 1M architecture teardown", Cut 1: DSA -- full attention runs only over the
// 2048 tokens the indexer kept; Cut 3: MLA -- each token's cache entry is one compressed
// row (512 latent, plus the 64-wide rope part), shared by all 64 heads.  In the absorbed
// form used here a head's logit is scale * q[h] . c[idx_j] over the 576-wide row and the
// value is the row's first 512 entries.
//
// One CTA handles one (query row, layer, key split).  The selected rows are gathered
// with 16-byte cp.async into a 3-stage shared-memory ring (32 rows per stage, XOR-swizzled
// 16-byte chunks so that ldmatrix is conflict-free); the queries of all heads stay in
// shared memory.  S = Q K^T and O = P V run on the tensor cores (m16n8k16, bf16 in, f32
// accumulate) with an online softmax in f32 (base-2 exponent, scale folded into the
// logits).  Warp w owns output columns [64w, 64w+64) for every head; the softmax row
// statistics are exchanged through shared memory.  With more than one split per
// (row, layer) each CTA writes an unnormalised partial (O, m, l) and a combine kernel
// merges them.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kThreads = 256;
constexpr int kBc = 32;                     // gathered rows per pipeline stage
constexpr int kStages = 3;
constexpr int kRowBytes = kDqk * 2;          // 1152
constexpr int kRowChunks = kDqk / 8;         // 72 chunks of 16 bytes
constexpr int kKSteps = kDqk / 16;           // 36
constexpr int kMaxHeads = 64;
constexpr int kMaxChunkKeys = kMaxTopk;

constexpr int kQBytes = kMaxHeads * kRowBytes;          // 73728
constexpr int kStageBytes = kBc * kRowBytes;            // 36864
constexpr int kPBytes = kMaxHeads * kBc * 2;            // 4096
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffP = kOffKV + kStages * kStageBytes;
constexpr int kOffIdx = kOffP + kPBytes;
constexpr int kOffRed = kOffIdx + kMaxChunkKeys * 4;
constexpr int kSmemBytes = kOffRed + (2 * kMaxHeads + kMaxHeads + 2 * kMaxHeads + kMaxHeads) * 4;

// byte offset of element (row, col) (col a multiple of 8) in a [rows][576] bf16 tile
__device__ __forceinline__ uint32_t swz576(int row, int col) {
  const int c = col >> 3;
  return (uint32_t)(row * kRowBytes + (((c & ~7) | ((c ^ row) & 7)) << 4));
}
// byte offset of element (row, col) (col a multiple of 8) in the [64][32] bf16 P tile
__device__ __forceinline__ uint32_t swzP(int row, int col) {
  const int c = col >> 3;
  return (uint32_t)(row * 64 + ((c ^ ((row >> 1) & 3)) << 4));
}

template <int MT>  // MT = heads / 16
__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_kernel(AttnLayers layers, const int32_t* __restrict__ idx, int T, int N, int k, int chunk,
                   float scale_log2, float* __restrict__ partial) {
  constexpr int H = MT * 16;
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sQ = smem_u32(smem + kOffQ);
  const uint32_t sKV = smem_u32(smem + kOffKV);
  const uint32_t sP = smem_u32(smem + kOffP);
  int* s_idx = reinterpret_cast<int*>(smem + kOffIdx);
  float* red_max = reinterpret_cast<float*>(smem + kOffRed);  // [2][64]
  float* alpha_s = red_max + 2 * kMaxHeads;                   // [64]
  float* lsum_s = alpha_s + kMaxHeads;                        // [2][64]
  float* m_s = lsum_s + 2 * kMaxHeads;                        // [64]

  const int split = blockIdx.x;
  const int row = blockIdx.y;
  const int layer = blockIdx.z;
  const int nsplit = gridDim.x;
  const int b = row / T;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;

  const uint16_t* qp = layers.q[layer] + (size_t)row * H * kDqk;
  const uint16_t* kvb = layers.kv[layer] + (size_t)b * N * kDqk;
  const int j0 = split * chunk;
  const int j1 = min(j0 + chunk, k);
  const int nkeys = max(j1 - j0, 0);
  const int ntiles = (nkeys + kBc - 1) / kBc;

  // selected rows of this split; out-of-range entries are treated as empty
  for (int j = tid; j < ntiles * kBc; j += kThreads) {
    int v = -1;
    if (j < nkeys) {
      v = __ldg(&idx[(size_t)row * k + j0 + j]);
      if (v >= N) v = -1;
    }
    s_idx[j] = v;
  }
  // queries of all heads
  for (int i = tid; i < H * kRowChunks; i += kThreads) {
    const int h = i / kRowChunks, c = i - h * kRowChunks;
    cp_async_16(sQ + swz576(h, c * 8), qp + (size_t)h * kDqk + c * 8, 16);
  }
  __syncthreads();

  auto load_tile = [&](int it, int st) {
    const uint32_t base = sKV + st * kStageBytes;
    for (int i = tid; i < kBc * kRowChunks; i += kThreads) {
      const int r = i / kRowChunks, c = i - r * kRowChunks;
      const int sel = s_idx[it * kBc + r];
      const uint16_t* src = sel >= 0 ? kvb + (size_t)sel * kDqk + c * 8 : kvb;
      cp_async_16(base + swz576(r, c * 8), src, sel >= 0 ? 16 : 0);
    }
  };

  if (ntiles > 0) load_tile(0, 0);
  cp_async_commit();
  if (ntiles > 1) load_tile(1, 1);
  cp_async_commit();

  // S-phase roles: warp (mt, nh) computes heads [16mt, 16mt+16) x tile rows [16nh, 16nh+16)
  const bool s_warp = warp < 2 * MT;
  const int mt_s = warp >> 1, nh = warp & 1;
  const int r0 = 16 * mt_s + g, r1 = r0 + 8;
  float m_run0 = -INFINITY, m_run1 = -INFINITY, l_run0 = 0.f, l_run1 = 0.f;

  float acc_o[MT][8][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) acc_o[mt][nt][0] = acc_o[mt][nt][1] = acc_o[mt][nt][2] = acc_o[mt][nt][3] = 0.f;

  // ldmatrix lane addressing
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8;  // A operands (Q, P)
  const int a_col = (lane >> 4) * 8;
  const int kb_row = (lane & 7) + (lane >> 4) * 8;       // B operand of S (gathered rows)
  const int kb_col = ((lane >> 3) & 1) * 8;
  const int vb_row = (lane & 7) + ((lane >> 3) & 1) * 8; // B operand of PV (transposed)
  const int vb_col = (lane >> 4) * 8;

  for (int it = 0; it < ntiles; ++it) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (it + 2 < ntiles) load_tile(it + 2, (it + 2) % kStages);
    cp_async_commit();
    const uint32_t stage = sKV + (it % kStages) * kStageBytes;

    float p_lo[2][2], p_hi[2][2];
    if (s_warp) {
      float acc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 4
      for (int kk = 0; kk < kKSteps; ++kk) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        ldmatrix_x4(sQ + swz576(16 * mt_s + a_row, 16 * kk + a_col), a0, a1, a2, a3);
        ldmatrix_x4(stage + swz576(16 * nh + kb_row, 16 * kk + kb_col), b0, b1, b2, b3);
        mma_bf16_16816(acc[0], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[1], a0, a1, a2, a3, b2, b3);
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = 16 * nh + 8 * nt + 2 * tq + e;
          const bool valid = s_idx[it * kBc + key] >= 0;
          acc[nt][e] = valid ? acc[nt][e] * scale_log2 : -INFINITY;
          acc[nt][2 + e] = valid ? acc[nt][2 + e] * scale_log2 : -INFINITY;
          mx0 = fmaxf(mx0, acc[nt][e]);
          mx1 = fmaxf(mx1, acc[nt][2 + e]);
        }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 2));
      if (tq == 0) {
        red_max[nh * kMaxHeads + r0] = mx0;
        red_max[nh * kMaxHeads + r1] = mx1;
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        p_lo[nt][0] = acc[nt][0];
        p_lo[nt][1] = acc[nt][1];
        p_hi[nt][0] = acc[nt][2];
        p_hi[nt][1] = acc[nt][3];
      }
    }
    __syncthreads();
    if (s_warp) {
      const float mn0 = fmaxf(m_run0, fmaxf(red_max[r0], red_max[kMaxHeads + r0]));
      const float mn1 = fmaxf(m_run1, fmaxf(red_max[r1], red_max[kMaxHeads + r1]));
      const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m_run0 - mn0);
      const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m_run1 - mn1);
      const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
      const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float e00 = exp2f(p_lo[nt][0] - mu0), e01 = exp2f(p_lo[nt][1] - mu0);
        const float e10 = exp2f(p_hi[nt][0] - mu1), e11 = exp2f(p_hi[nt][1] - mu1);
        ls0 += e00 + e01;
        ls1 += e10 + e11;
        const int col = 16 * nh + 8 * nt;
        *reinterpret_cast<uint32_t*>(smem + kOffP + swzP(r0, col) + 4 * tq) = pack_bf16x2(e00, e01);
        *reinterpret_cast<uint32_t*>(smem + kOffP + swzP(r1, col) + 4 * tq) = pack_bf16x2(e10, e11);
      }
      l_run0 = l_run0 * al0 + ls0;
      l_run1 = l_run1 * al1 + ls1;
      m_run0 = mn0;
      m_run1 = mn1;
      if (nh == 0 && tq == 0) {
        alpha_s[r0] = al0;
        alpha_s[r1] = al1;
      }
    }
    __syncthreads();

    // O = alpha * O + P V for output columns [64 warp, 64 warp + 64)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const float a0 = alpha_s[16 * mt + g], a1 = alpha_s[16 * mt + g + 8];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        acc_o[mt][nt][0] *= a0;
        acc_o[mt][nt][1] *= a0;
        acc_o[mt][nt][2] *= a1;
        acc_o[mt][nt][3] *= a1;
      }
    }
#pragma unroll
    for (int ks = 0; ks < kBc / 16; ++ks) {
      uint32_t bv[8][2];
#pragma unroll
      for (int np = 0; np < 4; ++np)
        ldmatrix_x4_trans(stage + swz576(16 * ks + vb_row, 64 * warp + 16 * np + vb_col), bv[2 * np][0],
                          bv[2 * np][1], bv[2 * np + 1][0], bv[2 * np + 1][1]);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(sP + swzP(16 * mt + a_row, 16 * ks + a_col), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) mma_bf16_16816(acc_o[mt][nt], a0, a1, a2, a3, bv[nt][0], bv[nt][1]);
      }
    }
  }
  cp_async_wait<0>();

  // row statistics: sum over the quad and the two key halves
  if (s_warp) {
    l_run0 += __shfl_xor_sync(0xFFFFFFFFu, l_run0, 1);
    l_run0 += __shfl_xor_sync(0xFFFFFFFFu, l_run0, 2);
    l_run1 += __shfl_xor_sync(0xFFFFFFFFu, l_run1, 1);
    l_run1 += __shfl_xor_sync(0xFFFFFFFFu, l_run1, 2);
    if (tq == 0) {
      lsum_s[nh * kMaxHeads + r0] = l_run0;
      lsum_s[nh * kMaxHeads + r1] = l_run1;
      if (nh == 0) {
        m_s[r0] = m_run0;
        m_s[r1] = m_run1;
      }
    }
  }
  if (ntiles == 0 && tid < H) {
    lsum_s[tid] = lsum_s[kMaxHeads + tid] = 0.f;
    m_s[tid] = -INFINITY;
  }
  __syncthreads();

  if (nsplit == 1) {
    float* out = layers.out[layer] + (size_t)row * H * kDv;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = 16 * mt + g + 8 * hh;
        const float l = lsum_s[h] + lsum_s[kMaxHeads + h];
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          float2 v = make_float2(acc_o[mt][nt][2 * hh] * inv, acc_o[mt][nt][2 * hh + 1] * inv);
          *reinterpret_cast<float2*>(out + (size_t)h * kDv + 64 * warp + 8 * nt + 2 * tq) = v;
        }
      }
  } else {
    const size_t unit = ((size_t)layer * gridDim.y + row) * nsplit + split;
    float* po = partial + unit * (size_t)H * (kDv + 2);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = 16 * mt + g + 8 * hh;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          float2 v = make_float2(acc_o[mt][nt][2 * hh], acc_o[mt][nt][2 * hh + 1]);
          *reinterpret_cast<float2*>(po + (size_t)h * kDv + 64 * warp + 8 * nt + 2 * tq) = v;
        }
      }
    if (tid < H) {
      po[(size_t)H * kDv + 2 * tid] = m_s[tid];
      po[(size_t)H * kDv + 2 * tid + 1] = lsum_s[tid] + lsum_s[kMaxHeads + tid];
    }
  }
}

// out[h][:] = sum_s 2^(m_s - M) O_s[h][:] / sum_s 2^(m_s - M) l_s
__global__ void __launch_bounds__(128)
attn_combine_kernel(AttnLayers layers, int H, int nsplit, const float* __restrict__ partial) {
  const int h = blockIdx.x;
  const int row = blockIdx.y;
  const int layer = blockIdx.z;
  const size_t unit0 = ((size_t)layer * gridDim.y + row) * nsplit;
  const size_t stride = (size_t)H * (kDv + 2);
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, partial[(unit0 + s) * stride + (size_t)H * kDv + 2 * h]);
  float den = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const int d = threadIdx.x * 4;
  for (int s = 0; s < nsplit; ++s) {
    const float* po = partial + (unit0 + s) * stride;
    const float m = po[(size_t)H * kDv + 2 * h];
    if (m == -INFINITY) continue;
    const float wgt = exp2f(m - M);
    den += wgt * po[(size_t)H * kDv + 2 * h + 1];
    const float4 o = *reinterpret_cast<const float4*>(po + (size_t)h * kDv + d);
    acc.x += wgt * o.x;
    acc.y += wgt * o.y;
    acc.z += wgt * o.z;
    acc.w += wgt * o.w;
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float* out = layers.out[layer] + ((size_t)row * H + h) * kDv + d;
  *reinterpret_cast<float4*>(out) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

}  // namespace

cudaError_t launch_attn_combine(const AttnLayers& layers, int L, long long rows, int H, int nsplit, const float* partial,
                                cudaStream_t stream) {
  attn_combine_kernel<<<dim3(H, (unsigned)rows, L), 128, 0, stream>>>(layers, H, nsplit, partial);
  return cudaGetLastError();
}

namespace {

template <int MT>
cudaError_t launch_mt(const AttnLayers& layers, int L, const int32_t* idx, long long rows, int T, int N, int k,
                      int nsplit, int chunk, float scale_log2, float* partial, cudaStream_t stream) {
  static DeviceOnce once;
  cudaError_t e = once.run(
      [] { return cudaFuncSetAttribute(sparse_attn_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes); });
  if (e != cudaSuccess) return e;
  sparse_attn_kernel<MT><<<dim3(nsplit, (unsigned)rows, L), kThreads, kSmemBytes, stream>>>(layers, idx, T, N, k, chunk,
                                                                                            scale_log2, partial);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (nsplit > 1) e = launch_attn_combine(layers, L, rows, MT * 16, nsplit, partial, stream);
  return e;
}

}  // namespace

// Keys per split: a multiple of the 64-row tile of the tensor-core kernel.
int attn_split_chunk(int k, int nsplit) {
  const int chunk = (k + nsplit - 1) / nsplit;
  return (chunk + kAttnTile - 1) / kAttnTile * kAttnTile;
}

// Splits per (query row, layer): about one CTA per SM in total.
int attn_num_splits(long long rows, int L, int k) {
  const long long units = rows * L;
  long long ns = kNumSMs / (units > 0 ? units : 1);
  if (ns < 1) ns = 1;
  const long long max_ns = (k + kAttnTile - 1) / kAttnTile;
  if (ns > max_ns) ns = max_ns;
  const int chunk = attn_split_chunk(k, (int)ns);
  return (k + chunk - 1) / chunk;
}

size_t attn_workspace_bytes(long long rows, int L, int H, int k) {
  const int ns = attn_num_splits(rows, L, k);
  if (ns <= 1) return 0;
  return (size_t)L * rows * ns * H * (kDv + 2) * sizeof(float);
}

cudaError_t launch_sparse_attn_mma(const AttnLayers& layers, int L, const int32_t* idx, int B, int T, int N, int H,
                                   int k, float scale, void* ws, cudaStream_t stream) {
  const long long rows = (long long)B * T;
  const int nsplit = attn_num_splits(rows, L, k);
  const int chunk = attn_split_chunk(k, nsplit);
  const float scale_log2 = scale * 1.4426950408889634f;
  float* partial = static_cast<float*>(ws);
  switch (H) {
    case 16: return launch_mt<1>(layers, L, idx, rows, T, N, k, nsplit, chunk, scale_log2, partial, stream);
    case 32: return launch_mt<2>(layers, L, idx, rows, T, N, k, nsplit, chunk, scale_log2, partial, stream);
    case 48: return launch_mt<3>(layers, L, idx, rows, T, N, k, nsplit, chunk, scale_log2, partial, stream);
    case 64: return launch_mt<4>(layers, L, idx, rows, T, N, k, nsplit, chunk, scale_log2, partial, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
