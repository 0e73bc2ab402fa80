// topk_cluster.cu -- per-query top-k for rows that one thread-block cluster holds on chip.
//
// "GLM-5.2 1M architecture teardown", Cut 1: DSA -- keep the index_topk (2048) best
// history tokens per query.  Same order and output as the scan kernels of topk.cu:
// composite C(s) = order_key(score[s]) << 32 | (0xFFFFFFFF - s), the k largest composites,
// written in ascending token order, -1 padding when fewer than k positions are visible.
//
// One cluster of C CTAs (C = 1, 2, 4 or 8) per query row; CTA r keeps the order keys of
// positions [r * chunk, (r + 1) * chunk) in shared memory (chunk = 1024 threads x kpt), so
// the scores are read from memory once.  Radix select, most significant digit first, over
// the 64-bit composite (digits of 12, 10, 10, 11, 11, 10 bits):
//   - each CTA histograms the digit of its elements that still match the prefix found
//     so far; the cluster adds the histograms through distributed shared memory (CTA r
//     sums bins [r * bins / C, (r + 1) * bins / C) over the peers, then every CTA reads all
//     the sums) and every CTA finds the same digit -- the bin where the count from the top
//     reaches the rank still needed.  The first digit's histogram may come ready-made
//     from the indexer epilogue;
//   - once the bin holds at most kFinal elements, they are gathered into every CTA and
//     ranked directly, which gives the threshold composite exactly;
//   - every CTA counts its selected elements, takes the counts of the lower ranks as its
//     output offset and writes its positions in order (warp ballots).
// No global workspace, no atomics on global memory and a single launch.  Every thread
// passes every cluster barrier: the control flow depends only on cluster-wide sums.
#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kCT = 1024;              // threads per CTA
constexpr int kCWarps = kCT / 32;
constexpr int kMaxBins = 1 << 12;
constexpr int kFinal = 512;            // final-bin sizes ranked directly
constexpr int kLevels = 6;
__constant__ int kDigitWidth[kLevels] = {12, 10, 10, 11, 11, 10};

struct ClusterSmem {
  uint32_t h[kMaxBins];                // this CTA's histogram of the current digit
  uint32_t part[kMaxBins];             // cluster sums of the bins this CTA owns
  uint32_t full[kMaxBins];             // cluster sums of every bin (local copy)
  unsigned long long fin[kFinal];      // this CTA's composites in the final bin
  unsigned long long all[kFinal];      // the whole cluster's, gathered
  uint32_t warp_tmp[kCWarps];
  uint32_t total;
  uint32_t nfin;                       // read by the peers
  uint32_t nsel;                       // read by the peers
  uint32_t base;
  uint32_t peer_cnt[8], peer_off[8];
  uint32_t digit, above, count;
  unsigned long long thr;
};

// the keys follow the struct, 16-byte aligned (they are written as uint4)
constexpr int kKeysOff = ((int)sizeof(ClusterSmem) + 127) & ~127;
static_assert(kKeysOff % 16 == 0, "uint4 key stores");

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ unsigned long long ld_cluster_u64(uint32_t addr) {
  unsigned long long v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr));
  return v;
}

// Exclusive scan of one value per thread over the CTA (kCT threads); *total gets the sum.
__device__ __forceinline__ uint32_t scan_excl(uint32_t v, ClusterSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.warp_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint32_t wv = sm.warp_tmp[lane];
    uint32_t z = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, z, o);
      if (lane >= o) z += y;
    }
    sm.warp_tmp[lane] = z - wv;
    if (lane == 31) sm.total = z;
  }
  __syncthreads();
  const uint32_t r = sm.warp_tmp[warp] + x - v;
  __syncthreads();
  return r;
}

// In the histogram `hist` of `bins` bins (bins >= kCT / 8 ... kMaxBins), find the digit d
// where the count from the top reaches r: above(d) < r <= above(d) + hist[d].  Results in
// sm.digit / sm.above / sm.count.  Every thread of the CTA calls it.
__device__ void digit_search(const uint32_t* hist, int bins, uint32_t r, ClusterSmem& sm) {
  const int per = bins >= kCT ? bins / kCT : 1;
  const int hi = bins - (int)threadIdx.x * per;  // this thread owns bins [hi - per, hi)
  uint32_t local[4];
  uint32_t lsum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = hi - 1 - i;
    local[i] = (i < per && b >= 0) ? hist[b] : 0u;
    lsum += local[i];
  }
  if (threadIdx.x == 0) {
    sm.digit = 0;
    sm.above = 0;
    sm.count = 0;
  }
  uint32_t run = scan_excl(lsum, sm);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i < per && hi - 1 - i >= 0 && run < r && run + local[i] >= r) {
      sm.digit = (uint32_t)(hi - 1 - i);
      sm.above = run;
      sm.count = local[i];
    }
    run += local[i];
  }
  __syncthreads();
}

// Cluster-wide sum of every CTA's sm.h[0, bins) into every CTA's sm.full.
__device__ void cluster_hist_sum(ClusterSmem& sm, int bins, int C, int me) {
  cluster_sync();  // every CTA's histogram is complete
  const int bpc = bins / C;
  for (int b = threadIdx.x; b < bpc; b += kCT) {
    const uint32_t a = smem_u32(&sm.h[me * bpc + b]);
    uint32_t s = 0;
    for (int p = 0; p < C; ++p) s += ld_cluster_u32(cluster_map(a, p));
    sm.part[b] = s;
  }
  cluster_sync();  // every owner's sums are complete
  for (int b = threadIdx.x; b < bins; b += kCT) {
    const int owner = b / bpc;
    sm.full[b] = ld_cluster_u32(cluster_map(smem_u32(&sm.part[b - owner * bpc]), owner));
  }
  __syncthreads();
}

template <int KPT>
__global__ void __launch_bounds__(kCT, 1)
topk_cluster_kernel(const float* __restrict__ scores, int T, int N, long long q_pos0, int k, int vec,
                    const uint32_t* __restrict__ hist_g, int32_t* __restrict__ idx_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ClusterSmem& sm = *reinterpret_cast<ClusterSmem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kKeysOff);
  constexpr int kChunk = kCT * KPT;
  constexpr int kSeg = 32 * KPT;  // positions of one warp, processed 32 at a time
  const int C = (int)gridDim.x, me = (int)blockIdx.x, row = (int)blockIdx.y;
  const long long V = visible_count(N, q_pos0, row % T);
  const long long c0 = (long long)me * kChunk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg0 = warp * kSeg;
  const float* sr = scores + (size_t)row * N;
  int32_t* out = idx_out + (size_t)row * k;

  // this CTA's scores, read once, as order keys (positions >= V are never used)
#pragma unroll
  for (int i = 0; i < KPT / 4; ++i) {
    const int p = seg0 + 128 * i + 4 * lane;
    const long long s = c0 + p;
    float4 v;
    if (vec && s + 3 < V) {
      v = __ldcg(reinterpret_cast<const float4*>(sr + s));
    } else {
      v.x = s < V ? __ldcg(sr + s) : 0.f;
      v.y = s + 1 < V ? __ldcg(sr + s + 1) : 0.f;
      v.z = s + 2 < V ? __ldcg(sr + s + 2) : 0.f;
      v.w = s + 3 < V ? __ldcg(sr + s + 3) : 0.f;
    }
    *reinterpret_cast<uint4*>(keys + p) = make_uint4(order_key(v.x), order_key(v.y), order_key(v.z), order_key(v.w));
  }
  __syncwarp();  // a warp only ever reads the keys of its own segment

  if (V <= k) {
    // every visible position is kept, in order; the rest of the row is padding
#pragma unroll 4
    for (int step = 0; step < KPT; ++step) {
      const long long s = c0 + seg0 + 32 * step + lane;
      if (s < V) out[s] = (int32_t)s;
    }
    if (me == 0)
      for (long long j = V + threadIdx.x; j < k; j += kCT) out[j] = -1;
    return;
  }

  auto comp = [&](int p) -> unsigned long long {
    return ((unsigned long long)keys[p] << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)(c0 + p));
  };

  // radix select over the composite, one digit per level, until the bin is small
  unsigned long long prefix = 0;
  int pos = 64;              // bits [pos, 64) of the threshold are fixed in `prefix`
  uint32_t r = (uint32_t)k;  // rank still needed inside the current bin (1-based)
  for (int level = 0; level < kLevels; ++level) {
    const int width = kDigitWidth[level];
    const int shift = pos - width;
    const int bins = 1 << width;
    if (level == 0 && hist_g) {
      for (int b = threadIdx.x; b < bins; b += kCT) sm.full[b] = __ldcg(&hist_g[(size_t)row * kHistBins + b]);
      __syncthreads();
    } else {
      for (int b = threadIdx.x; b < bins; b += kCT) sm.h[b] = 0;
      __syncthreads();
#pragma unroll 4
      for (int step = 0; step < KPT; ++step) {
        const int p = seg0 + 32 * step + lane;
        if (c0 + p < V) {
          const unsigned long long c = comp(p);
          if (pos == 64 || (c >> pos) == (prefix >> pos))
            atomicAdd(&sm.h[(uint32_t)(c >> shift) & (uint32_t)(bins - 1)], 1u);
        }
      }
      cluster_hist_sum(sm, bins, C, me);
    }
    digit_search(sm.full, bins, r, sm);
    r -= sm.above;
    prefix |= (unsigned long long)sm.digit << shift;
    pos = shift;
    if (sm.count <= (uint32_t)kFinal) break;  // the last level leaves one element
  }

  // the final bin: gather its elements from the whole cluster and rank them
  if (threadIdx.x == 0) sm.nfin = 0;
  __syncthreads();
#pragma unroll 4
  for (int step = 0; step < KPT; ++step) {
    const int p = seg0 + 32 * step + lane;
    if (c0 + p < V) {
      const unsigned long long c = comp(p);
      if ((c >> pos) == (prefix >> pos)) {
        const uint32_t slot = atomicAdd(&sm.nfin, 1u);
        if (slot < (uint32_t)kFinal) sm.fin[slot] = c;
      }
    }
  }
  __syncthreads();
  cluster_sync();  // every CTA's final-bin list is complete
  if (threadIdx.x < 32) {
    uint32_t cnt = lane < C ? ld_cluster_u32(cluster_map(smem_u32(&sm.nfin), lane)) : 0u;
    cnt = min(cnt, (uint32_t)kFinal);
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < 8) {
      sm.peer_cnt[lane] = cnt;
      sm.peer_off[lane] = incl - cnt;
    }
    if (lane == 31) sm.total = incl;
  }
  __syncthreads();
  const uint32_t nall = min(sm.total, (uint32_t)kFinal);
  for (int p = 0; p < C; ++p) {
    const uint32_t cnt = sm.peer_cnt[p], off = sm.peer_off[p];
    for (uint32_t i = threadIdx.x; i < cnt && off + i < (uint32_t)kFinal; i += kCT)
      sm.all[off + i] = ld_cluster_u64(cluster_map(smem_u32(&sm.fin[i]), p));
  }
  if (threadIdx.x == 0) sm.thr = 0;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < nall; i += kCT) {
    const unsigned long long c = sm.all[i];
    uint32_t rank = 0;
    for (uint32_t j = 0; j < nall; ++j) rank += sm.all[j] > c ? 1u : 0u;
    if (rank == r - 1) sm.thr = c;  // composites are distinct: exactly one thread writes
  }
  __syncthreads();
  const unsigned long long thr = sm.thr;

  // selected = composite >= thr; output offset = selected count of the lower ranks
  uint32_t wcnt = 0;
#pragma unroll 4
  for (int step = 0; step < KPT; ++step) {
    const int p = seg0 + 32 * step + lane;
    const bool sel = c0 + p < V && comp(p) >= thr;
    wcnt += __popc(__ballot_sync(0xFFFFFFFFu, sel));
  }
  uint32_t wbase = scan_excl(lane == 0 ? wcnt : 0u, sm);
  wbase = __shfl_sync(0xFFFFFFFFu, wbase, 0);
  if (threadIdx.x == 0) sm.nsel = sm.total;
  __syncthreads();
  cluster_sync();  // every CTA's selected count is published
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int p = 0; p < me; ++p) b += ld_cluster_u32(cluster_map(smem_u32(&sm.nsel), p));
    sm.base = b;
  }
  __syncthreads();
  uint32_t o = sm.base + wbase;
#pragma unroll 4
  for (int step = 0; step < KPT; ++step) {
    const int p = seg0 + 32 * step + lane;
    const bool sel = c0 + p < V && comp(p) >= thr;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, sel);
    if (sel) {
      const uint32_t at = o + __popc(m & ((1u << lane) - 1u));
      if (at < (uint32_t)k) out[at] = (int32_t)(c0 + p);
    }
    o += __popc(m);
  }
  cluster_sync();  // the peers are done reading this CTA's shared memory
}

template <int KPT>
cudaError_t launch_kpt(const float* scores, long long rows, int T, int N, long long q_pos0, int k, int C,
                       const uint32_t* hist, int32_t* idx, cudaStream_t stream) {
  const int smem = kKeysOff + kCT * KPT * 4;
  static DeviceOnce once;
  cudaError_t e = once.run([&] {
    return cudaFuncSetAttribute(topk_cluster_kernel<KPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (e != cudaSuccess) return e;
  const int vec = (N & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)C, (unsigned)rows, 1);
  cfg.blockDim = dim3(kCT);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel<KPT>, scores, T, N, q_pos0, k, vec, hist, idx);
}

}  // namespace

// Cluster size C and keys per thread for rows of up to vmax visible positions: the
// smallest C (1, 2, 4, 8) whose chunk of 1024 x kpt positions, kpt <= 16, covers a row,
// else C = 8 with kpt = 32.  False when a row is longer than that, or when the clusters
// would not fit the GPU in about one wave (many rows: the scan kernels do better).
bool topk_cluster_plan(long long rows, long long vmax, int* C, int* kpt) {
  for (int c = 1; c <= 8; c *= 2) {
    const long long per = (vmax + (long long)c * kCT - 1) / ((long long)c * kCT);
    int kp = per <= 4 ? 4 : per <= 8 ? 8 : per <= 16 ? 16 : per <= 32 ? 32 : 0;
    if (kp == 0 || (kp == 32 && c < 8)) continue;
    if (rows * c > kNumSMs) return false;
    *C = c;
    *kpt = kp;
    return true;
  }
  return false;
}

cudaError_t launch_topk_cluster(const float* scores, int B, int T, int N, long long q_pos0, int k, int C, int kpt,
                                const uint32_t* hist, int32_t* idx, cudaStream_t stream) {
  const long long rows = (long long)B * T;
  switch (kpt) {
    case 4: return launch_kpt<4>(scores, rows, T, N, q_pos0, k, C, hist, idx, stream);
    case 8: return launch_kpt<8>(scores, rows, T, N, q_pos0, k, C, hist, idx, stream);
    case 16: return launch_kpt<16>(scores, rows, T, N, q_pos0, k, C, hist, idx, stream);
    case 32: return launch_kpt<32>(scores, rows, T, N, q_pos0, k, C, hist, idx, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
