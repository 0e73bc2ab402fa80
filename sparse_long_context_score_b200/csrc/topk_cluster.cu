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
//   - first digit (the top 12 key bits): its per-row histogram comes from the indexer
//     epilogue, or the CTAs histogram their chunks and sum the histograms through
//     distributed shared memory (CTA r adds up bins [r * 4096 / C, (r + 1) * 4096 / C) of
//     every peer, then every CTA reads all the sums).  Every CTA finds the same threshold
//     bin b*: the bin where the count from the top reaches k.  From then on a thread only
//     looks at its elements with bin >= b* (a bit mask in a register): the selected
//     elements are among them;
//   - merge path, when b* holds at most kMergeCap elements of the row: every CTA compacts
//     its elements of b* (as composites) into a list in its shared memory; after one
//     cluster barrier every CTA copies all the lists through distributed shared memory and
//     selects the needed rank among them on its own (radix digits over the low 52 bits,
//     shared-memory histograms, CTA barriers only), which gives the threshold and every
//     rank's selected count without another exchange;
//   - digit path, otherwise: each CTA histograms the next digit of its elements that still
//     match the prefix and adds the non-empty bins into the bin's owner CTA (remote
//     reductions into shared memory); one cluster barrier later every CTA reads the sums it
//     needs; the digits stop once every element of the bin is needed (at the latest when
//     the 64 bits are fixed: composites are distinct); the threshold is then the prefix,
//     and every CTA sends its selected count to every peer;
//   - every CTA takes the selected counts of the lower ranks as its output offset and
//     writes its positions in order (warp ballots).
// No global workspace, no atomics on global memory and a single launch.  Every thread
// passes every cluster barrier: the control flow depends only on cluster-wide sums, and
// no CTA touches another's shared memory after the last barrier.
#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kCT = 1024;              // threads per CTA
constexpr int kCWarps = kCT / 32;
constexpr int kMaxBins = 1 << 12;
constexpr int kMaxC = 8;
constexpr int kLevels = 6;
__constant__ int kDigitWidth[kLevels] = {12, 10, 10, 11, 11, 10};

constexpr int kMergeCap = 4096;        // threshold-bin elements the merge path gathers

struct ClusterSmem {
  // The digit-by-digit path uses `d`; the merge path reuses the same 64 KB for its candidate
  // lists.  The path is chosen from the cluster-wide count of the threshold bin, so every
  // CTA of a cluster takes the same one.
  union {
    struct {
      uint32_t h[kMaxBins];               // first digit counted here: this CTA's histogram
      uint32_t full0[kMaxBins];           // ... the cluster sums of every bin
      uint32_t hl[2048];                  // this CTA's histogram of a later digit
      uint32_t fullb[3][2048];            // cluster sums of the later-digit bins this CTA owns
    } d;
    struct {
      unsigned long long loc[kMergeCap];  // this CTA's threshold-bin composites (peers read them)
      unsigned long long mrg[kMergeCap];  // every CTA's, in rank order
    } m;
  };
  uint32_t part[kMaxBins];                // first-digit sums of the bins this CTA owns (peers read
                                          // them); later the merge path's select histogram
  uint32_t nsel[kMaxC];                   // selected counts per sending rank
  uint32_t warp_tmp[kCWarps];
  uint32_t res[3];                        // digit search: digit, above, count
  uint32_t n_loc, n_above;                // merge path: this CTA's candidates and elements above
  uint32_t q_cnt[kMaxC], q_above[kMaxC], q_ge[kMaxC];  // merge path: the same per rank
};
static_assert(sizeof(unsigned long long) * 2 * kMergeCap <= sizeof(uint32_t) * (2 * kMaxBins + 4 * 2048),
              "the merge lists fit the digit path's arrays");

// the keys follow the struct, 16-byte aligned (they are written as uint4)
constexpr int kKeysOff = ((int)sizeof(ClusterSmem) + 127) & ~127;
static_assert(kKeysOff % 16 == 0, "uint4 key stores");

// Thread t owns bins [bins - (t + 1) * per, bins - t * per) of a histogram (per = bins /
// kCT, 1..4) and holds their counts in v[0..per), highest bin first.  Finds the bin d where
// the count from the top reaches r: above(d) < r <= above(d) + count(d).  Two barriers.
__device__ __forceinline__ void digit_search(const uint32_t (&v)[4], int per, int bins, uint32_t r, ClusterSmem& sm,
                                             uint32_t& d, uint32_t& above, uint32_t& count) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t lsum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) lsum += i < per ? v[i] : 0u;
  uint32_t x = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.warp_tmp[warp] = x;
  __syncthreads();
  const uint32_t wt = sm.warp_tmp[lane];
  uint32_t z = wt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, z, o);
    if (lane >= o) z += y;
  }
  uint32_t run = __shfl_sync(0xFFFFFFFFu, z - wt, warp) + x - lsum;
  const int hi = bins - (int)threadIdx.x * per;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i < per && run < r && run + v[i] >= r) {
      sm.res[0] = (uint32_t)(hi - 1 - i);
      sm.res[1] = run;
      sm.res[2] = v[i];
    }
    run += i < per ? v[i] : 0u;
  }
  __syncthreads();
  d = sm.res[0];
  above = sm.res[1];
  count = sm.res[2];
}

// Exclusive prefix sum of one value per thread over the CTA (kCT threads); *total gets the
// sum.  Two barriers; warp_tmp is free again on return.
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t v, ClusterSmem& sm, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.warp_tmp[warp] = x;
  __syncthreads();
  const uint32_t wt = sm.warp_tmp[lane];
  uint32_t z = wt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, z, o);
    if (lane >= o) z += y;
  }
  total = __shfl_sync(0xFFFFFFFFu, z, 31);
  const uint32_t r = __shfl_sync(0xFFFFFFFFu, z - wt, warp) + x - v;
  __syncthreads();
  return r;
}

// First digit counted by the CTAs: cluster-wide sum of every CTA's sm.h into sm.full0.
// CTA r adds up its share of the bins over all peers, then every CTA reads all the sums.
__device__ void first_digit_sum(ClusterSmem& sm, int C, int me) {
  cluster_sync();  // every CTA's histogram is complete
  const int bpc = kMaxBins / C;
  for (int b = threadIdx.x; b < bpc; b += kCT) {
    const uint32_t a = smem_u32(&sm.d.h[me * bpc + b]);
    uint32_t s = 0;
    for (int p = 0; p < C; ++p) s += ld_cluster_u32(cluster_map(a, p));
    sm.part[b] = s;
  }
  cluster_sync();  // every owner's sums are complete
  for (int b = threadIdx.x; b < kMaxBins; b += kCT) {
    const int owner = b / bpc;
    sm.d.full0[b] = ld_cluster_u32(cluster_map(smem_u32(&sm.part[b - owner * bpc]), owner));
  }
  __syncthreads();
}

template <int KPT>
__global__ void __launch_bounds__(kCT, 1)
topk_cluster_kernel(const float* __restrict__ scores, int T, int N, long long q_pos0, int k, int vec,
                    const uint32_t* __restrict__ hist_g, int32_t* __restrict__ idx_out, int* __restrict__ err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ClusterSmem& sm = *reinterpret_cast<ClusterSmem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kKeysOff);
  constexpr int kChunk = kCT * KPT;
  constexpr int kSeg = 32 * KPT;  // positions of one warp, taken 32 at a time (bit `step` of a mask)
  static_assert(KPT % 4 == 0 && KPT <= 32, "keys per thread");
  const int C = (int)gridDim.x, me = (int)blockIdx.x, row = (int)blockIdx.y;
  const long long V = visible_count(N, q_pos0, row % T);
  const long long c0 = (long long)me * kChunk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg0 = warp * kSeg;
  const float* sr = scores + (size_t)row * N;
  int32_t* out = idx_out + (size_t)row * k;
  grid_dep_launch();  // the attention may be scheduled on free SMs; it waits for this grid
  grid_dep_wait();    // the scores (and the histogram) of the preceding kernel

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

  // loads in flight together: the first digit's histogram (this thread's four bins,
  // highest first) and this CTA's scores
  uint32_t hv[4] = {0u, 0u, 0u, 0u};
  if (hist_g) {
    const uint4 q = __ldcg(reinterpret_cast<const uint4*>(hist_g + (size_t)row * kHistBins + kHistBins -
                                                          4 * (threadIdx.x + 1)));
    hv[0] = q.w;
    hv[1] = q.z;
    hv[2] = q.y;
    hv[3] = q.x;
  }
  float4 v[KPT / 4];
#pragma unroll
  for (int i = 0; i < KPT / 4; ++i) {
    const long long s = c0 + seg0 + 128 * i + 4 * lane;
    if (vec && s + 3 < V) {
      v[i] = __ldcg(reinterpret_cast<const float4*>(sr + s));
    } else {
      v[i].x = s < V ? __ldcg(sr + s) : 0.f;
      v[i].y = s + 1 < V ? __ldcg(sr + s + 1) : 0.f;
      v[i].z = s + 2 < V ? __ldcg(sr + s + 2) : 0.f;
      v[i].w = s + 3 < V ? __ldcg(sr + s + 3) : 0.f;
    }
  }
  // the later-digit histograms the peers add into start at zero: barrier S0 (arrive now,
  // wait before the first access to another CTA's shared memory)
  for (int i = threadIdx.x; i < 2048; i += kCT) {
    sm.d.fullb[1][i] = 0u;
    sm.d.hl[i] = 0u;  // the second digit is counted in the candidate pass below
  }
  cluster_arrive();
  bool s0_pending = true;
  auto wait_s0 = [&] {
    if (s0_pending) {
      cluster_wait();
      s0_pending = false;
    }
  };
#pragma unroll
  for (int i = 0; i < KPT / 4; ++i)
    *reinterpret_cast<uint4*>(keys + seg0 + 128 * i + 4 * lane) =
        make_uint4(order_key(v[i].x), order_key(v[i].y), order_key(v[i].z), order_key(v[i].w));
  __syncwarp();  // a warp only ever reads the keys of its own segment

  auto comp = [&](int p) -> unsigned long long {
    return ((unsigned long long)keys[p] << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)(c0 + p));
  };

  // first digit: the threshold bin b*
  uint32_t d, above, count;
  if (!hist_g) {
    for (int b = threadIdx.x; b < kMaxBins; b += kCT) sm.d.h[b] = 0u;
    __syncthreads();
#pragma unroll 4
    for (int step = 0; step < KPT; ++step) {
      const int p = seg0 + 32 * step + lane;
      if (c0 + p < V) atomicAdd(&sm.d.h[keys[p] >> kHistShift], 1u);
    }
    wait_s0();
    first_digit_sum(sm, C, me);
#pragma unroll
    for (int i = 0; i < 4; ++i) hv[i] = sm.d.full0[kMaxBins - 1 - 4 * (int)threadIdx.x - i];
  }
  digit_search(hv, 4, kMaxBins, (uint32_t)k, sm, d, above, count);
  uint32_t r = (uint32_t)k - above;  // rank still needed inside the current bin (1-based)
  unsigned long long prefix = (unsigned long long)d << 52;
  int pos = 52;                      // bits [pos, 64) of the threshold are fixed in `prefix`
  const uint32_t bstar = d;
  static_assert(kHistShift == 20, "second digit = key bits 19..10");

  // The threshold bin b* holds `count` elements of the row, r of which are selected.  When
  // they are few, every CTA gathers all of them and selects rank r on its own (merge path:
  // two cluster barriers); otherwise the digits are resolved one by one across the cluster.
  const bool merge = count != r && count <= (uint32_t)kMergeCap;  // the same in every CTA
  uint32_t sel = 0;      // this thread's selected elements (bit `step`)
  uint32_t base = 0;     // selected elements of the lower ranks
  uint32_t total = 0;    // selected elements of the row (k when the invariant holds)
  if (merge) {
    wait_s0();
    uint32_t above_bits = 0, cand_bits = 0;
#pragma unroll
    for (int step = 0; step < KPT; ++step) {
      const int p = seg0 + 32 * step + lane;
      if (c0 + p < V) {
        const uint32_t bin = keys[p] >> kHistShift;
        above_bits |= (bin > bstar ? 1u : 0u) << step;
        cand_bits |= (bin == bstar ? 1u : 0u) << step;
      }
    }
    // this CTA's b* elements, compacted into its list (at most `count` <= kMergeCap)
    // one scan of both counts: candidates in the low 16 bits, elements above b* in the high
    // 16 (at most 1024 x KPT <= 32768 of either per CTA)
    uint32_t packed_total = 0;
    uint32_t j = cta_excl_scan((uint32_t)__popc(cand_bits) | ((uint32_t)__popc(above_bits) << 16), sm,
                               packed_total) & 0xFFFFu;
    const uint32_t n_loc = packed_total & 0xFFFFu, n_above = packed_total >> 16;
    for (uint32_t m = cand_bits; m; m &= m - 1) {
      const int step = __ffs(m) - 1;
      if (j < (uint32_t)kMergeCap) sm.m.loc[j] = comp(seg0 + 32 * step + lane);
      ++j;
    }
    if (threadIdx.x == 0) {
      sm.n_loc = n_loc;
      sm.n_above = n_above;
    }
    cluster_sync();  // #A: every CTA's list and counts are complete
    if ((int)threadIdx.x < C) {
      sm.q_cnt[threadIdx.x] = ld_cluster_u32(cluster_map(smem_u32(&sm.n_loc), threadIdx.x));
      sm.q_above[threadIdx.x] = ld_cluster_u32(cluster_map(smem_u32(&sm.n_above), threadIdx.x));
      sm.q_ge[threadIdx.x] = 0u;
    }
    __syncthreads();
    // every CTA's list, in rank order: per round, each thread's element of every list is
    // loaded first (up to kMaxC remote loads in flight), then stored
    uint32_t off[kMaxC], cnt[kMaxC];
    uint32_t M = 0, nmax = 0;
#pragma unroll
    for (int q = 0; q < kMaxC; ++q) {
      cnt[q] = q < C ? min(sm.q_cnt[q], (uint32_t)kMergeCap - M) : 0u;
      off[q] = M;
      M += cnt[q];
      nmax = max(nmax, cnt[q]);
    }
    for (uint32_t i = threadIdx.x; i < nmax; i += kCT) {
      unsigned long long vq[kMaxC];
#pragma unroll
      for (int q = 0; q < kMaxC; ++q)
        if (i < cnt[q]) vq[q] = ld_cluster_u64(cluster_map(smem_u32(&sm.m.loc[i]), q));
#pragma unroll
      for (int q = 0; q < kMaxC; ++q)
        if (i < cnt[q]) sm.m.mrg[off[q] + i] = vq[q];
    }
    cluster_arrive();  // done with the peers' memory (#B; its wait is at the very end)
    __syncthreads();
    // rank r among the gathered elements, on their low 52 bits (the top 12 are b*), by
    // radix digits of 11, 11, 10, 10, 10 bits until every element of the digit is needed
    constexpr unsigned long long kLow52 = (1ull << 52) - 1;
    unsigned long long p52 = 0;
    int ps = 52;
    uint32_t rr = r;
#pragma unroll 1
    for (int pass = 0; pass < 5; ++pass) {
      const int width = pass < 2 ? 11 : 10;
      const int shift = ps - width;
      const int bins = 1 << width;
      for (int b2 = threadIdx.x; b2 < bins; b2 += kCT) sm.part[b2] = 0u;
      __syncthreads();
      for (uint32_t i = threadIdx.x; i < M; i += kCT) {
        const unsigned long long c = sm.m.mrg[i] & kLow52;
        if (ps == 52 || (c >> ps) == (p52 >> ps)) atomicAdd(&sm.part[(uint32_t)(c >> shift) & (uint32_t)(bins - 1)], 1u);
      }
      __syncthreads();
      const int per = bins / kCT;
      uint32_t lv[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (i < per) lv[i] = sm.part[bins - 1 - per * (int)threadIdx.x - i];
      uint32_t dd, ab, cn;
      digit_search(lv, per, bins, rr, sm, dd, ab, cn);
      rr -= ab;
      p52 |= (unsigned long long)dd << shift;
      ps = shift;
      if (cn == rr) break;  // every element of this digit is selected
    }
    const unsigned long long thr = ((unsigned long long)bstar << 52) | p52;
    // selected elements per rank: those above b* and the gathered ones >= thr
    uint32_t start[kMaxC + 1];
    start[0] = 0;
    for (int q = 0; q < C; ++q) start[q + 1] = start[q] + min(sm.q_cnt[q], (uint32_t)kMergeCap - start[q]);
    for (uint32_t i = threadIdx.x; i < M; i += kCT)
      if (sm.m.mrg[i] >= thr) {
        int q = 0;
        while (q + 1 < C && i >= start[q + 1]) ++q;
        atomicAdd(&sm.q_ge[q], 1u);
      }
    __syncthreads();
    for (int q = 0; q < C; ++q) {
      const uint32_t n = sm.q_above[q] + sm.q_ge[q];
      if (q < me) base += n;
      total += n;
    }
    sel = above_bits;
    for (uint32_t m = cand_bits; m; m &= m - 1) {
      const int step = __ffs(m) - 1;
      if (comp(seg0 + 32 * step + lane) >= thr) sel |= 1u << step;
    }
  } else {
    // the elements that can be selected: bin >= b*; those in b* also count their second
    // digit (key bits 19..10) into this CTA's histogram when a second digit is needed
    const bool second = count != r;
    uint32_t cand = 0;
#pragma unroll
    for (int step = 0; step < KPT; ++step) {
      const int p = seg0 + 32 * step + lane;
      if (c0 + p < V) {
        const uint32_t key = keys[p];
        if ((key >> kHistShift) >= bstar) cand |= 1u << step;
        if (second && (key >> kHistShift) == bstar) atomicAdd(&sm.d.hl[(key >> 10) & 1023u], 1u);
      }
    }

    // later digits, until every element of the bin is needed: then the threshold is the
    // prefix itself.  Each CTA adds its non-empty bins into the bin's owner (CTA
    // bin / (bins / C), triple-buffered arrays), and after one barrier every CTA reads the
    // sums of the bins it scans from their owners.
    for (int level = 1; level < kLevels && count != r; ++level) {
      const int width = kDigitWidth[level];
      const int shift = pos - width;
      const int bins = 1 << width;
      const int bpc = bins / C;
      uint32_t* fb = sm.d.fullb[level % 3];
      if (level > 1) {  // the second digit was counted in the candidate pass
        for (int b = threadIdx.x; b < bins; b += kCT) sm.d.hl[b] = 0u;
        __syncthreads();
        for (uint32_t m = cand; m; m &= m - 1) {
          const int p = seg0 + 32 * (__ffs(m) - 1) + lane;
          const unsigned long long c = comp(p);
          if ((c >> pos) == (prefix >> pos)) atomicAdd(&sm.d.hl[(uint32_t)(c >> shift) & (uint32_t)(bins - 1)], 1u);
        }
      }
      __syncthreads();
      wait_s0();
      for (int b = threadIdx.x; b < bins; b += kCT) {
        const uint32_t x = sm.d.hl[b];
        if (x) red_cluster_add(cluster_map(smem_u32(&fb[b % bpc]), b / bpc), x);
      }
      // the owned part of the next level's array: its last readers were done two barriers ago
      for (int i = threadIdx.x; i < bpc; i += kCT) sm.d.fullb[(level + 1) % 3][i] = 0u;
      cluster_sync();  // every addition is in its owner
      const int per = bins / kCT;
      uint32_t lv[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int b = bins - 1 - per * (int)threadIdx.x - i;
        if (i < per) lv[i] = ld_cluster_u32(cluster_map(smem_u32(&fb[b % bpc]), b / bpc));
      }
      digit_search(lv, per, bins, r, sm, d, above, count);
      r -= above;
      prefix |= (unsigned long long)d << shift;
      pos = shift;
    }
    wait_s0();
    const unsigned long long thr = prefix;  // every element of the final bin is selected
    for (uint32_t m = cand; m; m &= m - 1) {
      const int step = __ffs(m) - 1;
      if (comp(seg0 + 32 * step + lane) >= thr) sel |= 1u << step;
    }
    // the selected counts of every rank, exchanged
    uint32_t cta_total = 0;
    (void)cta_excl_scan((uint32_t)__popc(sel), sm, cta_total);
    if ((int)threadIdx.x < C) st_cluster_u32(cluster_map(smem_u32(&sm.nsel[me]), threadIdx.x), cta_total);
    cluster_sync();  // every CTA's count is in every CTA; no shared-memory access across CTAs after this
    for (int q = 0; q < C; ++q) {
      if (q < me) base += sm.nsel[q];
      total += sm.nsel[q];
    }
  }
  // every row selects exactly k elements (k < V here); anything else is a broken invariant
  if (me == 0 && threadIdx.x == 0 && total != (uint32_t)k) atomicCAS(err, 0, 41);

  // output offset: the selected count of the lower ranks, then of the lower warps
  uint32_t wcnt = __popc(sel);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wcnt += __shfl_xor_sync(0xFFFFFFFFu, wcnt, o);
  if (lane == 0) sm.warp_tmp[warp] = wcnt;
  __syncthreads();
  const uint32_t wt = sm.warp_tmp[lane];
  uint32_t z = wt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, z, o);
    if (lane >= o) z += y;
  }
  uint32_t o = base + __shfl_sync(0xFFFFFFFFu, z - wt, warp);
#pragma unroll 4
  for (int step = 0; step < KPT; ++step) {
    const bool b = (sel >> step) & 1u;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, b);
    if (b) {
      const uint32_t at = o + __popc(m & ((1u << lane) - 1u));
      if (at < (uint32_t)k) out[at] = (int32_t)(c0 + seg0 + 32 * step + lane);
    }
    o += __popc(m);
  }
  if (merge) cluster_wait();  // #B: no CTA leaves while a peer may still read its list
}
template <int KPT>
cudaError_t launch_kpt(const float* scores, long long rows, int T, int N, long long q_pos0, int k, int C,
                       const uint32_t* hist, int32_t* idx, int* err, cudaStream_t stream) {
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
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // waits in-kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel<KPT>, scores, T, N, q_pos0, k, vec, hist, idx, err);
}

}  // namespace

// Cluster size C and keys per thread for rows of up to vmax visible positions: the
// smallest C (1, 2, 4, 8) whose chunk of 1024 x kpt positions, kpt <= 16, covers a row,
// else C = 8 with kpt = 32.  False when a row is longer than that, or when the clusters
// would not fit the GPU in about one wave (many rows: the scan kernels do better).
bool topk_cluster_plan(long long rows, long long vmax, int sms, int* C, int* kpt) {
  for (int c = 1; c <= 8; c *= 2) {
    const long long per = (vmax + (long long)c * kCT - 1) / ((long long)c * kCT);
    int kp = per <= 4 ? 4 : per <= 8 ? 8 : per <= 16 ? 16 : per <= 32 ? 32 : 0;
    if (kp == 0 || (kp == 32 && c < 8)) continue;
    if (rows * c > sms) return false;
    *C = c;
    *kpt = kp;
    return true;
  }
  return false;
}

cudaError_t launch_topk_cluster(const float* scores, int B, int T, int N, long long q_pos0, int k, int C, int kpt,
                                const uint32_t* hist, int32_t* idx, int* err, cudaStream_t stream) {
  const long long rows = (long long)B * T;
  switch (kpt) {
    case 4: return launch_kpt<4>(scores, rows, T, N, q_pos0, k, C, hist, idx, err, stream);
    case 8: return launch_kpt<8>(scores, rows, T, N, q_pos0, k, C, hist, idx, err, stream);
    case 16: return launch_kpt<16>(scores, rows, T, N, q_pos0, k, C, hist, idx, err, stream);
    case 32: return launch_kpt<32>(scores, rows, T, N, q_pos0, k, C, hist, idx, err, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
