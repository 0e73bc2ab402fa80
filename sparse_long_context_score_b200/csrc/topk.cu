// topk.cu -- per-query top-k select over the indexer scores.
//
// "GLM-5.2 1M architecture teardown", Cut 1: DSA -- keep the index_topk (2048) best
// history tokens per query; Cut 2: IndexShare -- the top-k list is computed once per
// group of 4 layers.
//
// Order: higher score first, ties to the lower token index, a NaN below every number,
// -0 == +0.  Every visible element s gets the 64-bit composite
//     C(s) = order_key(score[s]) << 32 | (0xFFFFFFFF - s)
// which is distinct per element and orders exactly as required, so the selection is
// "the k largest composites" and the answer is unique: bit-exact and deterministic.
//
// launch_topk sends rows that one cluster of CTAs can hold on chip (decode shapes) to
// topk_cluster.cu; the kernels here take many rows or long rows.
//
// Radix select over C, most significant digit first:
//   1. histogram of the top 12 bits (4096 bins) per row -- built here, or folded into
//      the indexer epilogue;
//   2. select kernel, grid (rows, chunks of 8192): every CTA finds the threshold bin b*
//      from the histogram, counts its elements above b*, appends the elements of bin b*
//      to a per-row candidate list (one reservation per CTA) and histograms their next
//      10 key bits into a per-row second-level histogram; the last CTA of a row (atomic
//      ticket, no waiting) finds the second digit from that histogram, ranks the few
//      elements of the final sub-bin directly (radix passes over the candidates, or over
//      the row when bin b* overflows the list, are the fallbacks), which gives the exact
//      threshold composite, and turns per-chunk counts into output offsets;
//   3. compact kernel, grid (rows, chunks): every element with C(s) >= threshold is
//      written at its chunk offset plus its warp-ballot rank, so the output comes out
//      in ascending token order.
// When a row has no more than k visible positions all of them are kept (0..V-1) and the
// row is padded with -1.
#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

static __device__ int g_topk_error;
SymbolAddress g_topk_err_addr;

constexpr int kHistThreads = 256;
constexpr int kSelThreads = 512;
constexpr int kCmpThreads = 256;
constexpr uint64_t kLow52 = (1ull << 52) - 1;

// row_state words
constexpr int RS_CAND = 0;    // candidates appended (atomic)
constexpr int RS_TICKET = 1;  // select CTAs finished (atomic)
constexpr int RS_BSTAR = 2;
constexpr int RS_ABOVE = 3;
constexpr int RS_THR_LO = 4;
constexpr int RS_THR_HI = 5;

__device__ __forceinline__ uint64_t composite(uint32_t key, uint32_t s) {
  return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - s);
}

__device__ __forceinline__ int row_t(int row, int T) { return row % T; }

__global__ void __launch_bounds__(kHistThreads)
topk_hist_kernel(const float* __restrict__ scores, int T, int N, long long q_pos0, uint32_t* __restrict__ hist) {
  const int row = blockIdx.x;
  const long long V = visible_count(N, q_pos0, row_t(row, T));
  const long long s0 = (long long)blockIdx.y * kTopkChunk;
  if (s0 >= V) return;
  const long long s1 = min(s0 + (long long)kTopkChunk, V);
  __shared__ uint32_t sh[kHistBins];
  for (int i = threadIdx.x; i < kHistBins; i += kHistThreads) sh[i] = 0;
  __syncthreads();
  const float* sr = scores + (size_t)row * N;
  for (long long s = s0 + threadIdx.x; s < s1; s += kHistThreads) atomicAdd(&sh[order_key(sr[s]) >> kHistShift], 1u);
  __syncthreads();
  uint32_t* gh = hist + (size_t)row * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += kHistThreads)
    if (sh[i]) atomicAdd(&gh[i], sh[i]);
}

// Block-wide exclusive scan of one value per thread (kSelThreads threads).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t wv = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0u;
    uint32_t z = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xFFFFFFFFu, z, o);
      if (lane >= o) z += y;
    }
    if (lane < (int)(blockDim.x >> 5)) s_warp[lane] = z - wv;
    if (lane == 31) *total = z;
  }
  __syncthreads();
  const uint32_t r = s_warp[warp] + x - v;
  __syncthreads();
  return r;
}

constexpr int kRadixBins = 2048;  // digits of the resolve: 10, 10, 11, 11, 10 bits

constexpr int kMaxSmemChunks = 4096;  // rows up to 32M scores keep their chunk counts in SMEM

constexpr int kFinalCap = 1024;  // final sub-bin sizes ranked directly

struct SelectSmem {
  uint32_t radix[kRadixBins];
  uint32_t chunk_cnt[kMaxSmemChunks];
  uint32_t hist2[kHist2Bins];
  uint64_t fin[kFinalCap];
  uint32_t warp_tmp[32];
  uint32_t total;
  uint32_t digit, digit_above, digit_count, is_last, cand_base, nfin;
  unsigned long long thr;
};

// Digit search: with `bins` counts (bins <= 8 * kSelThreads), find the
// digit d where the count from the top reaches r:  above(d) < r <= above(d) + count(d).
// Every thread of the block must call it; results land in sm.digit / digit_above /
// digit_count.
template <class Load>
__device__ __forceinline__ void find_digit(SelectSmem& sm, int bins, uint32_t r, Load load) {
  const int per = bins > kSelThreads ? bins / kSelThreads : 1;
  const int hi = bins - (int)threadIdx.x * per;  // this thread owns bins [hi - per, hi)
  uint32_t local[8];
  uint32_t lsum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = hi - 1 - i;
    local[i] = (i < per && b >= 0) ? load(b) : 0u;
    lsum += local[i];
  }
  if (threadIdx.x == 0) {
    sm.digit = 0;
    sm.digit_above = 0;
    sm.digit_count = 0;
  }
  const uint32_t above = block_excl_scan(lsum, sm.warp_tmp, &sm.total);
  uint32_t run = above;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i < per && hi - 1 - i >= 0 && run < r && run + local[i] >= r) {
      sm.digit = (uint32_t)(hi - 1 - i);
      sm.digit_above = run;
      sm.digit_count = local[i];
    }
    run += local[i];
  }
  __syncthreads();
}

// Radix passes over the low 52 bits of the threshold-bin composites (key bits 19..0,
// then the inverted index).  `get(i, c)` yields element i's composite, or false when
// element i is not in the threshold bin.  Returns the threshold: the selected elements
// are exactly those whose composite is >= it.
template <class Get>
__device__ uint64_t resolve_threshold(SelectSmem& sm, long long count, uint32_t remaining, Get get) {
  constexpr int kWidths[5] = {10, 10, 11, 11, 10};
  unsigned long long prefix = 0;
  int shift = 52;
#pragma unroll 1
  for (int pass = 0; pass < 5; ++pass) {
    const int width = kWidths[pass];
    const int hi_shift = shift;
    shift -= width;
    const uint32_t mask = (1u << width) - 1u;
    for (int i = threadIdx.x; i < (1 << width); i += kSelThreads) sm.radix[i] = 0;
    __syncthreads();
    for (long long i = threadIdx.x; i < count; i += kSelThreads) {
      uint64_t c;
      if (!get(i, c)) continue;
      c &= kLow52;
      if (hi_shift >= 52 || (c >> hi_shift) == (prefix >> hi_shift))
        atomicAdd(&sm.radix[(uint32_t)(c >> shift) & mask], 1u);
    }
    __syncthreads();
    find_digit(sm, 1 << width, remaining, [&](int b) { return sm.radix[b]; });
    remaining -= sm.digit_above;
    prefix |= (unsigned long long)sm.digit << shift;
    const bool done = sm.digit_count == remaining;  // every element of this digit is selected
    __syncthreads();
    if (done) break;
  }
  return prefix;
}

__global__ void __launch_bounds__(kSelThreads)
topk_select_kernel(const float* __restrict__ scores, int T, int N, long long q_pos0, int k, TopkWorkspace ws,
                   int32_t* __restrict__ idx_out, int vec, int* __restrict__ err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smem_raw);
  const int row = blockIdx.x;
  const int chunk = blockIdx.y;
  const int nchunks = gridDim.y;
  const long long V = visible_count(N, q_pos0, row_t(row, T));
  uint32_t* state = ws.row_state + (size_t)row * kRowStateWords;

  if (V <= k) {
    // every visible position is kept; pad the rest of the row
    if (chunk == 0)
      for (long long j = V + threadIdx.x; j < k; j += kSelThreads) idx_out[(size_t)row * k + j] = -1;
    return;
  }

  // 1. threshold bin b*: the bin where the count from the top reaches k
  const uint32_t* gh = ws.hist + (size_t)row * kHistBins;
  find_digit(sm, kHistBins, (uint32_t)k, [&](int b) { return __ldcg(&gh[b]); });
  const uint32_t bstar = sm.digit;
  const uint32_t above = sm.digit_above;
  const uint32_t bcount = sm.digit_count;
  const bool use_cand = bcount <= (uint32_t)kCandCap;
  for (int i = threadIdx.x; i < kHist2Bins; i += kSelThreads) sm.hist2[i] = 0;

  // 2. scan this chunk: count the elements above b*, append the elements of b* (one
  //    reservation per CTA on the row's candidate counter, after a block scan)
  const float* sr = scores + (size_t)row * N;
  const long long s0 = (long long)chunk * kTopkChunk;
  const long long s1 = min(s0 + (long long)kTopkChunk, V);
  uint64_t* cand = ws.cand + (size_t)row * kCandCap;
  constexpr int kPerThread = kTopkChunk / kSelThreads;  // 16
  uint32_t keys[kPerThread];
  uint32_t cand_bits = 0, inb_bits = 0, n_above = 0;
  auto elem = [&](int i) -> long long {
    // element i of this thread: four consecutive scores per 16-byte group
    return s0 + 4LL * (threadIdx.x + kSelThreads * (i >> 2)) + (i & 3);
  };
  if (vec) {
    float4 v[kPerThread / 4];
#pragma unroll
    for (int g = 0; g < kPerThread / 4; ++g) {
      const long long e = elem(4 * g);
      v[g] = e + 3 < s1 ? __ldcg(reinterpret_cast<const float4*>(sr + e))
                        : make_float4(e < s1 ? sr[e] : 0.f, e + 1 < s1 ? sr[e + 1] : 0.f,
                                      e + 2 < s1 ? sr[e + 2] : 0.f, 0.f);
    }
#pragma unroll
    for (int g = 0; g < kPerThread / 4; ++g) {
      keys[4 * g + 0] = order_key(v[g].x);
      keys[4 * g + 1] = order_key(v[g].y);
      keys[4 * g + 2] = order_key(v[g].z);
      keys[4 * g + 3] = order_key(v[g].w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const long long e = elem(i);
      keys[i] = e < s1 ? order_key(sr[e]) : 0u;
    }
  }
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const bool in = elem(i) < s1;
    const uint32_t bin = keys[i] >> kHistShift;
    n_above += (in && bin > bstar) ? 1u : 0u;
    inb_bits |= (in && bin == bstar) ? (1u << i) : 0u;
  }
  if (use_cand) cand_bits = inb_bits;
  // the second digit of every element of b* is counted, whether or not the candidates fit
#pragma unroll
  for (int i = 0; i < kPerThread; ++i)
    if (inb_bits & (1u << i)) atomicAdd(&sm.hist2[(keys[i] >> 10) & (kHist2Bins - 1)], 1u);
  const uint32_t my_off = block_excl_scan((uint32_t)__popc(cand_bits), sm.warp_tmp, &sm.total);
  if (threadIdx.x == 0) sm.cand_base = sm.total ? atomicAdd(&state[RS_CAND], sm.total) : 0u;
  __syncthreads();
  {
    uint32_t pos = sm.cand_base + my_off;
#pragma unroll
    for (int i = 0; i < kPerThread; ++i)
      if (cand_bits & (1u << i)) {
        if (pos < (uint32_t)kCandCap) cand[pos] = composite(keys[i], (uint32_t)elem(i));
        ++pos;
      }
  }
  (void)block_excl_scan(n_above, sm.warp_tmp, &sm.total);
  if (threadIdx.x == 0) ws.chunk_above[(size_t)row * nchunks + chunk] = sm.total;
  {
    uint32_t* g2 = ws.hist2 + (size_t)row * kHist2Bins;
    for (int i = threadIdx.x; i < kHist2Bins; i += kSelThreads)
      if (sm.hist2[i]) atomicAdd(&g2[i], sm.hist2[i]);
  }

  // 3. the last CTA of the row resolves the threshold
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) sm.is_last = atomicAdd(&state[RS_TICKET], 1u) == (uint32_t)(nchunks - 1);
  __syncthreads();
  if (!sm.is_last) return;
  __threadfence();

  const uint32_t remaining = (uint32_t)k - above;  // 1 <= remaining <= bcount
  const bool smem_cnt = nchunks <= kMaxSmemChunks;
  uint32_t* csel = ws.chunk_sel + (size_t)row * nchunks;
  uint32_t* cnt = smem_cnt ? sm.chunk_cnt : csel;
  if (smem_cnt)
    for (int c = threadIdx.x; c < nchunks; c += kSelThreads) sm.chunk_cnt[c] = 0;
  if (threadIdx.x == 0) {
    sm.nfin = 0;
    sm.thr = 0;
  }
  uint64_t thr = 0;
  bool resolved = false;
  // 4. second digit from the row's second-level histogram (complete: every CTA counted all
  //    its elements of b*); the elements of the final sub-bin (usually a handful) are
  //    collected -- from the candidate list, or when that overflowed in one pass over the
  //    row -- and ranked directly
  const uint32_t* g2 = ws.hist2 + (size_t)row * kHist2Bins;
  find_digit(sm, kHist2Bins, remaining, [&](int bin) { return __ldcg(&g2[bin]); });
  const uint32_t d2 = sm.digit, r2 = remaining - sm.digit_above, n2 = sm.digit_count;
  if (n2 <= (uint32_t)kFinalCap) {
    if (use_cand) {
      for (long long i = threadIdx.x; i < bcount; i += kSelThreads) {
        const uint64_t c = __ldcg(&cand[i]);
        const uint32_t dg = (uint32_t)(c >> 42) & (kHist2Bins - 1);
        if (dg > d2) atomicAdd(&cnt[(0xFFFFFFFFu - (uint32_t)c) / kTopkChunk], 1u);
        else if (dg == d2) {
          const uint32_t pos = atomicAdd(&sm.nfin, 1u);
          if (pos < (uint32_t)kFinalCap) sm.fin[pos] = c;
        }
      }
    } else {
      for (long long s2 = threadIdx.x; s2 < V; s2 += kSelThreads) {
        const uint32_t key = order_key(__ldcg(&sr[s2]));
        if ((key >> kHistShift) != bstar) continue;
        const uint32_t dg = (key >> 10) & (kHist2Bins - 1);
        if (dg > d2) atomicAdd(&cnt[s2 / kTopkChunk], 1u);
        else if (dg == d2) {
          const uint32_t pos = atomicAdd(&sm.nfin, 1u);
          if (pos < (uint32_t)kFinalCap) sm.fin[pos] = composite(key, (uint32_t)s2);
        }
      }
    }
    __syncthreads();
    const uint32_t nf = min(sm.nfin, (uint32_t)kFinalCap);  // == n2
    for (uint32_t i = threadIdx.x; i < nf; i += kSelThreads) {
      const uint64_t c = sm.fin[i];
      uint32_t rank = 0;
      for (uint32_t j = 0; j < nf; ++j) rank += sm.fin[j] > c ? 1u : 0u;
      if (rank == r2 - 1) sm.thr = c;  // composites are distinct: exactly one thread writes
    }
    __syncthreads();
    thr = sm.thr;
    for (uint32_t i = threadIdx.x; i < nf; i += kSelThreads) {
      const uint64_t c = sm.fin[i];
      if (c >= thr) atomicAdd(&cnt[(0xFFFFFFFFu - (uint32_t)c) / kTopkChunk], 1u);
    }
    resolved = true;
  } else if (use_cand) {
    // many equal high bits: radix passes over the candidate list
    const uint64_t thr52 = resolve_threshold(sm, bcount, remaining, [&](long long i, uint64_t& c) {
      c = __ldcg(&cand[i]);
      return true;
    });
    thr = ((uint64_t)bstar << 52) | thr52;
    for (long long i = threadIdx.x; i < bcount; i += kSelThreads) {
      const uint64_t c = __ldcg(&cand[i]);
      if (c >= thr) atomicAdd(&cnt[(0xFFFFFFFFu - (uint32_t)c) / kTopkChunk], 1u);
    }
    resolved = true;
  }
  if (!resolved) {
    // the final sub-bin is large and the candidates overflowed: radix passes over the row
    const uint64_t thr52 = resolve_threshold(sm, V, remaining, [&](long long s2, uint64_t& c) {
      const uint32_t key = order_key(__ldcg(&sr[s2]));
      if ((key >> kHistShift) != bstar) return false;
      c = composite(key, (uint32_t)s2);
      return true;
    });
    thr = ((uint64_t)bstar << 52) | thr52;
    for (long long s2 = threadIdx.x; s2 < V; s2 += kSelThreads) {
      const uint32_t key = order_key(__ldcg(&sr[s2]));
      if ((key >> kHistShift) == bstar && composite(key, (uint32_t)s2) >= thr) atomicAdd(&cnt[s2 / kTopkChunk], 1u);
    }
  }
  __threadfence();
  __syncthreads();

  // 5. output offset of every chunk
  uint32_t carry = 0;
  for (int c0 = 0; c0 < nchunks; c0 += kSelThreads) {
    const int c = c0 + threadIdx.x;
    const uint32_t v = c < nchunks ? __ldcg(&ws.chunk_above[(size_t)row * nchunks + c]) + (smem_cnt ? sm.chunk_cnt[c] : __ldcg(&csel[c])) : 0u;
    const uint32_t off = block_excl_scan(v, sm.warp_tmp, &sm.total);
    if (c < nchunks) ws.chunk_off[(size_t)row * nchunks + c] = carry + off;
    carry += sm.total;
    __syncthreads();
  }
  // every row selects exactly k elements (k < V here); anything else is a broken invariant
  if (threadIdx.x == 0 && carry != (uint32_t)k) atomicCAS(err, 0, 42);
  if (threadIdx.x == 0) {
    state[RS_THR_LO] = (uint32_t)thr;
    state[RS_THR_HI] = (uint32_t)(thr >> 32);
    state[RS_BSTAR] = bstar;
    state[RS_ABOVE] = above;
  }
}

__global__ void __launch_bounds__(kCmpThreads)
topk_compact_kernel(const float* __restrict__ scores, int T, int N, long long q_pos0, int k, TopkWorkspace ws,
                    int32_t* __restrict__ idx_out, int vec) {
  const int row = blockIdx.x;
  const int chunk = blockIdx.y;
  const int nchunks = gridDim.y;
  const long long V = visible_count(N, q_pos0, row_t(row, T));
  const long long s0 = (long long)chunk * kTopkChunk;
  if (s0 >= V) return;
  const long long s1 = min(s0 + (long long)kTopkChunk, V);
  const bool take_all = V <= k;
  uint64_t thr = 0;
  long long base = s0;
  if (!take_all) {
    const uint32_t* state = ws.row_state + (size_t)row * kRowStateWords;
    thr = ((uint64_t)__ldcg(&state[RS_THR_HI]) << 32) | __ldcg(&state[RS_THR_LO]);
    base = __ldcg(&ws.chunk_off[(size_t)row * nchunks + chunk]);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarpsC = kCmpThreads / 32;
  constexpr int kSeg = kTopkChunk / kWarpsC;  // 1024 scores per warp
  constexpr int kGroups = kSeg / 128;          // 8 groups of 32 lanes x 4 scores
  const long long g0 = s0 + (long long)warp * kSeg;
  const float* sr = scores + (size_t)row * N;
  __shared__ uint32_t s_cnt[kWarpsC];
  int32_t* out = idx_out + (size_t)row * k;

  auto sel = [&](long long e, float v) {
    return e < s1 && (take_all || composite(order_key(v), (uint32_t)e) >= thr);
  };

  if (vec) {
    float4 v[kGroups];
#pragma unroll
    for (int i = 0; i < kGroups; ++i) {
      const long long e = g0 + 128LL * i + 4 * lane;
      v[i] = e + 3 < s1 ? __ldcg(reinterpret_cast<const float4*>(sr + e))
                        : make_float4(e < s1 ? sr[e] : 0.f, e + 1 < s1 ? sr[e + 1] : 0.f,
                                      e + 2 < s1 ? sr[e + 2] : 0.f, 0.f);
    }
    uint32_t bits[kGroups];
    uint32_t total = 0;
#pragma unroll
    for (int i = 0; i < kGroups; ++i) {
      const long long e = g0 + 128LL * i + 4 * lane;
      bits[i] = (sel(e, v[i].x) ? 1u : 0u) | (sel(e + 1, v[i].y) ? 2u : 0u) | (sel(e + 2, v[i].z) ? 4u : 0u) |
                (sel(e + 3, v[i].w) ? 8u : 0u);
      uint32_t c = __popc(bits[i]);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, c, o);
        if (lane >= o) c += y;
      }
      total += __shfl_sync(0xFFFFFFFFu, c, 31);
    }
    if (lane == 0) s_cnt[warp] = total;
    __syncthreads();
    long long off = base;
    for (int w = 0; w < warp; ++w) off += s_cnt[w];
#pragma unroll
    for (int i = 0; i < kGroups; ++i) {
      const uint32_t c = __popc(bits[i]);
      uint32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      const long long e = g0 + 128LL * i + 4 * lane;
      long long pos = off + incl - c;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (bits[i] & (1u << j)) {
          if (pos < k) out[pos] = (int32_t)(e + j);
          ++pos;
        }
      off += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
  } else {
    const long long g1 = min(g0 + kSeg, s1);
    uint32_t cnt = 0;
    for (long long s = g0; s < g1; s += 32) {
      const long long e = s + lane;
      cnt += __popc(__ballot_sync(0xFFFFFFFFu, e < g1 && sel(e, sr[e])));
    }
    if (lane == 0) s_cnt[warp] = cnt;
    __syncthreads();
    long long off = base;
    for (int w = 0; w < warp; ++w) off += s_cnt[w];
    for (long long s = g0; s < g1; s += 32) {
      const long long e = s + lane;
      const bool p = e < g1 && sel(e, sr[e]);
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, p);
      const long long pos = off + __popc(m & ((1u << lane) - 1u));
      if (p && pos < k) out[pos] = (int32_t)e;
      off += __popc(m);
    }
  }
}

// ---------------------------------------------------------------------------- long rows
// One launch for rows longer than a cluster holds (a 1M-token decode row), when all the
// CTAs of the launch fit the GPU at once (a cooperative launch checks it): CTA (chunk, row)
// keeps its 8192 order keys in shared memory, and the CTAs of a row meet at row barriers
// (a counter in the workspace, bounded spins) to refine the threshold digit by digit -- the
// first 12 bits from the row's histogram, then 10 bits at a time -- until the threshold
// bin holds at most kLongCap elements.  Those are appended to the row's candidate list,
// with every chunk's count above the bin; after one more row barrier every CTA ranks the
// candidates itself, takes the output offset of its chunk from the counts and writes its
// positions in order.  No CTA re-reads the scores from memory.
constexpr int kLongCap = 4096;             // threshold-bin elements ranked in shared memory
constexpr int kLongLevels = 6;             // digit widths after the first: 10,10,10,10,10,2
constexpr int RS_SYNC0 = 6;                // row_state words 6.. : row barrier counters
constexpr int kLongMaxChunks = 512;        // rows of up to 4M positions

// ~50 KB, so that four CTAs share an SM (the candidates are read from L2)
struct LongSmem {
  uint32_t keys[kTopkChunk];
  uint32_t radix[kHistBins];               // digit histograms (the first digit's too)
  uint32_t chunk_ge[kLongMaxChunks];
  uint32_t warp_tmp[32];
  uint32_t total;
  uint32_t digit, digit_above, digit_count, cand_base;
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Every CTA of the row arrives, then waits (bounded) until all `n` have: writes before it
// are visible to every CTA of the row after it.  Returns false after recording `code` when
// the wait ran out.
__device__ bool row_barrier(uint32_t* counter, uint32_t n, int* err, int code) {
  __syncthreads();
  __shared__ int ok_s;
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(counter, 1u);
    int ok = 1;
    const long long t0 = clock64();
    while (ld_acquire_gpu(counter) < n) {
      __nanosleep(64);
      if (clock64() - t0 > sm100::kWaitLimitCycles) {
        atomicCAS(err, 0, code);
        ok = 0;
        break;
      }
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// The LongSmem flavour of the block-wide digit search: sm.digit etc. (bins <= 8 x 512).
template <class Load>
__device__ __forceinline__ void find_digit_l(LongSmem& sm, int bins, uint32_t r, Load load) {
  const int per = bins > kSelThreads ? bins / kSelThreads : 1;
  const int hi = bins - (int)threadIdx.x * per;
  uint32_t local[8];
  uint32_t lsum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = hi - 1 - i;
    local[i] = (i < per && b >= 0) ? load(b) : 0u;
    lsum += local[i];
  }
  if (threadIdx.x == 0) {
    sm.digit = 0;
    sm.digit_above = 0;
    sm.digit_count = 0;
  }
  const uint32_t above = block_excl_scan(lsum, sm.warp_tmp, &sm.total);
  uint32_t run = above;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i < per && hi - 1 - i >= 0 && run < r && run + local[i] >= r) {
      sm.digit = (uint32_t)(hi - 1 - i);
      sm.digit_above = run;
      sm.digit_count = local[i];
    }
    run += local[i];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads)
topk_long_kernel(const float* __restrict__ scores, int T, int N, long long q_pos0, int k, TopkWorkspace ws,
                 int hist_ready, int32_t* __restrict__ idx_out, int* __restrict__ err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  LongSmem& sm = *reinterpret_cast<LongSmem*>(smem_raw);
  const int chunk = blockIdx.x, row = blockIdx.y, nchunks = gridDim.x;
  const long long V = visible_count(N, q_pos0, row_t(row, T));
  const long long s0 = (long long)chunk * kTopkChunk;
  const int n = (int)max(0LL, min((long long)kTopkChunk, V - s0));  // this chunk's visible positions
  int32_t* out = idx_out + (size_t)row * k;
  if (V <= k) {
    // every visible position is kept; the rest of the row is padding (the same in every CTA
    // of the row, so none of them waits at a row barrier)
    for (int i = threadIdx.x; i < n; i += kSelThreads) out[s0 + i] = (int32_t)(s0 + i);
    if (chunk == 0)
      for (long long j = V + threadIdx.x; j < k; j += kSelThreads) out[j] = -1;
    return;
  }
  uint32_t* state = ws.row_state + (size_t)row * kRowStateWords;
  uint32_t* hist = ws.hist + (size_t)row * kHistBins;
  const float* sr = scores + (size_t)row * N + s0;
  for (int i = threadIdx.x; i < kTopkChunk; i += kSelThreads) sm.keys[i] = i < n ? order_key(__ldcg(sr + i)) : 0u;
  auto comp = [&](int i) -> uint64_t { return composite(sm.keys[i], (uint32_t)(s0 + i)); };
  int sync = 0;
  bool ok = true;
  if (!hist_ready) {
    // the first digit's histogram of the row (the indexer counts it in decode)
    for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) sm.radix[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kSelThreads) atomicAdd(&sm.radix[sm.keys[i] >> kHistShift], 1u);
    __syncthreads();
    for (int i = threadIdx.x; i < kHistBins; i += kSelThreads)
      if (sm.radix[i]) atomicAdd(&hist[i], sm.radix[i]);
    ok = row_barrier(&state[RS_SYNC0 + sync++], nchunks, err, 45);
  }
  // first digit: the bin where the count from the top reaches k
  find_digit_l(sm, kHistBins, (uint32_t)k, [&](int b) { return __ldcg(&hist[b]); });
  uint64_t prefix = (uint64_t)sm.digit << 52;
  int pos = 52;                          // bits [pos, 64) of the threshold are fixed
  uint32_t r = (uint32_t)k - sm.digit_above;
  uint32_t cnt = sm.digit_count;
  // further digits while the bin is too large to rank in shared memory
  for (int level = 0; ok && cnt > (uint32_t)kLongCap && pos > 0 && level < kLongLevels; ++level) {
    const int width = level < 5 ? 10 : 2;
    const int shift = pos - width;
    const uint32_t mask = (1u << width) - 1u;
    uint32_t* buf = level % 3 == 0 ? ws.hist2 + (size_t)row * kHist2Bins
                                   : ws.lvl + ((size_t)row * 2 + (level % 3 - 1)) * kHist2Bins;
    for (int i = threadIdx.x; i < kHist2Bins; i += kSelThreads) sm.radix[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kSelThreads) {
      const uint64_t c = comp(i);
      if ((c >> pos) == (prefix >> pos)) atomicAdd(&sm.radix[(uint32_t)(c >> shift) & mask], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i <= (int)mask; i += kSelThreads)
      if (sm.radix[i]) atomicAdd(&buf[i], sm.radix[i]);
    // the buffer of level + 1 (last read two levels ago, before the previous barrier):
    // this CTA's share of it back to zero
    if (level >= 2) {
      uint32_t* nb = (level + 1) % 3 == 0 ? ws.hist2 + (size_t)row * kHist2Bins
                                          : ws.lvl + ((size_t)row * 2 + ((level + 1) % 3 - 1)) * kHist2Bins;
      const int per = (kHist2Bins + nchunks - 1) / nchunks;
      for (int i = chunk * per + (int)threadIdx.x; i < min(kHist2Bins, (chunk + 1) * per); i += kSelThreads) nb[i] = 0u;
    }
    ok = row_barrier(&state[RS_SYNC0 + sync++], nchunks, err, 45);
    find_digit_l(sm, (int)mask + 1, r, [&](int b) { return __ldcg(&buf[b]); });
    r -= sm.digit_above;
    prefix |= (uint64_t)sm.digit << shift;
    pos = shift;
    cnt = sm.digit_count;
  }
  // this chunk's elements above the threshold bin, and its elements in it (the candidates)
  uint32_t n_above = 0, n_in = 0;
  for (int i = threadIdx.x; i < n; i += kSelThreads) {
    const uint64_t hi = comp(i) >> pos, ph = prefix >> pos;
    n_above += hi > ph ? 1u : 0u;
    n_in += hi == ph ? 1u : 0u;
  }
  (void)block_excl_scan(n_above, sm.warp_tmp, &sm.total);
  if (threadIdx.x == 0) ws.chunk_above[(size_t)row * nchunks + chunk] = sm.total;
  const uint32_t off = block_excl_scan(n_in, sm.warp_tmp, &sm.total);
  if (threadIdx.x == 0) sm.cand_base = sm.total ? atomicAdd(&state[RS_CAND], sm.total) : 0u;
  __syncthreads();
  {
    uint64_t* cand = ws.cand + (size_t)row * kCandCap;
    uint32_t at = sm.cand_base + off;
    for (int i = threadIdx.x; i < n; i += kSelThreads) {
      const uint64_t c = comp(i);
      if ((c >> pos) == (prefix >> pos)) {
        if (at < (uint32_t)kCandCap) cand[at] = c;
        ++at;
      }
    }
  }
  ok = ok && row_barrier(&state[RS_SYNC0 + kLongLevels + 1], nchunks, err, 45);
  if (!ok) return;
  // every CTA ranks the candidates (at most kLongCap, read from L2) on their bits below `pos`
  const uint32_t M = min(cnt, (uint32_t)kLongCap);
  const uint64_t* cand = ws.cand + (size_t)row * kCandCap;
  uint64_t thr = prefix;
  if (cnt != r) {
    int ps = pos;
    uint64_t p2 = prefix;
#pragma unroll 1
    while (ps > 0) {
      const int width = ps >= 11 ? 11 : ps;
      const int shift = ps - width;
      const uint32_t mask = (1u << width) - 1u;
      for (int i = threadIdx.x; i <= (int)mask; i += kSelThreads) sm.radix[i] = 0u;
      __syncthreads();
      for (uint32_t i = threadIdx.x; i < M; i += kSelThreads) {
        const uint64_t c = __ldcg(&cand[i]);
        if ((c >> ps) == (p2 >> ps)) atomicAdd(&sm.radix[(uint32_t)(c >> shift) & mask], 1u);
      }
      __syncthreads();
      find_digit_l(sm, (int)mask + 1, r, [&](int b) { return sm.radix[b]; });
      r -= sm.digit_above;
      p2 |= (uint64_t)sm.digit << shift;
      ps = shift;
      const bool done = sm.digit_count == r;  // every element of this digit is selected
      __syncthreads();
      if (done) break;
    }
    thr = p2;
  }
  // selected = composite >= thr.  Output offset of this chunk: the selected elements of the
  // chunks before it (those above the bin, counted by each chunk, and the candidates >= thr)
  for (int i = threadIdx.x; i < nchunks; i += kSelThreads) sm.chunk_ge[i] = 0u;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < M; i += kSelThreads) {
    const uint64_t c = __ldcg(&cand[i]);
    if (c >= thr) atomicAdd(&sm.chunk_ge[(0xFFFFFFFFu - (uint32_t)c) / kTopkChunk], 1u);
  }
  __syncthreads();
  uint32_t before = 0, all = 0;
  for (int c = threadIdx.x; c < nchunks; c += kSelThreads) {
    const uint32_t v = __ldcg(&ws.chunk_above[(size_t)row * nchunks + c]) + sm.chunk_ge[c];
    if (c < chunk) before += v;
    all += v;
  }
  (void)block_excl_scan(before, sm.warp_tmp, &sm.total);
  const uint32_t base = sm.total;
  (void)block_excl_scan(all, sm.warp_tmp, &sm.total);
  if (chunk == 0 && threadIdx.x == 0 && sm.total != (uint32_t)k) atomicCAS(err, 0, 44);
  // this chunk's selected positions in ascending order: 16 per thread, consecutive
  constexpr int kPer = kTopkChunk / kSelThreads;
  uint32_t bits = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = (int)threadIdx.x * kPer + j;
    if (i < n && comp(i) >= thr) bits |= 1u << j;
  }
  uint32_t at = base + block_excl_scan((uint32_t)__popc(bits), sm.warp_tmp, &sm.total);
#pragma unroll
  for (int j = 0; j < kPer; ++j)
    if (bits & (1u << j)) {
      if (at < (uint32_t)k) out[at] = (int32_t)(s0 + (int)threadIdx.x * kPer + j);
      ++at;
    }
}

}  // namespace

cudaError_t topk_error_word(int** p) { return g_topk_err_addr.get(g_topk_error, p); }

size_t topk_workspace_bytes(long long rows, int N) {
  const long long nchunks = ((long long)N + kTopkChunk - 1) / kTopkChunk;
  size_t b = 0;
  b += (size_t)rows * kHistBins * 4;
  b += (size_t)rows * kRowStateWords * 4;
  b += (size_t)rows * nchunks * 4 * 3;
  b += (size_t)rows * kHist2Bins * 4 * 3;
  b = (b + 255) & ~(size_t)255;
  b += (size_t)rows * kCandCap * 8;
  return (b + 255) & ~(size_t)255;
}

TopkWorkspace topk_workspace(void* base, long long rows, int N) {
  const long long nchunks = ((long long)N + kTopkChunk - 1) / kTopkChunk;
  TopkWorkspace w;
  unsigned char* p = static_cast<unsigned char*>(base);
  w.hist = reinterpret_cast<uint32_t*>(p);
  p += (size_t)rows * kHistBins * 4;
  w.row_state = reinterpret_cast<uint32_t*>(p);
  p += (size_t)rows * kRowStateWords * 4;
  w.chunk_sel = reinterpret_cast<uint32_t*>(p);
  p += (size_t)rows * nchunks * 4;
  w.hist2 = reinterpret_cast<uint32_t*>(p);
  p += (size_t)rows * kHist2Bins * 4;
  w.lvl = reinterpret_cast<uint32_t*>(p);
  p += (size_t)rows * kHist2Bins * 4 * 2;
  w.zero_bytes = (size_t)(p - static_cast<unsigned char*>(base));
  w.chunk_above = reinterpret_cast<uint32_t*>(p);
  p += (size_t)rows * nchunks * 4;
  w.chunk_off = reinterpret_cast<uint32_t*>(p);
  p += (size_t)rows * nchunks * 4;
  size_t off = (size_t)(p - static_cast<unsigned char*>(base));
  off = (off + 255) & ~(size_t)255;
  w.cand = reinterpret_cast<uint64_t*>(static_cast<unsigned char*>(base) + off);
  return w;
}

namespace {
// CTAs of topk_long_kernel that one SM holds (0 if unknown), per device
int long_per_sm() {
  static std::atomic<int> cap[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int c = cap[dev].load(std::memory_order_relaxed);
  if (c > 0) return c;
  const int smem = (int)sizeof(LongSmem);
  if (cudaFuncSetAttribute(topk_long_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_long_kernel, kSelThreads, smem) != cudaSuccess) return 0;
  cap[dev].store(per_sm, std::memory_order_relaxed);
  return per_sm;
}

int budget_sms(int sm_budget) {
  const int sms = device_sm_count();
  return sm_budget > 0 && sm_budget < sms ? sm_budget : sms;
}
}  // namespace

bool topk_uses_workspace(long long rows, long long vmax) {
  int C = 0, kpt = 0;
  return !topk_cluster_plan(rows, vmax, budget_sms(0), &C, &kpt);
}

cudaError_t launch_topk(const float* scores, int B, int T, int N, long long q_pos0, int k, int32_t* idx,
                        const TopkWorkspace& ws, bool hist_ready, int sm_budget, cudaStream_t stream) {
  const long long rows = (long long)B * T;
  const long long vmax = visible_count(N, q_pos0, T - 1);
  const long long nchunks_all = ((long long)N + kTopkChunk - 1) / kTopkChunk;
  cudaError_t e;
  int C = 0, kpt = 0;
  int* err = nullptr;
  if ((e = g_topk_err_addr.get(g_topk_error, &err)) != cudaSuccess) return e;
  const int sms = budget_sms(sm_budget);
  if (topk_cluster_plan(rows, vmax, sms, &C, &kpt))
    return launch_topk_cluster(scores, B, T, N, q_pos0, k, C, kpt, hist_ready ? ws.hist : nullptr, idx, err, stream);
  // long rows, all of whose CTAs fit the GPU at once: one cooperative launch
  if (nchunks_all <= kLongMaxChunks && rows * nchunks_all <= (long long)long_per_sm() * sms) {
    if (!hist_ready && (e = cudaMemsetAsync(ws.hist, 0, ws.zero_bytes, stream)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nchunks_all, (unsigned)rows, 1);
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = sizeof(LongSmem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, topk_long_kernel, scores, T, N, q_pos0, k, ws, hist_ready ? 1 : 0, idx, err);
  }
  if (!hist_ready) {
    e = cudaMemsetAsync(ws.hist, 0, ws.zero_bytes, stream);
    if (e != cudaSuccess) return e;
    topk_hist_kernel<<<dim3((unsigned)rows, (unsigned)nchunks_all), kHistThreads, 0, stream>>>(scores, T, N, q_pos0,
                                                                                                ws.hist);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // float4 loads need 16-byte aligned rows
  const int vec = (N & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
  // the select kernel needs every chunk of the row to take a ticket, so it runs over all
  // chunks of N (chunks past the visible range count nothing)
  const size_t smem = sizeof(SelectSmem);
  static DeviceOnce once;
  if ((e = once.run([&] {
         return cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
       })) != cudaSuccess)
    return e;
  topk_select_kernel<<<dim3((unsigned)rows, (unsigned)nchunks_all), kSelThreads, smem, stream>>>(scores, T, N, q_pos0,
                                                                                                  k, ws, idx, vec, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  topk_compact_kernel<<<dim3((unsigned)rows, (unsigned)nchunks_all), kCmpThreads, 0, stream>>>(scores, T, N, q_pos0,
                                                                                                k, ws, idx, vec);
  return cudaGetLastError();
}

}  // namespace dsa
