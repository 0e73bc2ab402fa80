// indexer_tc.cu -- lightweight indexer score on the 5th-generation tensor cores.
//
// I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s])   ("GLM-5.2 1M architecture teardown",
// Cut 1: DSA -- index_n_heads 32, index_head_dim 128).
//
// For a tile of 128 cached keys and a group of QG queries the head dot products are one
// matrix product: D[key][(query, head)] = K[128 x 128] * Q[(QG*32) x 128]^T, M = 128,
// N = 32*QG, K = 128 (8 MMAs of K = 16).  QG = 1 for decode (the key stream is the whole
// cost; the tensor core is ~10% busy), QG = 8 for chunked prefill (a dense contraction).
//
// Warp roles (one CTA per SM, persistent over a contiguous range of (query group, key
// tile) items):
//   warp 0      TMA producer: 128x128 key tiles (bf16: two 64-column boxes; E4M3: one
//               128-column box; 128-byte swizzle) into a ring of shared-memory stages (in
//               decode under an L2 evict-first policy: each tile is read once); the query
//               group once per group change;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma into a ring of TMEM
//               accumulators (decode: 4 x 32 columns; prefill: 2 x 256) and commits to the
//               stage / accumulator barriers;
//   warps 2..9  epilogue, two warps per TMEM lane quarter (decode: the two take alternate
//               tiles, so two tiles are scored at once; prefill: each scores 4 of the 8
//               queries): each thread owns one key row of the accumulator (its warp's TMEM
//               lane quarter), loads the 32 head columns of a query, applies ReLU and the
//               head weights, sums, and stores the score (coalesced: a warp writes 32
//               consecutive keys).  In decode it can also count the first radix digit of
//               each score into a per-row histogram for the top-k select.
// Every mbarrier wait is bounded (see sm100.cuh); a timeout sets the device error word.
#include <cudaTypedefs.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

static __device__ int g_indexer_tc_error;

constexpr int kTileKeys = 128;
constexpr int kHalfBytesA = kTileKeys * 128;  // 128 rows x 128 bytes (64 bf16 or 128 E4M3) = 16 KB

// kF8: keys and queries in E4M3 (one 128-byte box per row, kind::f8f6f4 MMAs of K = 32);
// otherwise bf16 (two 64-column boxes per row, kind::f16 MMAs of K = 16)
template <int QG, bool kHist, bool kF8 = false>
struct TcCfg {
  // 8 epilogue warps, two per TMEM lane quarter: in decode the two take alternate tiles
  // (four accumulators, so the MMA runs up to four tiles ahead of the epilogue); in
  // prefill the two split the tile's 8 queries (two accumulators of 256 columns)
  static constexpr int kEpiWarps = 8;
  static constexpr int kAccBufs = QG == 1 ? 4 : 2;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kN = 32 * QG;                  // MMA N
  static constexpr int kHalves = kF8 ? 1 : 2;         // 128-byte column boxes per 128-wide row
  static constexpr int kStageBytesA = kHalves * kHalfBytesA;
  // decode: 96 KB of keys in flight per SM (three bf16 or six E4M3 stages).  Measured on
  // B200 over the 268 MB decode128k key stream on 148 SMs: 3 stages 46.0 us, 4 47.1, 5
  // 49.2, 6 50.5 -- more requests in flight than the HBM needs only slow it down (E4M3, 134
  // MB: 6 stages 30.7 us, 10 31.6).  Prefill: a ring of 4 (8 E4M3) beside the larger B.
  static constexpr int kStages = kF8 ? (QG == 1 ? 6 : 8) : (QG == 1 ? 3 : 4);
  static constexpr int kHalfBytesB = kN * 128;
  static constexpr int kBytesB = kHalves * kHalfBytesB;
  static constexpr int kTmemCols = kAccBufs * kN;  // 128 or 512: a power of two >= 32
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kStageBytesA;
  // two row histograms (a CTA spans <= 2 rows) of 16-bit counts, two bins per 32-bit word
  // (a CTA counts at most its item range: fewer than 2^16 keys at one CTA per SM)
  static constexpr int kOffHist = kOffB + kBytesB;
  static constexpr int kOffBar = kOffHist + (kHist ? 2 * kHistBins * 2 : 0);
  static constexpr int kNumBars = 2 * kStages + 2 * kAccBufs + 3;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffTmem + 16 + 1024;  // + alignment slack
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct Items {
  int B, T, N, G;  // G = query groups per sequence
  long long q_pos0;
  int QG;
  __device__ int tiles(int qg) const {
    const int t0 = (qg % G) * QG;
    const int tl = min(t0 + QG, T) - 1;
    const long long v = visible_count(N, q_pos0, tl);
    return (int)((v + kTileKeys - 1) / kTileKeys);
  }
};

// Walks the flattened (query group, key tile) items [begin, end).
struct Cursor {
  int qg, tile, left_in_qg;
  long long remaining;
  __device__ void start(const Items& it, long long begin, long long end) {
    remaining = end - begin;
    qg = 0;
    long long acc = 0;
    const int nqg = it.B * it.G;
    while (qg < nqg) {
      const int n = it.tiles(qg);
      if (acc + n > begin) break;
      acc += n;
      ++qg;
    }
    tile = (int)(begin - acc);
    left_in_qg = qg < nqg ? it.tiles(qg) - tile : 0;
  }
  __device__ bool valid() const { return remaining > 0; }
  __device__ void next(const Items& it) {
    --remaining;
    ++tile;
    if (--left_in_qg == 0 && remaining > 0) {
      do {
        ++qg;
        tile = 0;
        left_in_qg = it.tiles(qg);
      } while (left_in_qg == 0);
    }
  }
};

template <int QG, bool kHist, bool kF8>
__global__ void __launch_bounds__(TcCfg<QG, kHist, kF8>::kThreads, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                  const float* __restrict__ w, int B, int T, int N, long long q_pos0, long long total_items,
                  float* __restrict__ scores, uint32_t* __restrict__ hist, int* __restrict__ err) {
  using C = TcCfg<QG, kHist, kF8>;
  grid_dep_launch();  // the top-k may be scheduled as SMs free up; it waits for these scores
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase + C::kOffA;
  const uint32_t sB = sbase + C::kOffB;
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(smem + C::kOffHist);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + C::kAccBufs + b); };
  const uint32_t qfull_bar = bar0 + 8u * (2 * C::kStages + 2 * C::kAccBufs);
  const uint32_t qfree_bar = bar0 + 8u * (2 * C::kStages + 2 * C::kAccBufs + 1);
  const uint32_t done_bar = bar0 + 8u * (2 * C::kStages + 2 * C::kAccBufs + 2);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffTmem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  Items it{B, T, N, (T + QG - 1) / QG, q_pos0, QG};
  const long long per = total_items / gridDim.x, extra = total_items % gridDim.x;
  const long long begin = blockIdx.x * per + min((long long)blockIdx.x, extra);
  const long long end = begin + per + (blockIdx.x < extra ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), QG == 1 ? 32 * C::kEpiWarps / 2 : 32 * C::kEpiWarps);  // decode: one warp group per tile
    }
    mbar_init(qfull_bar, 1);
    mbar_init(qfree_bar, 1);
    mbar_init(done_bar, 1);
    fence_mbar_init();
    tma_prefetch(&kmap);
    tma_prefetch(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), C::kTmemCols);
    tmem_relinquish();
  }
  if (kHist)
    for (int i = threadIdx.x; i < kHistBins; i += C::kThreads) s_hist[i] = 0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      Cursor cur;
      cur.start(it, begin, end);
      const uint64_t key_policy = l2_evict_first_policy();
      int stage = 0;
      uint32_t phase = 0, qfree_phase = 0;
      int cur_qg = -1;
      long long issued = 0;
      bool ok = true, q_pending = false;
      uint32_t q_parity = 0;
      while (cur.valid() && ok) {
        if (cur.qg != cur_qg) {
          if (cur_qg >= 0) {
            ok = mbar_wait(qfree_bar, qfree_phase, err, 1);
            qfree_phase ^= 1;
            if (!ok) break;
          }
          const int b = cur.qg / it.G, t0 = (cur.qg % it.G) * QG;
          mbar_arrive_expect_tx(qfull_bar, C::kBytesB);
          for (int hh = 0; hh < C::kHalves; ++hh) tma_load_3d(sB + hh * C::kHalfBytesB, &qmap, qfull_bar, 64 * hh, t0 * 32, b);
          q_pending = true;
          q_parity = (cur_qg >= 0) ? (q_parity ^ 1) : 0;
          cur_qg = cur.qg;
        }
        ok = mbar_wait(empty_bar(stage), phase ^ 1, err, 2);
        if (!ok) break;
        const int b = cur.qg / it.G;
        const uint32_t dst = sA + stage * C::kStageBytesA;
        mbar_arrive_expect_tx(full_bar(stage), C::kStageBytesA);
        for (int hh = 0; hh < C::kHalves; ++hh) {
          if (QG == 1)  // decode: every key tile is read once per launch
            tma_load_3d_hint(dst + hh * kHalfBytesA, &kmap, full_bar(stage), 64 * hh, cur.tile * kTileKeys, b,
                             key_policy);
          else          // prefill: every query group re-reads the keys, which stay in L2
            tma_load_3d(dst + hh * kHalfBytesA, &kmap, full_bar(stage), 64 * hh, cur.tile * kTileKeys, b);
        }
        ++issued;
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1;
        }
        cur.next(it);
      }
      if (!ok) {
        // let the loads already in flight land before the CTA exits
        for (long long j = issued > C::kStages ? issued - C::kStages : 0; j < issued; ++j)
          mbar_wait_drain(full_bar((int)(j % C::kStages)), (uint32_t)((j / C::kStages) & 1));
        if (q_pending) mbar_wait_drain(qfull_bar, q_parity);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // the whole warp runs the loop (descriptor arithmetic stays warp-uniform); one
    // elected lane issues the tensor-core instructions
    const bool leader = elect_one();
    constexpr uint32_t idesc = kF8 ? idesc_e4m3_f32(kTileKeys, C::kN) : idesc_bf16_f32(kTileKeys, C::kN);
    Cursor cur;
    cur.start(it, begin, end);
    int stage = 0;
    uint32_t phase = 0, qfull_phase = 0;
    long long acc = 0;
    int cur_qg = -1;
    bool ok = true;
    const uint64_t bd0 = sdesc_kmajor_sw128(sB);
    while (cur.valid() && ok) {
      if (cur.qg != cur_qg) {
        if (cur_qg >= 0 && leader) mma_commit(qfree_bar);
        __syncwarp();
        ok = mbar_wait(qfull_bar, qfull_phase, err, 4);
        qfull_phase ^= 1;
        if (!ok) break;
        cur_qg = cur.qg;
      }
      const int buf = (int)(acc % C::kAccBufs);
      const uint32_t use = (uint32_t)(acc / C::kAccBufs);
      ok = mbar_wait(tempty_bar(buf), (use & 1) ^ 1, err, 5);
      if (!ok) break;
      tc_fence_after();
      ok = mbar_wait(full_bar(stage), phase, err, 6);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = tmem_base + buf * C::kN;
      const uint64_t ad0 = sdesc_kmajor_sw128(sA + stage * C::kStageBytesA);
      if (leader) {
        // each MMA takes 32 bytes of K: 16 bf16 or 32 E4M3 values
#pragma unroll
        for (int kh = 0; kh < C::kHalves; ++kh)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t a = ad0 + (uint64_t)((kh * kHalfBytesA + ks * 32) >> 4);
            const uint64_t bb = bd0 + (uint64_t)((kh * C::kHalfBytesB + ks * 32) >> 4);
            if (kF8)
              mma_e4m3(d, a, bb, idesc, (kh | ks) != 0);
            else
              mma_bf16(d, a, bb, idesc, (kh | ks) != 0);
          }
        mma_commit(empty_bar(stage));
        mma_commit(tfull_bar(buf));
      }
      __syncwarp();
      ++acc;
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1;
      }
      cur.next(it);
    }
    // every MMA issued so far has finished before TMEM is released
    if (leader) {
      mma_commit(done_bar);
      if (!mbar_wait_drain(done_bar, 0)) atomicCAS(err, 0, 7);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const int qhalf = (warp - 2) >> 2;  // prefill: which half of the 8 queries this warp scores;
                                        // decode: which of two alternate tiles it scores
    const int row_in_tile = 32 * quarter + lane;
    Cursor cur;
    cur.start(it, begin, end);
    const int b_first = cur.valid() ? cur.qg / it.G : 0;
    long long acc = 0;
    int cur_qg = -1;
    float wr[32];  // head weights of the current query (decode)
    bool ok = true;
    while (cur.valid() && ok) {
      if (QG == 1 && (int)(acc & 1) != qhalf) {  // the other warp group's tile
        ++acc;
        cur.next(it);
        continue;
      }
      const int b = cur.qg / it.G, t0 = (cur.qg % it.G) * QG;
      if (QG == 1 && cur.qg != cur_qg) {
        const float* wq = w + ((size_t)b * T + t0) * 32;
#pragma unroll
        for (int h = 0; h < 32; ++h) wr[h] = __ldg(&wq[h]);
        cur_qg = cur.qg;
      }
      const int buf = (int)(acc % C::kAccBufs);
      const uint32_t use = (uint32_t)(acc / C::kAccBufs);
      ok = mbar_wait(tfull_bar(buf), use & 1, err, 8);
      if (!ok) break;
      tc_fence_after();
      const long long key = (long long)cur.tile * kTileKeys + row_in_tile;
      int slot = kHist ? b - b_first : 0;
      if (slot > 1) {  // cannot happen for B <= 148 (checked by the host); never write past the slots
        atomicCAS(err, 0, 9);
        slot = 1;
      }
      uint32_t* hslot = s_hist + slot * (kHistBins / 2);
      (void)hslot;
      if (QG == 1) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(32 * quarter) << 16) + buf * C::kN, r);
        tmem_ld_wait();
        float sc = 0.f;
#pragma unroll
        for (int h = 0; h < 32; ++h) sc = fmaf(wr[h], fmaxf(__uint_as_float(r[h]), 0.f), sc);
        if (t0 < T && key < visible_count(N, q_pos0, t0)) {
          scores[((size_t)b * T + t0) * N + key] = sc;
          if (kHist) {
            const uint32_t bin = order_key(sc) >> kHistShift;
            atomicAdd(&hslot[bin >> 1], 1u << (16 * (bin & 1)));
          }
        }
      } else {
        // two queries (64 columns) per TMEM round trip; head weights as 16-byte loads
#pragma unroll 1
        for (int g = 4 * qhalf; g < 4 * qhalf + 4; g += 2) {
          uint32_t r0[32], r1[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * quarter) << 16) + buf * C::kN + 32 * g, r0);
          tmem_ld32(tmem_base + ((uint32_t)(32 * quarter) << 16) + buf * C::kN + 32 * g + 32, r1);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int t = t0 + g + u;
            const float4* wq = reinterpret_cast<const float4*>(w + ((size_t)b * T + (t < T ? t : T - 1)) * 32);
            float sc = 0.f;
#pragma unroll
            for (int h4 = 0; h4 < 8; ++h4) {
              const float4 w4 = __ldg(&wq[h4]);
              const uint32_t* rr = u ? r1 : r0;
              sc = fmaf(w4.x, fmaxf(__uint_as_float(rr[4 * h4 + 0]), 0.f), sc);
              sc = fmaf(w4.y, fmaxf(__uint_as_float(rr[4 * h4 + 1]), 0.f), sc);
              sc = fmaf(w4.z, fmaxf(__uint_as_float(rr[4 * h4 + 2]), 0.f), sc);
              sc = fmaf(w4.w, fmaxf(__uint_as_float(rr[4 * h4 + 3]), 0.f), sc);
            }
            if (t < T && key < visible_count(N, q_pos0, t)) scores[((size_t)b * T + t) * N + key] = sc;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(buf));
      ++acc;
      cur.next(it);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (kHist && begin < end) {
    // fold this CTA's counts into the per-row histograms (decode: row = sequence)
    Cursor cur;
    cur.start(it, begin, end);
    const int b_first = cur.qg / it.G;
    for (int i = threadIdx.x; i < kHistBins; i += C::kThreads) {  // word i: bins 2i, 2i + 1 of a slot
      const uint32_t c = s_hist[i];
      const int row = b_first + i / (kHistBins / 2);
      const int bin = 2 * (i % (kHistBins / 2));
      if (c && row < B) {
        if (c & 0xFFFFu) atomicAdd(&hist[(size_t)row * kHistBins + bin], c & 0xFFFFu);
        if (c >> 16) atomicAdd(&hist[(size_t)row * kHistBins + bin + 1], c >> 16);
      }
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D map over [d2][d1][128 values] with a box of one 128-byte column block x rows x 1 and
// the 128-byte swizzle: bf16 (64-value blocks) or E4M3 bytes (128-value blocks)
bool make_map(CUtensorMap* map, const void* base, long long d1, long long d2, int rows, bool f8) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int esz = f8 ? 1 : 2;
  cuuint64_t dims[3] = {128, (cuuint64_t)d1, (cuuint64_t)d2};
  cuuint64_t strides[2] = {(cuuint64_t)128 * esz, (cuuint64_t)d1 * 128 * esz};
  cuuint32_t box[3] = {(cuuint32_t)(128 / esz), (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

SymbolAddress g_err_addr;

template <int QG, bool kHist, bool kF8>
cudaError_t launch_tc(const void* q, const float* w, const void* k, int B, int T, int N, long long q_pos0,
                      float* scores, uint32_t* hist, int sm_budget, cudaStream_t stream) {
  using C = TcCfg<QG, kHist, kF8>;
  CUtensorMap kmap, qmap;
  if (!make_map(&kmap, k, N, B, kTileKeys, kF8) || !make_map(&qmap, q, (long long)T * 32, B, C::kN, kF8))
    return cudaErrorInvalidValue;
  int* err = nullptr;
  cudaError_t e = g_err_addr.get(g_indexer_tc_error, &err);
  if (e != cudaSuccess) return e;
  static DeviceOnce once;
  if ((e = once.run([] {
         return cudaFuncSetAttribute(indexer_tc_kernel<QG, kHist, kF8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::kSmem);
       })) != cudaSuccess)
    return e;
  // items = sum over query groups of the key tiles they see
  const int G = (T + QG - 1) / QG;
  long long total = 0;
  for (int j = 0; j < B * G; ++j) {
    const int t0 = (j % G) * QG;
    const int tl = (t0 + QG < T ? t0 + QG : T) - 1;
    const long long v = visible_count(N, q_pos0, tl);
    total += (v + kTileKeys - 1) / kTileKeys;
  }
  // persistent: one CTA per SM of the budget (all SMs by default)
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  if (total == 0) return cudaSuccess;
  const int cap = sm_budget > 0 && sm_budget < sms ? sm_budget : sms;
  const int grid = (int)(total < cap ? total : cap);
  indexer_tc_kernel<QG, kHist, kF8><<<grid, C::kThreads, C::kSmem, stream>>>(kmap, qmap, w, B, T, N, q_pos0, total, scores,
                                                                       hist, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_score_tc(const void* q, const float* w, const void* k, int B, int T, int N, long long q_pos0,
                                  float* scores, uint32_t* hist, int sm_budget, bool f8, cudaStream_t stream) {
  // the fused histogram keeps two row slots per CTA: with contiguous item ranges over at
  // most one CTA per SM of the budget, a range spans at most two sequences when B is no
  // more than the CTAs
  const int sms = device_sm_count();
  const int cap = sm_budget > 0 && sm_budget < sms ? sm_budget : sms;
  if (hist && (T != 1 || B > cap)) return cudaErrorNotSupported;
  if (f8) {
    if (T == 1)
      return hist ? launch_tc<1, true, true>(q, w, k, B, T, N, q_pos0, scores, hist, sm_budget, stream)
                  : launch_tc<1, false, true>(q, w, k, B, T, N, q_pos0, scores, nullptr, sm_budget, stream);
    return launch_tc<8, false, true>(q, w, k, B, T, N, q_pos0, scores, nullptr, sm_budget, stream);
  }
  if (T == 1)
    return hist ? launch_tc<1, true, false>(q, w, k, B, T, N, q_pos0, scores, hist, sm_budget, stream)
                : launch_tc<1, false, false>(q, w, k, B, T, N, q_pos0, scores, nullptr, sm_budget, stream);
  return launch_tc<8, false, false>(q, w, k, B, T, N, q_pos0, scores, nullptr, sm_budget, stream);
}

cudaError_t indexer_error_word(int** p) { return g_err_addr.get(g_indexer_tc_error, p); }

}  // namespace dsa
