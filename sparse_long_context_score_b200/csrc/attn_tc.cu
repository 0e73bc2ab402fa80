// attn_tc.cu -- sparse MLA attention on the 5th-generation tensor cores.
//
// "GLM-5.2 1M architecture teardown", Cut 1: DSA (full attention over only the 2048 keys
// the indexer kept) and Cut 3: MLA (one compressed 576-wide row per token, shared by all
// heads; in the absorbed form the logit of head h is scale * q[h] . c[j] and the value is
// the row's first 512 entries).
//
// One CTA per (query row, layer, key split); tiles of 32 selected rows.
//   S   = Q K^T   M = 64 heads, N = 32 keys, K = 576    (36 MMAs; TMEM lane = head)
//   O^T = V^T P^T M = 4 x 128 value dims, N = 64 heads, K = 32 keys (8 MMAs)
// Because S has one head per TMEM lane, each softmax thread owns one head: its running
// max and sum stay in registers and need no cross-thread reduction.  The running max is
// only moved (and O rescaled in TMEM) when a tile's max exceeds it by more than 2^8, so
// rescaling is rare; exponentials may then exceed 1 by at most 2^8, which f32 and bf16
// carry without loss of relative precision.
//
// Warp roles (416 threads):
//   warps 0..7  gather: the selected rows as 16-byte cp.async chunks written straight into
//               the 128-byte-swizzled tensor-core layout; warps 2s, 2s+1 own stage s
//               (16 rows each) and tiles s, s+4, ... (their row indices loaded into
//               registers up front), wait for their own copies, fence them to the async
//               proxy and arrive on the stage barrier, so four tiles are in flight and each
//               is published as soon as it lands (one TMA load brings the 64 query rows).
//               Random 1152-byte rows are too small for TMA: measured on B200 with the same
//               bytes in flight, a 128-byte box per row reached 0.57 TB/s, 4-row gather
//               boxes 1.6 TB/s, one bulk copy per row 2.8 TB/s, 16-byte cp.async 4.9 TB/s.
//   warp 8      TMEM allocation; one elected lane issues S(i) once tile i has landed and
//               O += P(j) V(j) once P(j) is published, whichever is ready (PV first), so
//               the softmax of one tile overlaps the next tile's logits and a stage is
//               released as soon as its PV completes;
//   warps 9..12 softmax (threads on lanes 0..15 of each warp own a head), P as bf16 in
//               shared memory.
// The key splits of one (row, layer) run as one thread-block cluster and are reduced on
// chip: each split stages its unnormalised O in its shared memory, and split r sums slice r
// of the [H][512] output over the cluster's shared memories with the normaliser shares.
// (A global-memory merge by the last split to finish -- 16 MB of partials written and
// read back at the end of the 32-unit decode batch -- made the kernel's tail longer than
// its whole main loop.)  The launch waits for the preceding kernel (programmatic dependent
// launch) only where it reads that kernel's results.
// All mbarrier waits are bounded (sm100.cuh).
#include <cudaTypedefs.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

static __device__ int g_attn_tc_error;

constexpr int kKeys = 32;                        // selected rows per tile
constexpr int kStages = 4;
constexpr int kBlocks = kDqk / 64;               // nine 64-wide column blocks of a row
constexpr int kQBlockBytes = 64 * 128;           // 64 heads x 64 bf16
constexpr int kBlockBytes = kKeys * 128;         // 32 rows x 64 bf16
constexpr int kQBytes = kBlocks * kQBlockBytes;  // 73728
constexpr int kStageBytes = kBlocks * kBlockBytes;  // 36864
constexpr int kPBytes = 64 * kKeys * 2;          // one P buffer: 64 heads x 64-byte rows (4 KB)
constexpr int kProducerWarps = 8;                // two warps per stage, 16 rows each
constexpr int kMmaWarp = kProducerWarps;
constexpr int kSoftmaxWarp0 = kProducerWarps + 1;
constexpr int kThreadsA = (kProducerWarps + 5) * 32;  // 416
static_assert(kSoftmaxWarp0 + 4 == kThreadsA / 32, "four softmax warps, one per TMEM lane quarter");
constexpr float kRescaleLog2 = 8.f;
// rounds of kStages tiles in the largest split (k <= kMaxTopk keys): the row indices a
// gather lane holds in registers
constexpr int kRounds = (kMaxTopk + kKeys * kStages - 1) / (kKeys * kStages);
constexpr int kMaxSplits = 8;                    // key splits of one (row, layer): one portable cluster
// float4 elements of the [64][512] output slice a thread sums when there are >= 2 splits
constexpr int kPullPerThread = (64 * 128 / 2 + kThreadsA - 1) / kThreadsA;

constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQBytes;
constexpr int kOffP = kOffStage + kStages * kStageBytes;
constexpr int kOffAlpha = kOffP + 2 * kPBytes;   // [2][64] f32 (tile parity)
constexpr int kOffL = kOffAlpha + 2 * 64 * 4;    // [64] f32
constexpr int kOffM = kOffL + 64 * 4;            // [64] f32
constexpr int kOffMask = kOffM + 64 * 4;         // [kStages][2] u16 (one half per producer warp)
constexpr int kOffVote = kOffMask + kStages * 4;  // [2] u32 (tile parity): one byte per softmax warp
// after the main loop the P buffers hold [kMaxSplits][64] f32: each split's share of the normaliser
constexpr int kOffCoef = kOffP;
static_assert(kMaxSplits * 64 * 4 <= 2 * kPBytes, "coefficients fit the P buffers");
constexpr int kNumBars = 2 * kStages + 11;
constexpr int kOffBar = kOffVote + 16;
constexpr int kOffTmem = kOffBar + kNumBars * 8;
constexpr int kSmemA = kOffTmem + 16 + 1024;
static_assert(kSmemA <= 232448, "shared memory budget");

constexpr int kTmemO = 0;      // O^T: 4 blocks x 64 columns, all 128 lanes
constexpr int kTmemS = 256;    // S: 2 buffers x 32 columns, lanes 0..15 of each quarter
constexpr int kTmemCols = 512;

struct AttnMaps {
  CUtensorMap q[kMaxLayers];
};

__global__ void __launch_bounds__(kThreadsA, 1)
attn_tc_kernel(const __grid_constant__ AttnMaps maps, AttnLayers layers, const int32_t* __restrict__ idx, int T, int N,
               int H, int k, int chunk, float scale_log2, int q_early, int* __restrict__ err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + kOffQ;
  const uint32_t sStage = sbase + kOffStage;
  const uint32_t sP = sbase + kOffP;
  float* s_alpha = reinterpret_cast<float*>(smem + kOffAlpha);
  float* s_l = reinterpret_cast<float*>(smem + kOffL);
  float* s_m = reinterpret_cast<float*>(smem + kOffM);
  uint16_t* s_mask = reinterpret_cast<uint16_t*>(smem + kOffMask);
  float* s_coef = reinterpret_cast<float*>(smem + kOffCoef);
  uint32_t* s_vote = reinterpret_cast<uint32_t*>(smem + kOffVote);
  const uint32_t bar0 = sbase + kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto sfull_bar = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
  auto sfree_bar = [&](int s) { return bar0 + 8u * (2 * kStages + 2 + s); };
  auto pfull_bar = [&](int pb) { return bar0 + 8u * (2 * kStages + 4 + pb); };
  auto pfree_bar = [&](int pb) { return bar0 + 8u * (2 * kStages + 6 + pb); };
  const uint32_t ofinal_bar = bar0 + 8u * (2 * kStages + 8);
  const uint32_t qfull_bar = bar0 + 8u * (2 * kStages + 9);
  const uint32_t grp_bar = bar0 + 8u * (2 * kStages + 10);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffTmem);

  const int split = blockIdx.x, row = blockIdx.y, layer = blockIdx.z;
  const int nsplit = gridDim.x;
  const int b = row / T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = split * chunk;
  const int nkeys = max(min(j0 + chunk, k) - j0, 0);
  const int ntiles = (nkeys + kKeys - 1) / kKeys;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 64);
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(sfull_bar(s), 1);
      mbar_init(sfree_bar(s), 128);
    }
    for (int pb = 0; pb < 2; ++pb) {
      mbar_init(pfull_bar(pb), 128);
      mbar_init(pfree_bar(pb), 1);
    }
    mbar_init(ofinal_bar, 1);
    mbar_init(qfull_bar, 1);
    mbar_init(grp_bar, 128);
    fence_mbar_init();
    tma_prefetch(&maps.q[layer]);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(s_tmem), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp < kProducerWarps) {
    // ------------------------------------------------------------------ gather
    // warps 2s and 2s+1 own stage s and fill rows [0,16) and [16,32) of tiles s, s+4, ...;
    // each waits for its own copies, fences them to the async proxy and arrives, so
    // four tiles are in flight and each is published as soon as it lands
    const int ps = warp >> 1, half = warp & 1;
    if (warp == 0 && lane == 0) {
      // the queries may be read before the preceding kernel completes only when the caller
      // knows that kernel does not write them (the top-k of the same group)
      if (!q_early) grid_dep_wait();
      const CUtensorMap* qm = &maps.q[layer];
      mbar_arrive_expect_tx(qfull_bar, kQBytes);
      for (int kb = 0; kb < kBlocks; ++kb) tma_load_2d(sQ + kb * kQBlockBytes, qm, qfull_bar, 64 * kb, row * H);
    }
    // the index list comes from the preceding kernel.  (Every other warp waits on the
    // gather through the pipeline barriers, and the output is written only after the
    // cluster barrier that follows this wait.)
    grid_dep_wait();
    const int32_t* sel = idx + (size_t)row * k + j0;
    const uint16_t* kvb = layers.kv[layer] + (size_t)b * N * kDqk;
    const uint32_t st = sStage + ps * kStageBytes;
    // this lane copies 16-byte chunks lane, lane+32, lane+64 (< 72) of every row: the
    // column block and in-row offset of each are constants
    const int c0 = lane, c1 = lane + 32, c2 = lane + 64;
    const uint32_t kb0 = (c0 >> 3) * kBlockBytes, kb1 = (c1 >> 3) * kBlockBytes, kb2 = (c2 >> 3) * kBlockBytes;
    // the row indices of all this warp's tiles (ps, ps + kStages, ...), loaded at once before
    // the first tile: no dependent index load sits in front of a tile's copies
    int pre[kRounds];
#pragma unroll
    for (int j = 0; j < kRounds; ++j) {
      const int key = (ps + kStages * j) * kKeys + 16 * half + (lane & 15);
      pre[j] = key < nkeys ? __ldg(&sel[key]) : -1;
    }
    for (int i = ps; i < ntiles; i += kStages) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(empty_bar(ps), ((i / kStages) & 1) ^ 1, err, 21);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      const int v = pre[0];
#pragma unroll
      for (int j = 0; j + 1 < kRounds; ++j) pre[j] = pre[j + 1];
      const bool valid = v >= 0 && v < N;
      const int my_row = valid ? v : 0;
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, valid) & 0xFFFFu;
      if (lane == 0) s_mask[2 * ps + half] = (uint16_t)m;
#pragma unroll 4
      for (int rr = 0; rr < 16; ++rr) {
        const int r = 16 * half + rr;
        const uint16_t* src = kvb + (size_t)__shfl_sync(0xFFFFFFFFu, my_row, rr) * kDqk;
        const uint32_t rbase = st + r * 128;
        const int x = r & 7;
        cp_async_16(rbase + kb0 + (((c0 & 7) ^ x) << 4), src + c0 * 8, 16);
        cp_async_16(rbase + kb1 + (((c1 & 7) ^ x) << 4), src + c1 * 8, 16);
        if (c2 < kDqk / 8) cp_async_16(rbase + kb2 + (((c2 & 7) ^ x) << 4), src + c2 * 8, 16);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async();  // the copies are visible to the tensor core (async proxy)
      mbar_arrive(full_bar(ps));
    }
    if (warp == 0 && lane == 0) mbar_wait_drain(qfull_bar, 0);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // the whole warp runs the loop (descriptor arithmetic stays warp-uniform); one
    // elected lane issues the tensor-core instructions
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16_f32(64, kKeys);              // Q (K-major) x K (K-major)
    constexpr uint32_t idPV = idesc_bf16_f32(128, 64, true, false);  // V^T (M-major) x P (K-major)
    bool ok = mbar_wait(qfull_bar, 0, err, 22);
    const uint64_t dq = sdesc_kmajor_sw128(sQ);
    const int leader_lane = __ffs(__ballot_sync(0xFFFFFFFFu, leader)) - 1;
    // S(i) needs tile i in its stage and a free S buffer; PV(j) needs P(j).  Each is issued
    // as soon as it can be, PV first: a stage is released by its PV, and waiting for the
    // next tile's data before issuing the previous tile's PV would keep one of the four
    // stages from gathering.  The leader polls; the warp follows its decisions.
    int is = 0, ipv = 0;
    long long idle_since = clock64();
    int spins = 0;
    while (ok && ipv < ntiles) {
      bool pv_ready = false, s_ready = false;
      if (leader) {
        pv_ready = ipv < is && mbar_try_wait(pfull_bar(ipv & 1), (ipv >> 1) & 1);
        s_ready = is < ntiles && mbar_try_wait(full_bar(is % kStages), (is / kStages) & 1) &&
                  mbar_try_wait(sfree_bar(is & 1), ((is >> 1) & 1) ^ 1);
      }
      pv_ready = __shfl_sync(0xFFFFFFFFu, pv_ready, leader_lane);
      s_ready = __shfl_sync(0xFFFFFFFFu, s_ready, leader_lane);
      if (pv_ready) {
        const int jt = ipv, sj = jt % kStages, pb = jt & 1;
        tc_fence_after();
        const uint64_t da = sdesc_mnmajor_sw128(sStage + sj * kStageBytes, kBlockBytes, 1024);
        const uint64_t dp = sdesc_kmajor_sw64(sP + pb * kPBytes);
        const uint32_t first = jt > 0 ? 1u : 0u;
        if (leader) {
#pragma unroll
          for (int mb = 0; mb < 4; ++mb)
#pragma unroll
            for (int ks = 0; ks < kKeys / 16; ++ks)
              mma_bf16(tmem + kTmemO + 64 * mb, da + (uint64_t)(((2 * mb) * kBlockBytes + ks * 16 * 128) >> 4),
                       dp + (uint64_t)((ks * 32) >> 4), idPV, first | (ks > 0 ? 1u : 0u));
          mma_commit(pfree_bar(pb));
          mma_commit(empty_bar(sj));
        }
        __syncwarp();
        ++ipv;
      }
      if (s_ready) {
        const int i = is, st = i % kStages, sb = i & 1;
        tc_fence_after();
        const uint32_t dS = tmem + kTmemS + kKeys * sb;
        // descriptors differ only in their start address: compile-time offsets from a base
        const uint64_t dk = sdesc_kmajor_sw128(sStage + st * kStageBytes);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 4 * kBlocks; ++kk)
            mma_bf16(dS, dq + (uint64_t)((((kk >> 2) * kQBlockBytes) + (kk & 3) * 32) >> 4),
                     dk + (uint64_t)((((kk >> 2) * kBlockBytes) + (kk & 3) * 32) >> 4), idS, kk > 0);
          mma_commit(sfull_bar(sb));
        }
        __syncwarp();
        ++is;
      }
      if (pv_ready || s_ready) {
        idle_since = clock64();
        spins = 0;
      } else if (++spins == 64) {
        // bounded like every other wait: give up after kWaitLimitCycles without progress,
        // or when another thread has already failed
        spins = 0;
        const bool late = __any_sync(0xFFFFFFFFu, clock64() - idle_since > kWaitLimitCycles);
        const bool failed = __any_sync(0xFFFFFFFFu, *reinterpret_cast<volatile int*>(err) != 0);
        if (late && leader) atomicCAS(err, 0, 23);
        ok = !(late || failed);
      }
    }
    if (leader) {
      mma_commit(ofinal_bar);
      if (!mbar_wait_drain(ofinal_bar, 0)) atomicCAS(err, 0, 26);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + read-out
    const int quarter = warp & 3;
    const bool owner = lane < 16;                 // this thread's TMEM lane holds a head of S
    const int head = 16 * quarter + (lane & 15);
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    float m_used = -INFINITY, l_run = 0.f;
    uint32_t grp_phase = 0;
    bool ok = true;
    for (int i = 0; i < ntiles && ok; ++i) {
      const int sb = i & 1, s = i % kStages;
      ok = mbar_wait(sfull_bar(sb), (i >> 1) & 1, err, 27);
      if (!ok) break;
      tc_fence_after();
      uint32_t r[kKeys];
      tmem_ld32(tmem + lane_addr + kTmemS + kKeys * sb, r);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(sfree_bar(sb));
      ok = mbar_wait(full_bar(s), (i / kStages) & 1, err, 28);  // orders the gather's mask write
      if (!ok) break;
      const uint32_t mask = (uint32_t)s_mask[2 * s] | ((uint32_t)s_mask[2 * s + 1] << 16);
      float* alpha = s_alpha + 64 * (i & 1);
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < kKeys; ++j) {
        const float z = ((mask >> j) & 1u) ? __uint_as_float(r[j]) * scale_log2 : -INFINITY;
        r[j] = __float_as_uint(z);
        mt = fmaxf(mt, z);
      }
      float a = 1.f;
      if (mt > m_used + kRescaleLog2 || (m_used == -INFINITY && mt > -INFINITY)) {
        a = m_used == -INFINITY ? 0.f : exp2f(m_used - mt);
        m_used = mt;
        l_run *= a;
      }
      if (owner) alpha[head] = a;
      // one vote per warp: does any of its heads need O rescaled?  (64 shared loads of
      // the factors per thread, serialised, cost about a microsecond per tile)
      const uint32_t vote = __ballot_sync(0xFFFFFFFFu, owner && head < H && a != 1.f);
      if (lane == 0) reinterpret_cast<volatile unsigned char*>(s_vote + (i & 1))[quarter] = vote != 0u ? 1 : 0;
      // every head's factor is known before O is touched
      mbar_arrive(grp_bar);
      ok = mbar_wait(grp_bar, grp_phase, err, 29);
      grp_phase ^= 1;
      if (!ok) break;
      const bool any = *reinterpret_cast<volatile uint32_t*>(s_vote + (i & 1)) != 0u;
      if (i > 0 && any) {
        // O^T is rescaled only once the previous tile's PV has finished with it
        ok = mbar_wait(pfree_bar((i - 1) & 1), ((i - 1) >> 1) & 1, err, 30);
        if (!ok) break;
        tc_fence_after();
        // rescale O^T: this thread's lane is one value dim, its columns the heads
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb)
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            uint32_t o[32];
            const uint32_t ta = tmem + lane_addr + kTmemO + 64 * mb + 32 * half;
            tmem_ld32(ta, o);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha[32 * half + c]);
            tmem_st32(ta, o);
          }
        tmem_st_wait();
      }
      if (i > 1) {
        // P buffer i&1 was last read by PV(i-2)
        ok = mbar_wait(pfree_bar(i & 1), ((i >> 1) & 1) ^ 1, err, 34);
        if (!ok) break;
      }
      if (owner) {
        const float mu = m_used == -INFINITY ? 0.f : m_used;
        float ls = 0.f;
        uint32_t packed[kKeys / 2];
#pragma unroll
        for (int j = 0; j < kKeys; j += 2) {
          const float p0 = exp2f(__uint_as_float(r[j]) - mu);
          const float p1 = exp2f(__uint_as_float(r[j + 1]) - mu);
          ls += p0 + p1;
          packed[j / 2] = pack_bf16x2(p0, p1);
        }
        l_run += ls;
        // P row `head` of buffer i&1: 32 keys = 64 bytes, K-major with the 64-byte swizzle
        unsigned char* prow = smem + kOffP + (i & 1) * kPBytes + head * 64;
#pragma unroll
        for (int c = 0; c < kKeys / 8; ++c)
          *reinterpret_cast<uint4*>(prow + ((c ^ ((head >> 1) & 3)) << 4)) =
              make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
        fence_proxy_async();
      }
      tc_fence_before();
      mbar_arrive(pfull_bar(i & 1));
    }
    if (owner) {
      s_l[head] = l_run;
      s_m[head] = m_used;
    }
  }

  // ------------------------------------------------------------------ split reduction
  // The splits of one (row, layer) form a cluster.  Each split publishes its running max
  // and sum per head and stages its unnormalised O in its own shared memory, in the
  // output's [head][512] layout; split r then owns slice r of that block and sums it over
  // the cluster through distributed shared memory,
  //   out[h] = sum_s c_s[h] O_s[h],  c_s[h] = 2^(m_s[h] - M[h]) / sum_r 2^(m_r[h] - M[h]) l_r[h],
  // M[h] = max_r m_r[h], writes the sum back over its own slice (no peer reads that
  // slice) and stores it with one bulk copy.  Nothing but the result goes through global
  // memory.  Every thread passes the three cluster barriers on every path (a failed wait
  // above only skips work), so none of them can be left waiting.
  tc_fence_before();
  cluster_sync();  // #1: (m, l) of every split published; this CTA's MMAs have completed
  tc_fence_after();
  if (threadIdx.x < 64) {
    const int h = threadIdx.x;
    float mr[kMaxSplits], lr[kMaxSplits];
    float M = -INFINITY;
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp) {
      mr[sp] = sp < nsplit ? ld_cluster_f32(cluster_map(smem_u32(s_m + h), sp)) : -INFINITY;
      lr[sp] = sp < nsplit ? ld_cluster_f32(cluster_map(smem_u32(s_l + h), sp)) : 0.f;
      M = fmaxf(M, mr[sp]);
    }
    float den = 0.f;
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp) {
      mr[sp] = mr[sp] == -INFINITY ? 0.f : exp2f(mr[sp] - M);
      den += mr[sp] * lr[sp];
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp)
      if (sp < nsplit) s_coef[sp * 64 + h] = mr[sp] * inv;
  }
  // O^T (TMEM lane = value dim, column = head) -> staging [64 heads][512] f32 over the idle
  // Q and stage buffers.  Twelve warps, three per TMEM lane quarter, take the eight
  // 32-column chunks (value block mb, head half) two loads at a time.  A single split
  // (no cluster peers) applies its normaliser here and stores the staging directly.
  float* stg = reinterpret_cast<float*>(smem + kOffQ);
  if (nsplit == 1) __syncthreads();  // s_coef
  if (warp != kMmaWarp) {
    const int quarter = warp & 3;
    const int j = warp < kProducerWarps ? warp >> 2 : 2;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16) + kTmemO;
    for (int c = j; c < 8; c += 6) {
      const bool two = c + 3 < 8;
      uint32_t o0[32], o1[32];
      if (ntiles > 0) {
        tmem_ld32(lane_base + 64 * (c >> 1) + 32 * (c & 1), o0);
        if (two) tmem_ld32(lane_base + 64 * ((c + 3) >> 1) + 32 * ((c + 3) & 1), o1);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) o0[c2] = o1[c2] = 0u;
      }
      if (nsplit == 1) {
        // the normalisers of these columns' heads, in registers before the stores
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 v0 = reinterpret_cast<const float4*>(s_coef + 32 * (c & 1))[c4];
          o0[4 * c4] = __float_as_uint(__uint_as_float(o0[4 * c4]) * v0.x);
          o0[4 * c4 + 1] = __float_as_uint(__uint_as_float(o0[4 * c4 + 1]) * v0.y);
          o0[4 * c4 + 2] = __float_as_uint(__uint_as_float(o0[4 * c4 + 2]) * v0.z);
          o0[4 * c4 + 3] = __float_as_uint(__uint_as_float(o0[4 * c4 + 3]) * v0.w);
          const float4 v1 = reinterpret_cast<const float4*>(s_coef + 32 * ((c + 3) & 1))[c4];
          o1[4 * c4] = __float_as_uint(__uint_as_float(o1[4 * c4]) * v1.x);
          o1[4 * c4 + 1] = __float_as_uint(__uint_as_float(o1[4 * c4 + 1]) * v1.y);
          o1[4 * c4 + 2] = __float_as_uint(__uint_as_float(o1[4 * c4 + 2]) * v1.z);
          o1[4 * c4 + 3] = __float_as_uint(__uint_as_float(o1[4 * c4 + 3]) * v1.w);
        }
      }
      float* d0 = stg + (32 * (c & 1)) * kDv + 128 * (c >> 1) + 32 * quarter + lane;
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) d0[c2 * kDv] = __uint_as_float(o0[c2]);
      if (two) {
        float* d1 = stg + (32 * ((c + 3) & 1)) * kDv + 128 * ((c + 3) >> 1) + 32 * quarter + lane;
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) d1[c2 * kDv] = __uint_as_float(o1[c2]);
      }
    }
  }
  cluster_sync();  // #2: every split's O is staged and its coefficients are known
  {
    // this split's slice of the output: float4 e = h * 128 + d/4 of the [H][512] block,
    // which is also its byte offset / 16 in every split's staging buffer
    const int total = H * (kDv / 4);
    const int e0 = (int)((long long)split * total / nsplit), e1 = (int)((long long)(split + 1) * total / nsplit);
    const uint32_t stg_s = smem_u32(stg);
    if (nsplit > 1) {
      // all loads of this thread's elements (at most kPullPerThread) are issued before
      // any result is written back
      float4 acc[kPullPerThread];
#pragma unroll
      for (int q = 0; q < kPullPerThread; ++q) {
        const int e = e0 + (int)threadIdx.x + q * kThreadsA;
        acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < e1) {
          const int h = e >> 7;
          const uint32_t off = stg_s + 16u * (uint32_t)e;
#pragma unroll
          for (int sp = 0; sp < kMaxSplits; ++sp) {
            if (sp < nsplit) {
              const float cf = s_coef[sp * 64 + h];
              const float4 v = ld_cluster_v4(cluster_map(off, sp));
              acc[q].x = fmaf(cf, v.x, acc[q].x);
              acc[q].y = fmaf(cf, v.y, acc[q].y);
              acc[q].z = fmaf(cf, v.z, acc[q].z);
              acc[q].w = fmaf(cf, v.w, acc[q].w);
            }
          }
        }
      }
#pragma unroll
      for (int q = 0; q < kPullPerThread; ++q) {
        const int e = e0 + (int)threadIdx.x + q * kThreadsA;
        if (e < e1) reinterpret_cast<float4*>(stg)[e] = acc[q];
      }
    }
    fence_proxy_async();  // the results are visible to the bulk copy (async proxy)
    __syncthreads();
    if (threadIdx.x == 0 && e1 > e0) {
      bulk_store(layers.out[layer] + (size_t)row * H * kDv + 4 * (size_t)e0, stg_s + 16u * (uint32_t)e0,
                 (uint32_t)(e1 - e0) * 16u);
      bulk_commit();
      bulk_wait_all();
    }
  }
  tc_fence_before();
  cluster_sync();  // #3: the peers are done reading this CTA's staging buffer
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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

// 2-D bf16 map over [rows][576] with a 64-column x box_rows box and 128-byte swizzle
bool make_map_576(CUtensorMap* map, const void* base, long long rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDqk, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDqk * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

SymbolAddress g_err_addr;

}  // namespace

// Keys per split: a multiple of the 64-row granularity.
int attn_split_chunk(int k, int nsplit) {
  const int chunk = (k + nsplit - 1) / nsplit;
  return (chunk + kAttnTile - 1) / kAttnTile * kAttnTile;
}

namespace {
// How many clusters of each size (1..kMaxSplits) of this kernel fit on the GPU at once,
// per device; filled on the first launch on a device (before any stream capture).
int g_cluster_fit[64][kMaxSplits + 1];

cudaError_t query_cluster_fit() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  for (int c = 1; c <= kMaxSplits; ++c) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c, 1, 1);
    cfg.blockDim = dim3(kThreadsA);
    cfg.dynamicSmemBytes = kSmemA;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel, &cfg)) != cudaSuccess) return e;
    g_cluster_fit[dev][c] = n;
  }
  return cudaSuccess;
}
}  // namespace

// Splits per (query row, layer): the most (<= kMaxSplits, about one CTA per SM in total)
// whose clusters all fit on the GPU at once -- a second wave of clusters would double
// the time.  Without the device's figures (fit == nullptr) the SM count alone decides.
int attn_num_splits(long long rows, int L, int k, int sm_budget, const int* fit) {
  const long long units = rows * L > 0 ? rows * L : 1;
  const long long max_ns = (k + kAttnTile - 1) / kAttnTile;
  int best = 1;
  for (int ns = 1; ns <= kMaxSplits && ns <= max_ns; ++ns) {
    if (units * ns > sm_budget) break;
    if (fit && ns > 1 && units > fit[ns]) continue;  // (a size that cannot run at all reports 0)
    best = ns;
  }
  const int chunk = attn_split_chunk(k, best);
  return (k + chunk - 1) / chunk;
}

// The splits are reduced on chip (cluster shared memory): no global workspace.
size_t attn_workspace_bytes(long long, int, int, int) { return 0; }

cudaError_t launch_sparse_attn_tc(const AttnLayers& layers, int L, const int32_t* idx, int B, int T, int N, int H,
                                  int k, float scale, void*, bool q_early, cudaStream_t stream) {
  const long long rows = (long long)B * T;
  AttnMaps maps;
  for (int l = 0; l < L; ++l)
    if (!make_map_576(&maps.q[l], layers.q[l], rows * H, 64)) return cudaErrorInvalidValue;
  int* err = nullptr;
  cudaError_t e = g_err_addr.get(g_attn_tc_error, &err);
  if (e != cudaSuccess) return e;
  static DeviceOnce once;
  if ((e = once.run([] {
         cudaError_t e2 = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemA);
         return e2 != cudaSuccess ? e2 : query_cluster_fit();
       })) != cudaSuccess)
    return e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int nsplit = attn_num_splits(rows, L, k, sms, dev >= 0 && dev < 64 ? g_cluster_fit[dev] : nullptr);
  const int chunk = attn_split_chunk(k, nsplit);
  // the splits of one (row, layer) are one cluster along x
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nsplit, (unsigned)rows, L);
  cfg.blockDim = dim3(kThreadsA);
  cfg.dynamicSmemBytes = kSmemA;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nsplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // waits in-kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel, maps, layers, idx, T, N, H, k, chunk, scale * 1.4426950408889634f,
                            q_early ? 1 : 0, err);
}

cudaError_t attn_error_word(int** p) { return g_err_addr.get(g_attn_tc_error, p); }

}  // namespace dsa
