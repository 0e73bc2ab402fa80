// attn_tc.cu -- sparse MLA attention on the 5th-generation tensor cores.
//
// "GLM-5.2 1M architecture teardown", Cut 1: DSA (full attention over only the 2048 keys
// the indexer kept) and Cut 3: MLA (one compressed 576-wide row per token, shared by all
// heads; in the absorbed form the logit of head h is scale * q[h] . c[j] and the value is
// the row's first 512 entries).
//
// One CTA per (query row, layer, key split); tiles of 64 selected rows, two stages.
//   S   = Q K^T   M = 64 heads, N = 64 keys, K = 576    (36 MMAs; TMEM lane = head)
//   O^T = V^T P^T M = 4 x 128 value dims, N = 64 heads, K = 64 keys (16 MMAs)
// A tcgen05.mma costs about 54 cycles whatever its size up to N = 64 (measured on B200:
// M = 64 reaches ~600 MAC/cycle at N = 32, ~1200 at N = 64, ~2000 at N >= 128), so the
// S product is issued with the widest N the shared memory allows: two stages of 64 rows
// (73.7 KB each) beside the 73.7 KB of Q.
// S has one head per TMEM lane, so a head's logits stay within one warp: its running max
// and sum live in registers (four threads per head, two shuffles per reduction).  The running max is
// only moved (and O rescaled in TMEM) when a tile's max exceeds it by more than 2^8, so
// rescaling is rare; exponentials may then exceed 1 by at most 2^8, which f32 and bf16
// carry without loss of relative precision.
//
// Warp roles (448 threads):
//   warps 0..7  gather: warps 4s..4s+3 own stage s and its tiles s, s+2, s+4, ...; each
//               brings 16 of the 64 selected rows as 16-byte cp.async chunks written
//               straight into the 128-byte-swizzled tensor-core layout (a lane holds its
//               own rows' indices, and one instruction moves four whole 128-byte lines),
//               waits for its own copies, fences them to the async proxy and arrives on the
//               stage barrier, so both stages gather at once; the row indices of the warp's
//               next tile are loaded while the current one is copied; a decode step's
//               rows, read once, are copied under an L2 evict-first policy.  (Random 1152-byte
//               rows are too small for TMA: measured on B200 with the same bytes in flight,
//               a 128-byte box per row reached 0.57 TB/s, 4-row gather boxes 1.6 TB/s, one
//               bulk copy per row 2.8 TB/s, 16-byte cp.async 4.9 TB/s.)
//   warp 8      TMEM allocation and the query load (one TMA load of the 64 query rows);
//               one elected lane issues S(i) once tile i has landed and its S buffer is
//               free, so the softmax of one tile overlaps the next tile's logits;
//   warps 9..12 softmax (warp q reads TMEM lanes 0..15 of quarter q, heads 16q..16q+15;
//               four threads per head), P as bf16 in shared memory;
//   warp 13     one elected lane issues O += P(i) V(i) once P(i) is published; as a warp
//               of its own it does not wait behind the next S, whose MMAs its own
//               interleave with in the tensor pipe, and a stage is released as soon as its
//               PV completes.
// A (row, layer) whose keys are split over several CTAs: each split writes its unnormalised
// O (straight from TMEM, 32 consecutive value dims of a head per warp store) and its
// running max and sum per head to a global partial block (L2-resident), and the combine
// kernel launched behind it (programmatic dependent launch: its CTAs wait on the device
// for this grid) merges the splits.  A single split writes the normalised output directly.
// The launch waits for the preceding kernel only where it reads that kernel's results.
// All mbarrier waits are bounded (sm100.cuh).
#include <cudaTypedefs.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

static __device__ int g_attn_tc_error;

constexpr int kKeys = kAttnTile;                 // selected rows per tile (64)
constexpr int kStages = 2;
constexpr int kBlocks = kDqk / 64;               // nine 64-wide column blocks of a row
constexpr int kQBlockBytes = 64 * 128;           // 64 heads x 64 bf16
constexpr int kBlockBytes = kKeys * 128;         // 64 rows x 64 bf16
constexpr int kQBytes = kBlocks * kQBlockBytes;  // 73728
constexpr int kStageBytes = kBlocks * kBlockBytes;  // 73728
// P of a tile (64 heads x 64 keys bf16, K-major 128-byte rows: 8 KB) is written over the
// tile's rope block (column block 8), which only the S product reads: P is then
// double-buffered with the stages at no cost in shared memory
constexpr int kPBlock = kDv / 64;                // column block 8
static_assert(64 * kKeys * 2 == kBlockBytes, "P fills one column block");
constexpr int kProducerWarps = 8;                // four warps per stage, 16 rows each
constexpr int kWarpsPerStage = kProducerWarps / kStages;
constexpr int kRowsPerWarp = kKeys / kWarpsPerStage;           // 16
constexpr int kMmaWarp = kProducerWarps;           // Q load, TMEM allocation, S = Q K^T
constexpr int kSoftmaxWarp0 = kProducerWarps + 1;
constexpr int kPvWarp = kSoftmaxWarp0 + 4;         // O^T += V^T P^T
constexpr int kThreadsA = (kPvWarp + 1) * 32;      // 448
static_assert(kThreadsA == 448, "8 gather, 1 S, 4 softmax and 1 PV warp");
static_assert(kRowsPerWarp == 16, "a gather warp copies 4 x 4 rows");
constexpr float kRescaleLog2 = 8.f;
constexpr int kMaxSplits = 32;                   // key splits of one (row, layer): a combine warp's lanes

constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQBytes;
constexpr int kOffAlpha = kOffStage + kStages * kStageBytes;  // [2][64] f32 (tile parity)
constexpr int kOffL = kOffAlpha + 2 * 64 * 4;    // [64] f32
constexpr int kOffM = kOffL + 64 * 4;            // [64] f32
constexpr int kOffCoef = kOffM + 64 * 4;         // [64] f32: this split's share of the normaliser
constexpr int kOffMask = kOffCoef + 64 * 4;      // [kStages] u64: valid rows of the tile in the stage
constexpr int kOffVote = kOffMask + kStages * 8;  // [2] u32 (tile parity): one byte per softmax warp
constexpr int kNumBars = 2 * kStages + 11;
constexpr int kOffBar = kOffVote + 8;
constexpr int kOffTmem = kOffBar + kNumBars * 8;
constexpr int kSmemA = kOffTmem + 16 + 1024;     // + alignment slack
static_assert(kSmemA <= 232448, "shared memory budget");
static_assert(kOffBar % 8 == 0 && kOffMask % 8 == 0, "barrier and mask alignment");

constexpr int kTmemO = 0;      // O^T: 4 blocks x 64 columns, all 128 lanes
constexpr int kTmemS = 256;    // S: 2 buffers x 64 columns, lanes 0..15 of each quarter
constexpr int kTmemCols = 512;

constexpr int kPartialFloats = 64 * kDv;         // one split's [64][512] partial output
constexpr int kPartialMl = 64 * 2;               // ... and its (m, l) per head

struct AttnMaps {
  CUtensorMap q[kMaxLayers];
};

// kernel flags
constexpr int kAttnQEarly = 1;     // the queries may be loaded before the preceding kernel ends
constexpr int kAttnRowsOnce = 2;   // gathered rows are read once: L2 evict-first policy

// 13 warps: one SM sub-partition hosts four of them, so 128 registers per thread at most
__global__ void __launch_bounds__(kThreadsA, 1)
attn_tc_kernel(const __grid_constant__ AttnMaps maps, AttnLayers layers, const int32_t* __restrict__ idx, int T, int N,
               int H, int k, int chunk, float scale_log2, int flags, long long idx_offset, float* __restrict__ partials,
               float2* __restrict__ partial_ml, int* __restrict__ err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + kOffQ;
  const uint32_t sStage = sbase + kOffStage;
  float* s_alpha = reinterpret_cast<float*>(smem + kOffAlpha);
  float* s_l = reinterpret_cast<float*>(smem + kOffL);
  float* s_m = reinterpret_cast<float*>(smem + kOffM);
  float* s_coef = reinterpret_cast<float*>(smem + kOffCoef);
  unsigned long long* s_mask = reinterpret_cast<unsigned long long*>(smem + kOffMask);
  uint32_t* s_vote = reinterpret_cast<uint32_t*>(smem + kOffVote);
  const uint32_t bar0 = sbase + kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto sfull_bar = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
  auto sfree_bar = [&](int s) { return bar0 + 8u * (2 * kStages + 2 + s); };
  // P of the tile in stage s published (one phase per use of the stage)
  auto pfull_bar = [&](int s) { return bar0 + 8u * (2 * kStages + 4 + s); };
  const uint32_t pfree_bar = bar0 + 8u * (2 * kStages + 6);
  const uint32_t ofinal_bar = bar0 + 8u * (2 * kStages + 7);
  const uint32_t qfull_bar = bar0 + 8u * (2 * kStages + 8);
  const uint32_t grp_bar = bar0 + 8u * (2 * kStages + 9);
  const uint32_t sdone_bar = bar0 + 8u * (2 * kStages + 10);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffTmem);

  const int split = blockIdx.x, row = blockIdx.y, layer = blockIdx.z;
  const int nsplit = gridDim.x;
  const int b = row / T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = split * chunk;
  const int nkeys = max(min(j0 + chunk, k) - j0, 0);
  const int ntiles = (nkeys + kKeys - 1) / kKeys;
  // the split combine behind this grid may be scheduled once every CTA of it has started;
  // it waits on the device for this grid to complete
  grid_dep_launch();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), kWarpsPerStage);
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(sfull_bar(s), 1);
      mbar_init(sfree_bar(s), 128);
    }
    for (int s = 0; s < kStages; ++s) mbar_init(pfull_bar(s), 128);
    mbar_init(pfree_bar, 1);
    mbar_init(ofinal_bar, 1);
    mbar_init(qfull_bar, 1);
    mbar_init(grp_bar, 128);
    mbar_init(sdone_bar, 1);
    fence_mbar_init();
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
    // warps 4s..4s+3 fill rows [16 (w % 4), 16 (w % 4) + 16) of tiles s, s + 2, ...: lane l
    // copies chunks l + 32 j (j < 36) of the warp's 16 x 72 chunks of 16 bytes, in row
    // (l + 32 j) / 72 of the warp's rows; lanes 0..15 hold the row indices
    const int ps = warp / kWarpsPerStage, wq = warp % kWarpsPerStage;
    const int r0 = kRowsPerWarp * wq;
    // the index list comes from the preceding kernel.  (Every other warp waits on the
    // gather through the pipeline barriers, and the output is written only after the CTA
    // barrier that follows this wait.)
    grid_dep_wait();
    const int32_t* sel = idx + (size_t)row * k + j0;
    const uint16_t* kvb = layers.kv[layer] + (size_t)b * N * kDqk;
    const uint32_t st = sStage + ps * kStageBytes;
    // lane l copies, for g < 4, row r0 + 4g + l/8 of the tile: its 16-byte chunks l%8 + 8m
    // (m < 9), i.e. 16 bytes of each of the row's nine 128-byte column blocks.  One
    // instruction thus moves four whole 128-byte lines (four rows, one column block), and
    // every lane holds its own rows' indices (no shuffles in the copy loop).
    const int rsub = lane >> 3, c8 = lane & 7;
    auto load_index = [&](int tile, int (&out)[4]) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int key = tile * kKeys + r0 + 4 * g + rsub;
        // a selected global position, as a row of this cache (which holds positions
        // [idx_offset, idx_offset + N)); -1 when it is padding or outside
        const long long gp = (tile < ntiles && key < nkeys) ? (long long)__ldg(&sel[key]) - idx_offset : -1;
        out[g] = gp >= 0 && gp < N ? (int)gp : -1;
      }
    };
    const bool rows_once = (flags & kAttnRowsOnce) != 0;
    const uint64_t row_policy = l2_evict_first_policy();
    int cur[4], nxt[4];
    load_index(ps, cur);
    for (int i = ps; i < ntiles; i += kStages) {
      load_index(i + kStages, nxt);  // in flight while this tile is copied
      bool ok = true;
      if (lane == 0) ok = mbar_wait(empty_bar(ps), ((i / kStages) & 1) ^ 1, err, 21);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      uint32_t vm = 0;  // bit 4g + t: row r0 + 4g + t of the tile is a valid selection
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, cur[g] >= 0 && cur[g] < N);
#pragma unroll
        for (int t = 0; t < 4; ++t) vm |= ((bal >> (8 * t)) & 1u) << (4 * g + t);
      }
      if (lane == 0) reinterpret_cast<uint16_t*>(s_mask + ps)[wq] = (uint16_t)vm;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const bool v = cur[g] >= 0 && cur[g] < N;
        const uint16_t* src = kvb + (size_t)(v ? cur[g] : 0) * kDqk + c8 * 8;
        const int r = r0 + 4 * g + rsub;
        const uint32_t dst = st + r * 128 + ((c8 ^ (r & 7)) << 4);
        if (rows_once) {
#pragma unroll
          for (int m = 0; m < kBlocks; ++m) cp_async_16_hint(dst + m * kBlockBytes, src + m * 64, v ? 16 : 0, row_policy);
        } else {
#pragma unroll
          for (int m = 0; m < kBlocks; ++m) cp_async_16(dst + m * kBlockBytes, src + m * 64, v ? 16 : 0);
        }
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async();  // the copies are visible to the tensor core (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(full_bar(ps));
#pragma unroll
      for (int g = 0; g < 4; ++g) cur[g] = nxt[g];
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ S issuer
    // the whole warp runs the loop (descriptor arithmetic stays warp-uniform); one
    // elected lane issues the tensor-core instructions
    const bool leader = elect_one();
    if (leader) {
      // the queries may be read before the preceding kernel completes only when the caller
      // knows that kernel does not write them (the top-k of the same group)
      tma_prefetch(&maps.q[layer]);
      if (!(flags & kAttnQEarly)) grid_dep_wait();
      const CUtensorMap* qm = &maps.q[layer];
      mbar_arrive_expect_tx(qfull_bar, kQBytes);
      for (int kb = 0; kb < kBlocks; ++kb) tma_load_2d(sQ + kb * kQBlockBytes, qm, qfull_bar, 64 * kb, row * H);
    }
    __syncwarp();
    constexpr uint32_t idS = idesc_bf16_f32(64, kKeys);              // Q (K-major) x K (K-major)
    bool ok = mbar_wait(qfull_bar, 0, err, 22);
    const uint64_t dq = sdesc_kmajor_sw128(sQ);
    // S(i) needs tile i in its stage and a free S buffer.  PV is issued by its own warp, so
    // a PV that becomes ready enters the tensor pipe between the MMAs of the next S
    // instead of behind all of them.
    for (int i = 0; i < ntiles && ok; ++i) {
      const int st = i % kStages, sb = i & 1;
      ok = mbar_wait(full_bar(st), (i / kStages) & 1, err, 24) &&
           mbar_wait(sfree_bar(sb), ((i >> 1) & 1) ^ 1, err, 25);
      if (!ok) break;
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
    }
    if (leader) {
      mma_commit(sdone_bar);
      if (!mbar_wait_drain(sdone_bar, 0)) atomicCAS(err, 0, 26);
      // the query load has landed even when the loop gave up early
      mbar_wait_drain(qfull_bar, 0);
    }
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------------ PV issuer
    const bool leader = elect_one();
    constexpr uint32_t idPV = idesc_bf16_f32(128, 64, true, false);  // V^T (M-major) x P (K-major)
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int sj = j % kStages;
      ok = mbar_wait(pfull_bar(sj), (j / kStages) & 1, err, 23);
      if (!ok) break;
      tc_fence_after();
      const uint64_t da = sdesc_mnmajor_sw128(sStage + sj * kStageBytes, kBlockBytes, 1024);
      const uint64_t dp = sdesc_kmajor_sw128(sStage + sj * kStageBytes + kPBlock * kBlockBytes);
      if (leader) {
#pragma unroll
        for (int mb = 0; mb < 4; ++mb)
#pragma unroll
          for (int ks = 0; ks < kKeys / 16; ++ks)
            mma_bf16(tmem + kTmemO + 64 * mb, da + (uint64_t)(((2 * mb) * kBlockBytes + ks * 16 * 128) >> 4),
                     dp + (uint64_t)((ks * 32) >> 4), idPV, (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(pfree_bar);
        mma_commit(empty_bar(sj));  // the stage's rows and P are consumed
      }
      __syncwarp();
    }
    if (leader) {
      mma_commit(ofinal_bar);
      if (!mbar_wait_drain(ofinal_bar, 0)) atomicCAS(err, 0, 26);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax
    // One 16-lane x 64-column TMEM load per tile gives every thread of the warp 32 logits:
    // heads hA = 16 quarter + t/4 and hB = hA + 8, keys 8j + 2(t % 4) + {0, 1} (j < 8).  The
    // four threads of a head hold identical copies of its running max (reduced over them
    // with two shuffles) and partial sums of its normaliser.
    const int quarter = warp & 3;
    const int c4 = lane & 3;
    const int hA = 16 * quarter + (lane >> 2), hB = hA + 8;
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    uint32_t grp_phase = 0;
    bool ok = true;
    unsigned char* pbase = smem + kOffStage + kPBlock * kBlockBytes;
    for (int i = 0; i < ntiles && ok; ++i) {
      const int sb = i & 1, s = i % kStages;
      ok = mbar_wait(sfull_bar(sb), (i >> 1) & 1, err, 27);
      if (!ok) break;
      tc_fence_after();
      ok = mbar_wait(full_bar(s), (i / kStages) & 1, err, 28);  // orders the gather's mask write
      if (!ok) break;
      // this thread's keys: 8j + 2 c4 + e; shifted so that bit 2j + e is key 8j + 2 c4 + e
      const unsigned long long mask = s_mask[s] >> (2 * c4);
      float* alpha = s_alpha + 64 * (i & 1);
      uint32_t r[32];
      tmem_ld16x256b_x8(tmem + lane_addr + kTmemS + kKeys * sb, r);
      tmem_ld_wait();
      float tA = -INFINITY, tB = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool v = (mask >> (8 * j + e)) & 1ull;
          const float zA = v ? __uint_as_float(r[4 * j + e]) * scale_log2 : -INFINITY;
          const float zB = v ? __uint_as_float(r[4 * j + 2 + e]) * scale_log2 : -INFINITY;
          r[4 * j + e] = __float_as_uint(zA);
          r[4 * j + 2 + e] = __float_as_uint(zB);
          tA = fmaxf(tA, zA);
          tB = fmaxf(tB, zB);
        }
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        tA = fmaxf(tA, __shfl_xor_sync(0xFFFFFFFFu, tA, o));
        tB = fmaxf(tB, __shfl_xor_sync(0xFFFFFFFFu, tB, o));
      }
      // The running max moves only on a head's first tile with a valid key (O and l are
      // still zero) or when the tile's max exceeds it by more than 2^8 (O is rescaled).
      auto update = [&](float& m, float& l, float t) {
        float a = 1.f;
        if (m == -INFINITY) {
          m = t;
        } else if (t > m + kRescaleLog2) {
          a = exp2f(m - t);
          m = t;
          l *= a;
        }
        return a;
      };
      const float aA = update(mA, lA, tA), aB = update(mB, lB, tB);
      const float muA = mA == -INFINITY ? 0.f : mA, muB = mB == -INFINITY ? 0.f : mB;
      unsigned char* prowA = pbase + s * kStageBytes + hA * 128 + 4 * c4;
      unsigned char* prowB = pbase + s * kStageBytes + hB * 128 + 4 * c4;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float pA0 = exp2f(__uint_as_float(r[4 * j]) - muA), pA1 = exp2f(__uint_as_float(r[4 * j + 1]) - muA);
        const float pB0 = exp2f(__uint_as_float(r[4 * j + 2]) - muB), pB1 = exp2f(__uint_as_float(r[4 * j + 3]) - muB);
        lA += pA0 + pA1;
        lB += pB0 + pB1;
        // P rows are K-major with the 128-byte swizzle: 16-byte chunk j of row h sits at
        // chunk j ^ (h % 8)
        *reinterpret_cast<uint32_t*>(prowA + ((j ^ (hA & 7)) << 4)) = pack_bf16x2(pA0, pA1);
        *reinterpret_cast<uint32_t*>(prowB + ((j ^ (hB & 7)) << 4)) = pack_bf16x2(pB0, pB1);
      }
      if (c4 == 0) {
        alpha[hA] = aA;
        alpha[hB] = aB;
      }
      // one vote per warp: does any of its heads need O rescaled?
      const uint32_t vote = __ballot_sync(0xFFFFFFFFu, (hA < H && aA != 1.f) || (hB < H && aB != 1.f));
      if (lane == 0) reinterpret_cast<volatile unsigned char*>(s_vote + (i & 1))[quarter] = vote != 0u ? 1 : 0;
      // every head's factor is known before O is touched
      mbar_arrive(grp_bar);
      ok = mbar_wait(grp_bar, grp_phase, err, 29);
      grp_phase ^= 1;
      if (!ok) break;
      const bool any = *reinterpret_cast<volatile uint32_t*>(s_vote + (i & 1)) != 0u;
      if (i > 0 && any) {
        // O^T is rescaled only once the previous tile's PV has finished with it
        ok = mbar_wait(pfree_bar, (i - 1) & 1, err, 30);
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
      fence_proxy_async();  // the P stores are visible to the tensor core (async proxy)
      // S of this tile has been read: its TMEM buffer is free for the next-but-one tile
      tc_fence_before();
      mbar_arrive(sfree_bar(sb));
      tc_fence_before();
      mbar_arrive(pfull_bar(s));
    }
    // the normaliser of each head: the sum of its four threads' partial sums
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      lA += __shfl_xor_sync(0xFFFFFFFFu, lA, o);
      lB += __shfl_xor_sync(0xFFFFFFFFu, lB, o);
    }
    if (c4 == 0) {
      s_l[hA] = lA;
      s_m[hA] = mA;
      s_l[hB] = lB;
      s_m[hB] = mB;
    }
  }

  // ------------------------------------------------------------------ epilogue
  // A single split writes O / l; a split of several writes its unnormalised O to its
  // [64][512] partial block and its (m, l) per head, which the combine kernel merges.
  tc_fence_before();
  __syncthreads();  // (m, l) of this split published; its MMAs have completed
  tc_fence_after();
  const bool split_mode = nsplit > 1;
  const size_t unit = (size_t)layer * gridDim.y + row;
  if (threadIdx.x < 64) {
    const int h = threadIdx.x;
    s_coef[h] = split_mode ? 1.f : (s_l[h] > 0.f ? 1.f / s_l[h] : 0.f);
    if (split_mode) {
      partial_ml[(unit * nsplit + split) * 64 + h] = make_float2(s_m[h], s_l[h]);
    } else if (layers.lse[layer] && h < H) {
      // natural log-sum-exp of the logits: m and l are in base 2 (sum_j 2^(z_j) = 2^m l)
      layers.lse[layer][(size_t)row * H + h] = s_l[h] > 0.f ? (s_m[h] + log2f(s_l[h])) * 0.69314718055994531f : -INFINITY;
    }
  }
  __syncthreads();  // s_coef
  // Twelve warps, three per TMEM lane quarter, take the eight 32-column chunks of O^T (TMEM
  // lane = value dim, column = head); for each head a warp stores 32 consecutive value dims
  // (128 bytes) from its registers.  The output holds H heads, a partial block all 64.
  float* dst = split_mode ? partials + (unit * nsplit + split) * kPartialFloats : layers.out[layer] + (size_t)row * H * kDv;
  const int hmax = split_mode ? 64 : H;
  if (warp != kMmaWarp && warp != kPvWarp) {
    const int quarter = warp & 3;
    const int jw = warp < kProducerWarps ? warp >> 2 : 2;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16) + kTmemO;
    // chunks jw, jw + 3 (loaded together), then jw + 6
    for (int c0 = jw; c0 < 8; c0 += 6) {
      const int c1 = c0 + 3;
      const bool two = c1 < 8;
      uint32_t o0[32], o1[32];
      if (ntiles > 0) {
        tmem_ld32(lane_base + 64 * (c0 >> 1) + 32 * (c0 & 1), o0);
        if (two) tmem_ld32(lane_base + 64 * (c1 >> 1) + 32 * (c1 & 1), o1);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) o0[c2] = o1[c2] = 0u;
      }
      {
        const int hh = 32 * (c0 & 1), lim = hmax - hh;
        float* d = dst + hh * kDv + 128 * (c0 >> 1) + 32 * quarter + lane;
        const float* cf = s_coef + hh;
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2)
          if (c2 < lim) d[c2 * kDv] = __uint_as_float(o0[c2]) * cf[c2];
      }
      if (two) {
        const int hh = 32 * (c1 & 1), lim = hmax - hh;
        float* d = dst + hh * kDv + 128 * (c1 >> 1) + 32 * quarter + lane;
        const float* cf = s_coef + hh;
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2)
          if (c2 < lim) d[c2 * kDv] = __uint_as_float(o1[c2]) * cf[c2];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
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

// Merges the key splits of every (row, layer):
//   out[h] = sum_s 2^(m_s[h] - M[h]) O_s[h] / sum_s 2^(m_s[h] - M[h]) l_s[h],  M[h] = max_s m_s[h],
// and the natural log-sum-exp (M[h] + log2 of the denominator) * ln 2 when asked.  One CTA
// per (8 heads, row, layer); warp w takes head 8 x + w: lane s < nsplit reads split s's
// (m, l) and forms its coefficient, then every lane sums four float4 of the head's 512
// values over the splits.  Launched behind the attention as its programmatic dependent.
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ partials,
                                                           const float2* __restrict__ partial_ml, AttnLayers layers,
                                                           int H, int nsplit) {
  grid_dep_wait();  // the attention's partials
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * 8 + warp, row = blockIdx.y, layer = blockIdx.z;
  if (h >= H) return;
  const size_t unit = (size_t)layer * gridDim.y + row;
  float m = -INFINITY, l = 0.f;
  if (lane < nsplit) {
    const float2 v = partial_ml[(unit * nsplit + lane) * 64 + h];
    m = v.x;
    l = v.y;
  }
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
  float c = m == -INFINITY ? 0.f : exp2f(m - M);  // (M is finite when m is)
  float den = c * l;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xFFFFFFFFu, den, o);
  c = den > 0.f ? c / den : 0.f;
  if (lane == 0 && layers.lse[layer])
    layers.lse[layer][(size_t)row * H + h] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
  const float4* p = reinterpret_cast<const float4*>(partials + unit * nsplit * kPartialFloats) + h * (kDv / 4) + lane;
  float4 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int sp = 0; sp < nsplit; ++sp) {
    const float cs = __shfl_sync(0xFFFFFFFFu, c, sp);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldcg(p + (size_t)sp * (kPartialFloats / 4) + 32 * i);
      acc[i].x += cs * v.x;
      acc[i].y += cs * v.y;
      acc[i].z += cs * v.z;
      acc[i].w += cs * v.w;
    }
  }
  float4* out = reinterpret_cast<float4*>(layers.out[layer] + ((size_t)row * H + h) * kDv) + lane;
#pragma unroll
  for (int i = 0; i < 4; ++i) out[32 * i] = acc[i];
}

// kernel attributes, once per device
cudaError_t attn_setup() {
  static DeviceOnce once;
  return once.run([] { return cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemA); });
}

// splits of the launch on the current device, within an SM budget (0: all SMs); 0 when
// the device cannot be queried
int launch_splits(long long rows, int L, int k, int sm_budget) {
  const int sms = device_sm_count();
  if (sms <= 0 || attn_setup() != cudaSuccess) return 0;
  return attn_num_splits(rows, L, k, sm_budget > 0 && sm_budget < sms ? sm_budget : sms);
}

}  // namespace

// Keys per split: a multiple of the 64-row tile.
int attn_split_chunk(int k, int nsplit) {
  const int chunk = (k + nsplit - 1) / nsplit;
  return (chunk + kAttnTile - 1) / kAttnTile * kAttnTile;
}

// Splits per (query row, layer): the most (<= kMaxSplits, one per 64-row tile at most)
// with at most one CTA per SM of the budget in total -- a second wave of CTAs would double
// the time.
int attn_num_splits(long long rows, int L, int k, int sm_budget) {
  const long long units = rows * L > 0 ? rows * L : 1;
  const long long max_ns = (k + kAttnTile - 1) / kAttnTile;
  int best = 1;
  for (int ns = 1; ns <= kMaxSplits && ns <= max_ns; ++ns) {
    if (units * ns > sm_budget) break;
    best = ns;
  }
  const int chunk = attn_split_chunk(k, best);
  return (k + chunk - 1) / chunk;
}

// The split partials: one [64][512] f32 block and 64 (m, l) pairs per (layer, row, split)
// when a (row, layer) is split, none otherwise; sized for the splits of the launch on the
// current device.
size_t attn_workspace_bytes(long long rows, int L, int, int k, int sm_budget) {
  const int ns = launch_splits(rows, L, k, sm_budget);
  return ns > 1 ? (size_t)rows * L * ns * (kPartialFloats + kPartialMl) * sizeof(float) : 0;
}

cudaError_t launch_sparse_attn_tc(const AttnLayers& layers, int L, const int32_t* idx, int B, int T, int N, int H,
                                  int k, float scale, long long idx_offset, void* ws, size_t ws_bytes, bool q_early,
                                  bool rows_once, int sm_budget, cudaStream_t stream) {
  const long long rows = (long long)B * T;
  AttnMaps maps;
  for (int l = 0; l < L; ++l)
    if (!make_map_576(&maps.q[l], layers.q[l], rows * H, 64)) return cudaErrorInvalidValue;
  int* err = nullptr;
  cudaError_t e = g_err_addr.get(g_attn_tc_error, &err);
  if (e != cudaSuccess) return e;
  const int nsplit = launch_splits(rows, L, k, sm_budget);
  if (nsplit <= 0) return cudaErrorInvalidDevice;
  const int chunk = attn_split_chunk(k, nsplit);
  const size_t part_floats = (size_t)rows * L * nsplit * kPartialFloats;
  if (nsplit > 1 && (!ws || ws_bytes < (size_t)rows * L * nsplit * (kPartialFloats + kPartialMl) * sizeof(float)))
    return cudaErrorInvalidValue;
  float* partials = static_cast<float*>(ws);
  float2* partial_ml = nsplit > 1 ? reinterpret_cast<float2*>(partials + part_floats) : nullptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nsplit, (unsigned)rows, L);
  cfg.blockDim = dim3(kThreadsA);
  cfg.dynamicSmemBytes = kSmemA;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // waits in-kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int flags = (q_early ? kAttnQEarly : 0) | (rows_once ? kAttnRowsOnce : 0);
  e = cudaLaunchKernelEx(&cfg, attn_tc_kernel, maps, layers, idx, T, N, H, k, chunk, scale * 1.4426950408889634f, flags,
                         idx_offset, partials, partial_ml, err);
  if (e != cudaSuccess || nsplit == 1) return e;
  // the split combine, as the attention's programmatic dependent
  cudaLaunchConfig_t ccfg = {};
  ccfg.gridDim = dim3((unsigned)((H + 7) / 8), (unsigned)rows, L);
  ccfg.blockDim = dim3(256);
  ccfg.stream = stream;
  ccfg.attrs = attr;
  ccfg.numAttrs = 1;
  return cudaLaunchKernelEx(&ccfg, attn_combine_kernel, static_cast<const float*>(partials),
                            static_cast<const float2*>(partial_ml), layers, H, nsplit);
}

cudaError_t attn_error_word(int** p) { return g_err_addr.get(g_attn_tc_error, p); }

}  // namespace dsa
