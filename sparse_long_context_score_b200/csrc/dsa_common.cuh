// dsa_common.cuh -- small device helpers shared by the libdsa kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "dsa.h"

namespace dsa {

// ---------------------------------------------------------------------------- bf16
// pack two floats into a bf16x2 word (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------------------- loads
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// cp.async 16 B global -> shared; src_bytes = 0 gives a zero fill
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes));
}
// the same copy under an L2 cache policy (createpolicy)
__device__ __forceinline__ void cp_async_16_hint(uint32_t dst, const void* src, int src_bytes, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst), "l"(src), "r"(src_bytes),
               "l"(policy));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------- ordering
// Monotone map from float to uint32: a > b (as numbers) <=> key(a) > key(b).
// -0 maps like +0 and every NaN maps to 0, below -inf.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;  // NaN
  if (u == 0x80000000u) u = 0u;                     // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ __forceinline__ long long visible_count(long long N, long long q_pos0, long long t) {
  long long v = q_pos0 + t + 1;
  return v < 0 ? 0 : (v > N ? N : v);
}

}  // namespace dsa
