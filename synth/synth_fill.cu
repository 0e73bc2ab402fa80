// Device fill kernels for the seeded synthetic inputs.
//
// Same generator as the host module synth/__init__.py (SplitMix64 counter hash;
// integer-only arithmetic, so both produce bit-identical tensors).  This library holds
// no part of the DSA method; it only fills buffers with test and benchmark inputs.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t j) { return mix64(key + kGamma * (j + 1)); }

__device__ __forceinline__ uint16_t f32_bits_to_bf16_rne(uint32_t u) {
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

__global__ void fill_int17_bf16(uint16_t* out, int64_t n, uint64_t key, int64_t offset) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t h = draw(key, (uint64_t)(offset + i));
    int v = (int)((h >> 32) % 17u) - 8;
    float f = (float)v;
    out[i] = f32_bits_to_bf16_rne(__float_as_uint(f));
  }
}

// E4M3 bytes of the integers 0..8 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits)
__constant__ uint8_t kE4M3OfInt[9] = {0x00, 0x38, 0x40, 0x44, 0x48, 0x4A, 0x4C, 0x4E, 0x50};

__global__ void fill_int17_e4m3(uint8_t* out, int64_t n, uint64_t key, int64_t offset) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t h = draw(key, (uint64_t)(offset + i));
    int v = (int)((h >> 32) % 17u) - 8;
    out[i] = (uint8_t)(kE4M3OfInt[v < 0 ? -v : v] | (v < 0 ? 0x80 : 0));
  }
}

__global__ void fill_pow2_f32(float* out, int64_t n, uint64_t key, int64_t offset) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t h = draw(key, (uint64_t)(offset + i));
    int e = (int)((h >> 32) % 6u);
    out[i] = __uint_as_float((uint32_t)(127 - 1 - e) << 23);
  }
}

__global__ void fill_normal_bf16(uint16_t* out, int64_t n, uint64_t key, int64_t offset) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t base = 3ull * (uint64_t)(offset + i);
    int64_t s = 0;
#pragma unroll
    for (int sub = 0; sub < 3; ++sub) {
      uint64_t h = draw(key, base + sub);
#pragma unroll
      for (int fld = 0; fld < 4; ++fld) s += (int64_t)((h >> (16 * fld)) & 0xFFFFu);
    }
    // (s - 393210) * 2^-16 is exact in float32 (|s - 393210| < 2^19)
    float x = (float)(int32_t)(s - 393210) * (1.0f / 65536.0f);
    out[i] = f32_bits_to_bf16_rne(__float_as_uint(x));
  }
}

__global__ void fill_unit_f32(float* out, int64_t n, uint64_t key, int64_t offset) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t h = draw(key, (uint64_t)(offset + i));
    // (h >> 40) * 2^-24 - 0.5: exact in float32 (24-bit integer times a power of two)
    out[i] = (float)(uint32_t)(h >> 40) * (1.0f / 16777216.0f) - 0.5f;
  }
}

inline int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  return (int)(g < 148 * 32 ? (g < 1 ? 1 : g) : 148 * 32);
}

}  // namespace

extern "C" {

int synth_fill_int17_bf16(void* out, int64_t n, uint64_t key, int64_t offset, cudaStream_t s) {
  if (n <= 0) return 0;
  fill_int17_bf16<<<grid_for(n), 256, 0, s>>>((uint16_t*)out, n, key, offset);
  return (int)cudaGetLastError();
}
int synth_fill_int17_e4m3(void* out, int64_t n, uint64_t key, int64_t offset, cudaStream_t s) {
  if (n <= 0) return 0;
  fill_int17_e4m3<<<grid_for(n), 256, 0, s>>>((uint8_t*)out, n, key, offset);
  return (int)cudaGetLastError();
}
int synth_fill_pow2_f32(void* out, int64_t n, uint64_t key, int64_t offset, cudaStream_t s) {
  if (n <= 0) return 0;
  fill_pow2_f32<<<grid_for(n), 256, 0, s>>>((float*)out, n, key, offset);
  return (int)cudaGetLastError();
}
int synth_fill_normal_bf16(void* out, int64_t n, uint64_t key, int64_t offset, cudaStream_t s) {
  if (n <= 0) return 0;
  fill_normal_bf16<<<grid_for(n), 256, 0, s>>>((uint16_t*)out, n, key, offset);
  return (int)cudaGetLastError();
}
int synth_fill_unit_f32(void* out, int64_t n, uint64_t key, int64_t offset, cudaStream_t s) {
  if (n <= 0) return 0;
  fill_unit_f32<<<grid_for(n), 256, 0, s>>>((float*)out, n, key, offset);
  return (int)cudaGetLastError();
}

}  // extern "C"
