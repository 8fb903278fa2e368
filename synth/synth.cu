// CUDA twin of the seeded input generator defined in synth/__init__.py.
//
// Element n of the stream with 64-bit key K: three SplitMix64 outputs
// w_r = mix64(K + (3n + r + 1) * GOLDEN), the Irwin-Hall sum s of their twelve
// 16-bit lanes, x = (s - 393210) / 65536 (exact in fp32), then fp32 -> bf16
// round-to-nearest-even on the bit pattern. SplitMix64: Steele, Lea & Flood,
// "Fast splittable pseudorandom number generators", OOPSLA 2014.
//
// This file is test / benchmark infrastructure: it holds no arithmetic of the
// attention, RoPE, cache or sampler path.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void fill_normal_bf16_kernel(uint16_t* __restrict__ out, long long count,
                                        uint64_t key, long long start) {
  long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    uint64_t n = (uint64_t)(start + i);
    int32_t s = 0;
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      uint64_t w = mix64(key + (3ull * n + (uint64_t)(r + 1)) * kGolden);
#pragma unroll
      for (int lane = 0; lane < 4; ++lane) s += (int32_t)((w >> (16 * lane)) & 0xFFFFull);
    }
    float x = (float)(s - 393210) * (1.0f / 65536.0f);
    uint32_t u = __float_as_uint(x);
    u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
    out[i] = (uint16_t)u;
  }
}

}  // namespace

extern "C" int synth_fill_normal_bf16(void* out, long long count, unsigned long long key,
                                      long long start, void* stream) {
  if (count <= 0) return 0;
  if (out == nullptr) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (count + 255) / 256;
  long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  fill_normal_bf16_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      (uint16_t*)out, count, (uint64_t)key, start);
  return (int)cudaGetLastError();
}
