// Seeded synthetic-input generator, device side (libzcsynth.so).
//
// Bit-identical twin of the numpy generator in __init__.py: Philox4x32-10
// (Salmon et al., SC'11) keyed by the seed, counter (lo32(i), hi32(i), tid, block),
// turned into values by the Irwin-Hall normal recipe and the exact uniform recipe
// documented there.  It contains none of the MoE layer's arithmetic and is only
// used to put test and benchmark inputs into device memory.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

struct U4 { uint32_t x, y, z, w; };

__device__ __forceinline__ U4 philox10(U4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = U4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
  }
  return c;
}

__device__ __forceinline__ uint32_t halves(uint32_t w) { return (w & 0xFFFFu) + (w >> 16); }

__device__ __forceinline__ float normal_at(uint64_t i, uint32_t tid, uint64_t seed, float stdv) {
  const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  const U4 a = philox10(U4{(uint32_t)i, (uint32_t)(i >> 32), tid, 0u}, k0, k1);
  const U4 b = philox10(U4{(uint32_t)i, (uint32_t)(i >> 32), tid, 1u}, k0, k1);
  const int32_t s = (int32_t)(halves(a.x) + halves(a.y) + halves(a.z) + halves(a.w) + halves(b.x) + halves(b.y));
  const float z = __fdiv_rn((float)(s - 393210), 65536.0f);  // exact: |s - 393210| < 2**20
  return __fmul_rn(z, stdv);
}

__global__ void k_normal(void* dst, int64_t n, int bf16, uint32_t tid, uint64_t seed, float stdv) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float v = normal_at((uint64_t)i, tid, seed, stdv);
    if (bf16) static_cast<__nv_bfloat16*>(dst)[i] = __float2bfloat16_rn(v);
    else static_cast<float*>(dst)[i] = v;
  }
}

__global__ void k_uniform(float* dst, int64_t n, uint32_t tid, uint64_t seed, float lo, float hi) {
  const float span = __fsub_rn(hi, lo);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const U4 a = philox10(U4{(uint32_t)i, (uint32_t)((uint64_t)i >> 32), tid, 0u}, (uint32_t)seed, (uint32_t)(seed >> 32));
    const float u = __fmul_rn((float)(2u * (a.x >> 9) + 1u), 5.9604644775390625e-08f);  // * 2**-24, exact
    dst[i] = __fadd_rn(lo, __fmul_rn(span, u));
  }
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (n + 255) / 256;
  int64_t cap = (int64_t)sms * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

extern "C" {

// Fills dst[0..n) (device, float32 if bf16 == 0 else bfloat16) with the normal recipe.
// Returns 0 or the cudaError_t of the launch.
__attribute__((visibility("default"))) int zcsynth_normal(void* dst, int64_t n, int bf16, uint32_t tid, uint64_t seed, float stdv, cudaStream_t stream) {
  if (n <= 0) return 0;
  k_normal<<<grid_for(n), 256, 0, stream>>>(dst, n, bf16, tid, seed, stdv);
  return (int)cudaGetLastError();
}

// Fills dst[0..n) (device float32) with the uniform recipe on (lo, hi).
__attribute__((visibility("default"))) int zcsynth_uniform(float* dst, int64_t n, uint32_t tid, uint64_t seed, float lo, float hi, cudaStream_t stream) {
  if (n <= 0) return 0;
  k_uniform<<<grid_for(n), 256, 0, stream>>>(dst, n, tid, seed, lo, hi);
  return (int)cudaGetLastError();
}

}  // extern "C"
