// Data movement of the backward pass (the GEMMs are in gemm_bwd.cu).
//
//   k_gather_pad   X rows of the FFN pairs into padded rows (expert e's pairs from
//                  row 128 mb_off[e] on); padding rows of X_pad and dY_pad set to 0
//   k_combine_bwd  dY_pad[pair] = g * dy_t; dg_tj = <dy_t, Y[pair]> (FFN slot) or
//                  <dy_t, x_t> (zero slot), a fixed-order block reduction
//   k_final_dx     dx_t = zsum_t dy_t + sum over FFN slots j in slot order of
//                  dX_pad[pair] + dx_router_t: the deterministic ScatterAdd
//                  (technical summary, 五 訓練基礎設施 確定性ScatterAdd) -- a gather per
//                  token in a fixed order, no atomics, one rounding to bf16
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_internal.h"

namespace zc {
namespace {

__device__ __forceinline__ void ld8f(const __nv_bfloat16* p, float* f) {
  const uint4 r = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ uint4 st8f(const float* f) {
  uint4 r;
  uint32_t* w = &r.x;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return r;
}

// Padded row q -> the pair it holds, or -1 for a padding row.
__device__ __forceinline__ int padded_pair(int64_t q, const int32_t* row_off, const int32_t* mb_off, int N) {
  const int b = (int)(q >> 7);
  int lo = 0, hi = N - 1;  // largest g with mb_off[g] <= b
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (mb_off[mid] <= b) lo = mid;
    else hi = mid - 1;
  }
  const int local = (int)(q - (int64_t)mb_off[lo] * 128);
  return local < row_off[lo + 1] - row_off[lo] ? row_off[lo] + local : -1;
}

__global__ void __launch_bounds__(256) k_gather_pad(const uint4* __restrict__ x, int vecs, const int32_t* __restrict__ perm,
                                                    int k, const int32_t* __restrict__ row_off,
                                                    const int32_t* __restrict__ mb_off, int N,
                                                    uint4* __restrict__ xpad, uint4* __restrict__ dypad) {
  const int64_t rows = (int64_t)mb_off[N] * 128;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < rows; q += nwarps) {
    const int p = padded_pair(q, row_off, mb_off, N);
    uint4* xd = xpad + q * vecs;
    if (p >= 0) {
      const uint4* xs = x + (int64_t)(perm[p] / k) * vecs;
      for (int v = lane; v < vecs; v += 32) xd[v] = xs[v];
    } else {
      uint4* dd = dypad + q * vecs;
      const uint4 z = make_uint4(0, 0, 0, 0);
      for (int v = lane; v < vecs; v += 32) {
        xd[v] = z;
        dd[v] = z;
      }
    }
  }
}

// One block per token, 128 threads, dy row staged in shared memory (d <= 16384).
__global__ void __launch_bounds__(128) k_combine_bwd(const __nv_bfloat16* __restrict__ x,
                                                     const __nv_bfloat16* __restrict__ dy,
                                                     const __nv_bfloat16* __restrict__ Y,
                                                     const float* __restrict__ gate, const int32_t* __restrict__ pos,
                                                     const int32_t* __restrict__ idx, const int32_t* __restrict__ offsets,
                                                     const int32_t* __restrict__ mb_off, int k, int d,
                                                     __nv_bfloat16* __restrict__ dypad, float* __restrict__ dg) {
  extern __shared__ __align__(16) uint8_t sm[];
  __nv_bfloat16* sdy = reinterpret_cast<__nv_bfloat16*>(sm);
  __shared__ float red[4];
  const int t = blockIdx.x;
  const int vecs = d / 8;
  const uint4* dyt = reinterpret_cast<const uint4*>(dy + (int64_t)t * d);
  for (int v = threadIdx.x; v < vecs; v += blockDim.x) reinterpret_cast<uint4*>(sdy)[v] = dyt[v];
  __syncthreads();
  for (int j = 0; j < k; ++j) {
    const int p = pos[(int64_t)t * k + j];
    const float g = gate[(int64_t)t * k + j];
    const __nv_bfloat16* src;
    uint4* dst = nullptr;
    if (p >= 0) {
      const int e = idx[(int64_t)t * k + j];
      src = Y + (int64_t)p * d;
      dst = reinterpret_cast<uint4*>(dypad + ((int64_t)(p - offsets[e]) + (int64_t)mb_off[e] * 128) * d);
    } else {
      src = x + (int64_t)t * d;
    }
    float part = 0.0f;
    for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
      float a[8], b[8];
      ld8f(sdy + v * 8, a);
      ld8f(src + v * 8, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) part = fmaf(a[i], b[i], part);
      if (dst) {
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] *= g;
        dst[v] = st8f(a);
      }
    }
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) part += __shfl_xor_sync(0xffffffffu, part, w);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
    __syncthreads();
    if (threadIdx.x == 0) dg[(int64_t)t * k + j] = (red[0] + red[1]) + (red[2] + red[3]);
    __syncthreads();
  }
}

__global__ void __launch_bounds__(128) k_final_dx(const __nv_bfloat16* __restrict__ dy,
                                                  const __nv_bfloat16* __restrict__ dxp,
                                                  const __nv_bfloat16* __restrict__ dxr,
                                                  const float* __restrict__ gate, const int32_t* __restrict__ pos,
                                                  const int32_t* __restrict__ idx, const int32_t* __restrict__ offsets,
                                                  const int32_t* __restrict__ mb_off, int k, int d,
                                                  __nv_bfloat16* __restrict__ dx) {
  __shared__ int64_t srow[32];
  __shared__ float szsum;
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    const int p = pos[(int64_t)t * k + threadIdx.x];
    const int e = idx[(int64_t)t * k + threadIdx.x];
    srow[threadIdx.x] = p >= 0 ? (int64_t)(p - offsets[e]) + (int64_t)mb_off[e] * 128 : -1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float z = 0.0f;
    for (int j = 0; j < k; ++j)
      if (srow[j] < 0) z = __fadd_rn(z, gate[(int64_t)t * k + j]);
    szsum = z;
  }
  __syncthreads();
  const float zsum = szsum;
  const int vecs = d / 8;
  for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
    float acc[8], a[8];
    ld8f(dy + (int64_t)t * d + v * 8, a);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = zsum * a[i];
    for (int j = 0; j < k; ++j) {
      const int64_t r = srow[j];
      if (r < 0) continue;
      ld8f(dxp + r * d + v * 8, a);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += a[i];
    }
    ld8f(dxr + (int64_t)t * d + v * 8, a);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += a[i];
    reinterpret_cast<uint4*>(dx + (int64_t)t * d)[v] = st8f(acc);
  }
}

}  // namespace

cudaError_t launch_gather_pad(const void* x, int d, const int32_t* perm, int k, const int32_t* row_off,
                              const int32_t* mb_off, int N, void* xpad, void* dypad, int sms, cudaStream_t s) {
  k_gather_pad<<<sms * 8, 256, 0, s>>>(static_cast<const uint4*>(x), d / 8, perm, k, row_off, mb_off, N,
                                        static_cast<uint4*>(xpad), static_cast<uint4*>(dypad));
  return cudaGetLastError();
}

cudaError_t launch_combine_bwd(const void* x, const void* dy, const void* Y, const float* gate, const int32_t* pos,
                               const int32_t* idx, const int32_t* offsets, const int32_t* mb_off, int T, int k, int d,
                               void* dypad, float* dg, cudaStream_t s) {
  k_combine_bwd<<<T, 128, (size_t)d * 2, s>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(dy), static_cast<const __nv_bfloat16*>(Y),
      gate, pos, idx, offsets, mb_off, k, d, static_cast<__nv_bfloat16*>(dypad), dg);
  return cudaGetLastError();
}

cudaError_t launch_final_dx(const void* dy, const void* dxp, const void* dxr, const float* gate, const int32_t* pos,
                            const int32_t* idx, const int32_t* offsets, const int32_t* mb_off, int T, int k, int d,
                            void* dx, cudaStream_t s) {
  k_final_dx<<<T, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(dy), static_cast<const __nv_bfloat16*>(dxp),
                               static_cast<const __nv_bfloat16*>(dxr), gate, pos, idx, offsets, mb_off, k, d,
                               static_cast<__nv_bfloat16*>(dx));
  return cudaGetLastError();
}

}  // namespace zc
