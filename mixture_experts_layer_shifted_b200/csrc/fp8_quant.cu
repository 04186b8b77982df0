// Block quantizers to FP8 E4M3 with E8M0 power-of-two scales (rule in zc_fp8.cuh):
//   k_quant_rows  : [1,128] blocks (activations), one warp per block
//   k_quant_tiles : [128,128] blocks (weights), one CTA per block
//   k_scatter_quant: the FFN pairs' token rows, quantized on the way into the padded,
//                   expert-sorted operand of the block-scaled gate/up GEMM (all formats)
// and their W4A4 forms: MXFP4 ([1,32] blocks, k_quant_mx4) and NVFP4 ([1,16] blocks with a
// tensor scale: k_matrix_amax + k_nv4_global, then k_quant_nv4).
// Scales go out either plain ([row blocks, cols/128], for zcmoe_quantize_e4m3)
// or as the GEMM's scale atoms.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_fp8.cuh"
#include "zc_internal.h"

namespace zc {
namespace {

__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ld_f(const float* p) { return *p; }

// four consecutive elements (8- or 16-byte aligned)
__device__ __forceinline__ void ld4(const __nv_bfloat16* p, float* v) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
  v[0] = a.x;
  v[1] = a.y;
  v[2] = b.x;
  v[3] = b.y;
}
__device__ __forceinline__ void ld4(const float* p, float* v) {
  const float4 r = *reinterpret_cast<const float4*>(p);
  v[0] = r.x;
  v[1] = r.y;
  v[2] = r.z;
  v[3] = r.w;
}

__device__ __forceinline__ float warp_max(float a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  return a;
}

template <typename TIN, bool ATOM>
__global__ void __launch_bounds__(256) k_quant_rows(const TIN* __restrict__ src, int64_t rows, int cols,
                                                    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                    int groups) {
  const int lane = threadIdx.x & 31;
  const int ncb = cols >> 7;
  const int64_t nblk = rows * ncb;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < nblk; i += nwarps) {
    const int64_t r = i / ncb;
    const int cb = (int)(i - r * ncb);
    const int64_t off = r * cols + cb * 128 + lane * 4;
    float v[4];
    ld4(src + off, v);
    const float amax = warp_max(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
    const uint32_t code = e8m0_code(amax);
    const float inv = e8m0_inverse(code);
    *reinterpret_cast<uint32_t*>(codes + off) = pack_e4m3x4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
    if (lane == 0) scales[ATOM ? atom_offset(r, cb, groups) : r * ncb + cb] = (uint8_t)code;
  }
}

template <typename TIN, bool ATOM>
__global__ void __launch_bounds__(128) k_quant_tiles(const TIN* __restrict__ src, int64_t rows, int cols,
                                                     uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                     int groups) {
  __shared__ float part[4];
  const int cb = blockIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * 128;
  const int nr = (int)(rows - r0 < 128 ? rows - r0 : 128);
  const int c = cb * 128 + threadIdx.x;
  float amax = 0.0f;
  for (int r = 0; r < nr; ++r) amax = fmaxf(amax, fabsf(ld_f(src + (r0 + r) * cols + c)));
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(part[0], part[1]), fmaxf(part[2], part[3]));
  const uint32_t code = e8m0_code(amax);
  const float inv = e8m0_inverse(code);
  for (int r = 0; r < nr; ++r)
    codes[(r0 + r) * cols + c] = (uint8_t)(pack_e4m3x4(ld_f(src + (r0 + r) * cols + c) * inv, 0.f, 0.f, 0.f) & 0xFFu);
  if (ATOM) {
    if ((int)threadIdx.x < nr) scales[atom_offset(r0 + threadIdx.x, cb, groups)] = (uint8_t)code;
  } else if (threadIdx.x == 0) {
    scales[blockIdx.y * (cols >> 7) + cb] = (uint8_t)code;
  }
}

// Largest value over the 16 lanes of a half warp: an FP8 [1,128] block, eight elements a lane.
__device__ __forceinline__ float half_warp_max(float a) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  return a;
}

// ---------------------------------------------------------------- MXFP4 ([1,32] blocks)
// eight consecutive elements (16- or 32-byte aligned)
__device__ __forceinline__ void ld8(const __nv_bfloat16* p, float* v) {
  const uint4 r = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void ld8(const float* p, float* v) {
  ld4(p, v);
  ld4(p + 4, v + 4);
}

// The eight values of one lane, its 32-element block spread over four lanes:
// the lane's packed codes (x) and the block's scale code (y, shared by the four lanes).
__device__ __forceinline__ uint2 quant8_mx4(const float* v) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  const uint32_t code = mx4_code(a);
  return make_uint2(pack_e2m1x8(v, e8m0_inverse(code)), code);
}

// src [rows, cols] -> codes [rows, cols/2], scales plain [rows, cols/32] or atoms
// (groups = ceil(cols/128)).  cols a multiple of 256; one warp per 256 elements.
template <typename TIN, bool ATOM>
__global__ void __launch_bounds__(256) k_quant_mx4(const TIN* __restrict__ src, int64_t rows, int cols,
                                                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                   int groups) {
  const int lane = threadIdx.x & 31;
  const int nch = cols >> 8;
  const int64_t nwork = rows * nch;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < nwork; i += nwarps) {
    const int64_t r = i / nch;
    const int c = (int)(i - r * nch) * 256 + lane * 8;
    float v[8];
    ld8(src + r * cols + c, v);
    const uint2 q = quant8_mx4(v);
    *reinterpret_cast<uint32_t*>(codes + r * (cols >> 1) + (c >> 1)) = q.x;
    if ((lane & 3) == 0) scales[ATOM ? atom_offset(r, c >> 5, groups) : r * (cols >> 5) + (c >> 5)] = (uint8_t)q.y;
  }
}

// ---------------------------------------------------------------- NVFP4 ([1,16] blocks, two-level scale)
// The eight values of one lane, its 16-element block shared with the neighbouring lane,
// under tensor scale g: the lane's packed codes (x) and the block's UE4M3 code (y).
__device__ __forceinline__ uint2 quant8_nv4(const float* v, float g) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  const uint32_t code = nv4_code(a, g);
  return make_uint2(pack_e2m1x8(v, nv4_inverse(code, g)), code);
}

// Largest magnitude of each of `nmat` matrices of `mrows` rows x cols (consecutive in src):
// amax_bits[m] (zeroed by the caller) receives it as fp32 bits.  grid (x, nmat).
template <typename TIN>
__global__ void __launch_bounds__(256) k_matrix_amax(const TIN* __restrict__ src, int64_t mrows, int cols,
                                                     uint32_t* __restrict__ amax_bits) {
  __shared__ float part[8];
  const int64_t n = mrows * cols;  // a multiple of 8
  const TIN* base = src + (int64_t)blockIdx.y * n;
  float a = 0.0f;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < n; i += (int64_t)gridDim.x * blockDim.x * 8) {
    float v[8];
    ld8(base + i, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(v[j]));
  }
  a = warp_max(a);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) a = fmaxf(a, part[w]);
    atomicMax(amax_bits + blockIdx.y, __float_as_uint(a));  // non-negative floats order as their bits
  }
}

// amax (as bits) -> the tensor scale g = fl32(amax / 2688) (1 for an all-zero matrix), in place.
__global__ void k_nv4_global(uint32_t* __restrict__ v, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = __uint_as_float(v[i]);
    v[i] = __float_as_uint(a > 0.0f ? __fdiv_rn(a, 2688.0f) : 1.0f);
  }
}

// src [rows, cols] -> codes [rows, cols/2], scales plain [rows, cols/16] or atoms
// (groups = ceil(cols/64)); row r takes tensor scale gvec[r / rows_per_g] (g_const when gvec
// is null).  cols a multiple of 256; one warp per 256 elements.
template <typename TIN, bool ATOM>
__global__ void __launch_bounds__(256) k_quant_nv4(const TIN* __restrict__ src, int64_t rows, int cols,
                                                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                   int groups, const float* __restrict__ gvec, int64_t rows_per_g,
                                                   float g_const) {
  const int lane = threadIdx.x & 31;
  const int nch = cols >> 8;
  const int64_t nwork = rows * nch;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < nwork; i += nwarps) {
    const int64_t r = i / nch;
    const int c = (int)(i - r * nch) * 256 + lane * 8;
    const float g = gvec ? gvec[r / rows_per_g] : g_const;
    float v[8];
    ld8(src + r * cols + c, v);
    const uint2 q = quant8_nv4(v, g);
    *reinterpret_cast<uint32_t*>(codes + r * (cols >> 1) + (c >> 1)) = q.x;
    if ((lane & 1) == 0) scales[ATOM ? atom_offset(r, c >> 4, groups) : r * (cols >> 4) + (c >> 4)] = (uint8_t)q.y;
  }
}

// ---------------------------------------------------------------- the FFN pairs' rows, quantized
// The x rows of the FFN pairs into the padded expert-order operand (pair p of expert e at row
// p - offsets[e] + 128 mb_off[e]), written from the token side: a warp takes one (token, 1024
// columns) item at a time, reads and quantizes it once (the codes and scales depend only on
// the row), then writes them to each of the token's FFN rows.  FMT 0: FP8 E4M3 per [1,128];
// 1: MXFP4 per [1,32]; 2: NVFP4 per [1,16] (g = 1).  d a multiple of 512 (a last item may hold
// 512 columns); lanes hold eight consecutive elements, a warp-wide load 256 columns.
template <int FMT>
__global__ void __launch_bounds__(256) k_scatter_quant(const __nv_bfloat16* __restrict__ x, int d,
                                                       const int32_t* __restrict__ pos,
                                                       const int32_t* __restrict__ idx, int T, int k,
                                                       const int32_t* __restrict__ offsets,
                                                       const int32_t* __restrict__ mb_off,
                                                       uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                       int groups) {
  const int lane = threadIdx.x & 31;
  const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
  const int64_t row_bytes = FMT == 0 ? d : d / 2;
  const int nchunks = (d + 1023) / 1024;
  const int64_t items = (int64_t)T * nchunks;
  for (int64_t it = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
    const int t = (int)(it / nchunks);
    const int c0 = (int)(it - (int64_t)t * nchunks) * 1024;
    int my_pad = -1;  // lane j < k: the padded row of the token's slot j (-1: a zero expert)
    if (lane < k) {
      const int p = pos[(int64_t)t * k + lane];
      if (p >= 0) {
        const int e = idx[(int64_t)t * k + lane];
        my_pad = p - offsets[e] + mb_off[e] * 128;
      }
    }
    const __nv_bfloat16* src = x + (int64_t)t * d;
    {
      const int nu = d - c0 >= 1024 ? 4 : 2;  // d is a multiple of 512: a last 512 columns
      float v[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (u < nu) ld8(src + c0 + 256 * u + lane * 8, v[u]);
      uint2 q[4];       // the lane's codes: FMT 0 eight E4M3 bytes; FP4 eight E2M1 nibbles in x
      uint32_t sc[4];   // the scale code of the lane's block
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (u >= nu) break;
        if (FMT == 0) {
          float m = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[u][i]));
          sc[u] = e8m0_code(half_warp_max(m));
          const float inv = e8m0_inverse(sc[u]);
          q[u] = make_uint2(pack_e4m3x4(v[u][0] * inv, v[u][1] * inv, v[u][2] * inv, v[u][3] * inv),
                            pack_e4m3x4(v[u][4] * inv, v[u][5] * inv, v[u][6] * inv, v[u][7] * inv));
        } else {
          q[u] = FMT == 1 ? quant8_mx4(v[u]) : quant8_nv4(v[u], 1.0f);
          sc[u] = q[u].y;
        }
      }
      for (int j = 0; j < k; ++j) {
        const int pad = __shfl_sync(0xffffffffu, my_pad, j);
        if (pad < 0) continue;
        uint8_t* dst = codes + (int64_t)pad * row_bytes;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (u >= nu) break;
          const int c = c0 + 256 * u + lane * 8;
          if (FMT == 0) {
            *reinterpret_cast<uint2*>(dst + c) = q[u];
            if ((lane & 15) == 0) scales[atom_offset(pad, c >> 7, groups)] = (uint8_t)sc[u];
          } else {
            *reinterpret_cast<uint32_t*>(dst + (c >> 1)) = q[u].x;
            if ((lane & (FMT == 1 ? 3 : 1)) == 0) scales[atom_offset(pad, c >> (FMT == 1 ? 5 : 4), groups)] = (uint8_t)sc[u];
          }
        }
      }
    }
  }
}

// Debug copy: pair p's expert output from its padded row to row p.
__global__ void __launch_bounds__(256) k_unpad_rows(const uint4* __restrict__ ypad, int row_vecs,
                                                    const int32_t* __restrict__ perm, const int32_t* __restrict__ idx,
                                                    const int32_t* __restrict__ offsets,
                                                    const int32_t* __restrict__ mb_off,
                                                    const int32_t* __restrict__ scal, uint4* __restrict__ out) {
  const int P = scal[0];
  const int lane = threadIdx.x & 31;
  const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
  for (int p = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5); p < P; p += nwarps) {
    const int e = idx[perm[p]];
    const int64_t pad = (int64_t)(p - offsets[e]) + (int64_t)mb_off[e] * 128;
    for (int v = lane; v < row_vecs; v += 32) out[(int64_t)p * row_vecs + v] = ypad[pad * row_vecs + v];
  }
}

}  // namespace

cudaError_t launch_unpad_rows(const void* ypad, int row_bytes, const int32_t* perm, const int32_t* idx,
                              const int32_t* offsets, const int32_t* mb_off, const int32_t* scal, void* out, int sms,
                              cudaStream_t s) {
  k_unpad_rows<<<sms * 4, 256, 0, s>>>(static_cast<const uint4*>(ypad), row_bytes / 16, perm, idx, offsets, mb_off,
                                        scal, static_cast<uint4*>(out));
  return cudaGetLastError();
}

cudaError_t launch_quant_rows(int bf16, const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                              int atom_groups, int sms, cudaStream_t s) {
  const int64_t warps = rows * (cols / 128);
  int64_t blocks = (warps + 7) / 8;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  if (blocks < 1) blocks = 1;
  const bool atom = atom_groups > 0;
  if (bf16) {
    auto src_ = static_cast<const __nv_bfloat16*>(src);
    if (atom) k_quant_rows<__nv_bfloat16, true><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, atom_groups);
    else k_quant_rows<__nv_bfloat16, false><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, 0);
  } else {
    auto src_ = static_cast<const float*>(src);
    if (atom) k_quant_rows<float, true><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, atom_groups);
    else k_quant_rows<float, false><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, 0);
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_mx4(int bf16, const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                             int atom_groups, int sms, cudaStream_t s) {
  const int64_t warps = rows * (cols / 256);
  int64_t blocks = (warps + 7) / 8;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  if (blocks < 1) blocks = 1;
  const bool atom = atom_groups > 0;
  if (bf16) {
    auto src_ = static_cast<const __nv_bfloat16*>(src);
    if (atom) k_quant_mx4<__nv_bfloat16, true><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, atom_groups);
    else k_quant_mx4<__nv_bfloat16, false><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, 0);
  } else {
    auto src_ = static_cast<const float*>(src);
    if (atom) k_quant_mx4<float, true><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, atom_groups);
    else k_quant_mx4<float, false><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, 0);
  }
  return cudaGetLastError();
}

cudaError_t launch_scatter_quant(int fmt, const void* x, int d, const int32_t* pos, const int32_t* idx, int T, int k,
                                 const int32_t* offsets, const int32_t* mb_off, uint8_t* codes, uint8_t* scales,
                                 int groups, int sms, cudaStream_t s) {
  const int64_t items = (int64_t)T * ((d + 1023) / 1024);  // one warp per (token, 1024 columns)
  int64_t blocks = (items + 7) / 8;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  if (blocks < 1) blocks = 1;
  auto x_ = static_cast<const __nv_bfloat16*>(x);
  if (fmt == 0)
    k_scatter_quant<0><<<(int)blocks, 256, 0, s>>>(x_, d, pos, idx, T, k, offsets, mb_off, codes, scales, groups);
  else if (fmt == 1)
    k_scatter_quant<1><<<(int)blocks, 256, 0, s>>>(x_, d, pos, idx, T, k, offsets, mb_off, codes, scales, groups);
  else if (fmt == 2)
    k_scatter_quant<2><<<(int)blocks, 256, 0, s>>>(x_, d, pos, idx, T, k, offsets, mb_off, codes, scales, groups);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_nv4_global(int bf16, const void* src, int nmat, int64_t mrows, int cols, float* g,
                              cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(g, 0, (size_t)nmat * sizeof(float), s);
  if (e != cudaSuccess) return e;
  int64_t bx = mrows * cols / (256 * 8 * 16);  // ~16 vectors of 8 per thread
  if (bx < 1) bx = 1;
  if (bx > 64) bx = 64;
  const dim3 grid((unsigned)bx, (unsigned)nmat);
  uint32_t* bits = reinterpret_cast<uint32_t*>(g);
  if (bf16) k_matrix_amax<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src), mrows, cols, bits);
  else k_matrix_amax<float><<<grid, 256, 0, s>>>(static_cast<const float*>(src), mrows, cols, bits);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_nv4_global<<<(nmat + 255) / 256, 256, 0, s>>>(bits, nmat);
  return cudaGetLastError();
}

cudaError_t launch_quant_nv4(int bf16, const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                             int atom_groups, const float* gvec, int64_t rows_per_g, float g_const, int sms,
                             cudaStream_t s) {
  const int64_t warps = rows * (cols / 256);
  int64_t blocks = (warps + 7) / 8;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  if (blocks < 1) blocks = 1;
  const bool atom = atom_groups > 0;
  if (bf16) {
    auto src_ = static_cast<const __nv_bfloat16*>(src);
    if (atom)
      k_quant_nv4<__nv_bfloat16, true>
          <<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, atom_groups, gvec, rows_per_g, g_const);
    else
      k_quant_nv4<__nv_bfloat16, false><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, 0, gvec, rows_per_g, g_const);
  } else {
    auto src_ = static_cast<const float*>(src);
    if (atom)
      k_quant_nv4<float, true><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, atom_groups, gvec, rows_per_g, g_const);
    else
      k_quant_nv4<float, false><<<(int)blocks, 256, 0, s>>>(src_, rows, cols, codes, scales, 0, gvec, rows_per_g, g_const);
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_tiles(int bf16, const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                               int atom_groups, cudaStream_t s) {
  const dim3 grid(cols / 128, (unsigned)((rows + 127) / 128));
  const bool atom = atom_groups > 0;
  if (bf16) {
    auto src_ = static_cast<const __nv_bfloat16*>(src);
    if (atom) k_quant_tiles<__nv_bfloat16, true><<<grid, 128, 0, s>>>(src_, rows, cols, codes, scales, atom_groups);
    else k_quant_tiles<__nv_bfloat16, false><<<grid, 128, 0, s>>>(src_, rows, cols, codes, scales, 0);
  } else {
    auto src_ = static_cast<const float*>(src);
    if (atom) k_quant_tiles<float, true><<<grid, 128, 0, s>>>(src_, rows, cols, codes, scales, atom_groups);
    else k_quant_tiles<float, false><<<grid, 128, 0, s>>>(src_, rows, cols, codes, scales, 0);
  }
  return cudaGetLastError();
}

}  // namespace zc
