// fp32 grouped GEMM on the CUDA cores, for layers kept entirely in fp32 (no
// TF32 anywhere, so results stay within ~1e-6 relative of fp64).  Same three
// contractions and the same expert/row-block bookkeeping as the tensor-core
// kernel: router logits (+ offset), gate/up with SwiGLU, down projection.
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_internal.h"

namespace zc {
namespace {

constexpr int SBM = kBM;  // 128 rows per block (same row blocks as the integer stage)
constexpr int SBN = 32;   // output columns per block
constexpr int SBK = 32;   // k slice

template <int MODE>
__global__ void __launch_bounds__(256) k_simt_gemm(const SimtArgs a) {
  __shared__ float sA[SBK][SBM + 1];
  __shared__ float sB0[SBK][SBN + 1];
  __shared__ float sB1[SBK][SBN + 1];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const int mb = blockIdx.y;
  int a_row, rows_valid, b_row0, b_rows_end;
  if (MODE == kRouter) {
    a_row = mb * SBM;
    if (a_row >= a.M) return;
    rows_valid = min(SBM, a.M - a_row);
    b_row0 = 0;
    b_rows_end = a.n_out;
  } else {
    if (mb >= a.mb_off[a.ngroups]) return;
    int lo = 0, hi = a.ngroups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.mb_off[mid] <= mb) lo = mid;
      else hi = mid - 1;
    }
    const int g = lo;
    a_row = a.row_off[g] + (mb - a.mb_off[g]) * SBM;
    rows_valid = min(SBM, a.row_off[g + 1] - a_row);
    b_row0 = g * a.b_rows_per_group;
    b_rows_end = b_row0 + a.n_out;
  }
  const int col0 = blockIdx.x * SBN;
  float acc0[16], acc1[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc0[i] = acc1[i] = 0.0f;
  for (int k0 = 0; k0 < a.K; k0 += SBK) {
    // A tile: 128 rows x 32 k (16 per thread), zero outside the tile's rows / K
    for (int i = threadIdx.x; i < SBM * SBK; i += 256) {
      const int r = i / SBK, kk = i % SBK;
      float v = 0.0f;
      if (r < rows_valid && k0 + kk < a.K) v = a.A[(int64_t)(a_row + r) * a.K + k0 + kk];
      sA[kk][r] = v;
    }
    for (int i = threadIdx.x; i < SBN * SBK; i += 256) {
      const int c = i / SBK, kk = i % SBK;
      const int br = b_row0 + col0 + c;
      float v0 = 0.0f, v1 = 0.0f;
      if (br < b_rows_end && k0 + kk < a.K) {
        v0 = a.B0[(int64_t)br * a.K + k0 + kk];
        if (MODE == kGateUp) v1 = a.B1[(int64_t)br * a.K + k0 + kk];
      }
      sB0[kk][c] = v0;
      sB1[kk][c] = v1;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < SBK; ++kk) {
      const float b0 = sB0[kk][tx];
      const float b1 = sB1[kk][tx];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float av = sA[kk][ty + 8 * i];
        acc0[i] = __fmaf_rn(av, b0, acc0[i]);
        if (MODE == kGateUp) acc1[i] = __fmaf_rn(av, b1, acc1[i]);
      }
    }
    __syncthreads();
  }
  const int col = col0 + tx;
  if (col >= a.n_out) return;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = ty + 8 * i;
    if (r >= rows_valid) continue;
    float v = acc0[i];
    if (MODE == kGateUp) v = v / (1.0f + expf(-v)) * acc1[i];
    if (MODE == kRouter && a.col_add) v = v + a.col_add[col];
    a.out[(int64_t)(a_row + r) * a.ldo + col] = v;
  }
}

}  // namespace

cudaError_t launch_simt_gemm(int mode, const SimtArgs& args, int max_mblocks, cudaStream_t s) {
  dim3 grid((args.n_out + SBN - 1) / SBN, max_mblocks);
  switch (mode) {
    case kRouter:
      k_simt_gemm<kRouter><<<grid, 256, 0, s>>>(args);
      break;
    case kGateUp:
      k_simt_gemm<kGateUp><<<grid, 256, 0, s>>>(args);
      break;
    case kDown:
      k_simt_gemm<kDown><<<grid, 256, 0, s>>>(args);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace zc
