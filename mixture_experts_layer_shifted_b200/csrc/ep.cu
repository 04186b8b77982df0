// Expert parallelism: the row regrouping around the local experts' GEMMs.
//
// LongCat-Flash technical summary (zhangjingwei.cn), 五 訓練基礎設施: the FFN layers
// are partitioned by expert (EP groups, no tensor parallelism); the dispatch sends
// each (token, FFN expert) row to the rank that holds the expert, the combine
// brings the expert output back.  Zero-computation experts need no weights, so
// their picks never leave the token's rank.
//
// Rows arrive from the source ranks in rank order, each source's rows grouped by
// the receiving rank's local experts: segment (s, e) = the rows source s sent for
// local expert e, segments ordered s-major.  The grouped GEMM wants them e-major
// (all of expert e's rows together, so the row blocks of an expert share its
// weight tiles through L2), sources in order within an expert.  k_ep_regroup moves
// row q of segment (s, e) to row seg_dst[(s, e)] + (q - seg_src[(s, e)]) (or back).
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_internal.h"

namespace zc {
namespace {

// One warp per row; seg_src [nseg + 1] are the s-major segment starts (non-decreasing,
// seg_src[nseg] = P), seg_dst [nseg] the e-major starts.  inverse: copy back.
__global__ void __launch_bounds__(256) k_ep_regroup(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                    int64_t P, int row_vecs, const int32_t* __restrict__ seg_src,
                                                    const int32_t* __restrict__ seg_dst, int nseg, int inverse) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < P; q += nwarps) {
    // the first segment whose end lies past q holds q (empty segments end where they start)
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (seg_src[mid + 1] > q) hi = mid;
      else lo = mid + 1;
    }
    const int64_t r = (int64_t)seg_dst[lo] + (q - seg_src[lo]);
    const uint4* a = src + (inverse ? r : q) * row_vecs;
    uint4* b = dst + (inverse ? q : r) * row_vecs;
    for (int v = lane; v < row_vecs; v += 32) b[v] = a[v];
  }
}

}  // namespace

cudaError_t launch_ep_regroup(const void* src, void* dst, int64_t P, int row_bytes, const int32_t* seg_src,
                              const int32_t* seg_dst, int nseg, int inverse, int sms, cudaStream_t s) {
  if (P <= 0) return cudaSuccess;
  k_ep_regroup<<<sms * 8, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), P, row_bytes / 16,
                                       seg_src, seg_dst, nseg, inverse);
  return cudaGetLastError();
}

}  // namespace zc
