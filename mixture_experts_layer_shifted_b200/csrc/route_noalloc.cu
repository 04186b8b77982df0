// zcmoe_route_noalloc: the routing stage (softmax + bias-shifted top-k + the
// integer stage) for callers that must not allocate device memory.
//
// Who needs this: code that runs under a framework's memory pool or a fixed
// device-memory budget (a raw cudaMalloc would bypass the pool or break the
// budget), and latency-critical loops that cannot afford cudaMalloc/cudaFree,
// which may synchronise the whole device.  Such a caller still owns and passes
// every input and output buffer; the only extra memory the routing stage needs
// (per-block expert counts, block offsets, small counters) lives in the fixed
// array below, which the library reserves when it is loaded.
//
// The regular path (zcmoe_forward) is unchanged and keeps its scratch in the
// handle's workspace; this file only adds a second way in.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <cmath>
#include <mutex>

#include "../../include/zcmoe.h"
#include "zc_internal.h"

namespace {

// 1 MiB of device memory, reserved on every GPU that loads the library, kept
// until the process exits.  Layout per call: per-block counts (ceil(T/256) x E
// int32), then 8-byte aligned: E int64 count accumulators + 1 int64 token
// counter, then (N+1) int32 row-block offsets and 4 int32 scalars.
constexpr size_t kScratchBytes = size_t(1) << 20;
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

// Message buffer; copied into the library's last-error slot on failure.
thread_local char g_msg[256] = "";

int report(int code) {
  zc::set_last_error(g_msg);
  return code;
}

// Device address of g_route_scratch, looked up with the device current (the
// host-side symbol is only a stand-in and must never be handed to a kernel) and
// cached per device together with the context it was looked up in.  A new
// primary context (after cudaDeviceReset) reloads the module, which can move the
// array, so a changed context triggers a fresh lookup.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
std::mutex g_mu;
struct ScratchSlot {
  CUcontext ctx;
  void* addr;
};
ScratchSlot g_slot[128] = {};
CtxGetCurrentFn g_ctx_fn = nullptr;
std::once_flag g_ctx_once;

int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof(g_msg), "cudaGetDevice: %s", cudaGetErrorString(e));
    return report(ZCMOE_ECUDA);
  }
  if (dev < 0 || dev >= 128) {
    snprintf(g_msg, sizeof(g_msg), "device ordinal %d out of range", dev);
    return report(ZCMOE_EUNSUPPORTED);
  }
  std::call_once(g_ctx_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  if (!g_ctx_fn) {
    snprintf(g_msg, sizeof(g_msg), "cuCtxGetCurrent entry point unavailable");
    return report(ZCMOE_ECUDA);
  }
  // Before this thread's first runtime call that needs a context there is none
  // current yet: the lookup below binds the primary context, then it is read.
  CUcontext ctx = nullptr;
  if (g_ctx_fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!ctx || !g_slot[dev].addr || g_slot[dev].ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p) {
      snprintf(g_msg, sizeof(g_msg), "cudaGetSymbolAddress(route scratch): %s", cudaGetErrorString(e));
      return report(ZCMOE_ECUDA);
    }
    if (g_ctx_fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    g_slot[dev].ctx = ctx;
    g_slot[dev].addr = p;
  }
  *out = g_slot[dev].addr;
  return ZCMOE_OK;
}

size_t align8(size_t x) { return (x + 7) & ~size_t(7); }

// Scratch layout of one call: per-block counts, then (8-byte aligned) the count
// accumulators and token counter, the row-block offsets and four scalars.
struct Layout {
  size_t off_acc, off_mb, off_scal, need;
};
Layout layout(int nchunks, int N, int E) {
  Layout l;
  l.off_acc = align8((size_t)nchunks * E * sizeof(int32_t));
  l.off_mb = l.off_acc + (size_t)(E + 1) * sizeof(int64_t);
  l.off_scal = l.off_mb + (size_t)(N + 1) * sizeof(int32_t);
  l.need = l.off_scal + 4 * sizeof(int32_t);
  return l;
}

// The largest T whose layout fits the array (a multiple of the 256-token block).
int64_t max_tokens(int N, int E) {
  const Layout l0 = layout(0, N, E);
  int64_t nb = (int64_t)((kScratchBytes - l0.need) / ((size_t)E * sizeof(int32_t)));
  // the 8-byte alignment of the first region adds at most 4 bytes: one step back at most
  for (int i = 0; i < 2 && nb > 0 && layout((int)nb, N, E).need > kScratchBytes; ++i) --nb;
  return nb * zc::kChunk;
}

}  // namespace

extern "C" {

int zcmoe_route_noalloc(const float* logits, const float* bias, int64_t T, int32_t n_ffn, int32_t n_zero,
                        int32_t top_k, float routed_scale, int32_t* idx, float* gate, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* pos, cudaStream_t stream) {
  g_msg[0] = 0;
  zc::set_last_error("");
  const int N = n_ffn, Z = n_zero, E = n_ffn + n_zero, k = top_k;
  if (N < 1 || Z < 0 || E > 1024 || k < 1 || k > E || k > 32) {
    snprintf(g_msg, sizeof(g_msg), "need 1 <= n_ffn, n_ffn + n_zero <= 1024, 1 <= top_k <= min(E, 32)");
    return report(ZCMOE_EINVAL);
  }
  if (!std::isfinite(routed_scale)) {
    snprintf(g_msg, sizeof(g_msg), "routed_scale must be finite");
    return report(ZCMOE_EINVAL);
  }
  if (T < 0 || T > (1 << 20)) {
    snprintf(g_msg, sizeof(g_msg), "T=%lld outside [0, 2^20]", (long long)T);
    return report(ZCMOE_ERANGE);
  }
  if (T == 0) return ZCMOE_OK;
  if (!logits || !bias || !idx || !gate || !counts || !offsets || !perm || !pos) {
    snprintf(g_msg, sizeof(g_msg), "a pointer argument is NULL");
    return report(ZCMOE_EINVAL);
  }
  const int Ti = (int)T;
  const int nchunks = (Ti + zc::kChunk - 1) / zc::kChunk;
  const Layout lay = layout(nchunks, N, E);
  if (lay.need > kScratchBytes) {
    snprintf(g_msg, sizeof(g_msg),
             "T=%d with %d experts (%d FFN) needs %zu bytes of routing scratch; the fixed scratch holds %zu, "
             "enough for T <= %lld",
             Ti, E, N, lay.need, kScratchBytes, (long long)max_tokens(N, E));
    return report(ZCMOE_ERANGE);
  }
  void* base = nullptr;
  int rc = scratch_address(&base);
  if (rc != ZCMOE_OK) return rc;
  unsigned char* s = static_cast<unsigned char*>(base);
  int32_t* chunk = reinterpret_cast<int32_t*>(s);
  int64_t* acc = reinterpret_cast<int64_t*>(s + lay.off_acc);
  int32_t* mb_off = reinterpret_cast<int32_t*>(s + lay.off_mb);
  int32_t* scal = reinterpret_cast<int32_t*>(s + lay.off_scal);

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

  // The count accumulators are added to by the scan kernel: they start at zero
  // on every call (the array keeps whatever the previous call left).
  cudaError_t e = cudaMemsetAsync(acc, 0, (size_t)(E + 1) * sizeof(int64_t), stream);
  if (e == cudaSuccess)
    e = zc::launch_softmax_topk(logits, bias, Ti, E, k, routed_scale, idx, gate, nullptr, sms, stream);
  if (e == cudaSuccess) e = zc::launch_route_count(idx, Ti, k, E, chunk, stream);
  if (e == cudaSuccess)
    e = zc::launch_route_scan(chunk, nchunks, Ti, N, E, counts, offsets, mb_off, scal, acc, acc + E, stream);
  if (e == cudaSuccess) e = zc::launch_route_scatter(idx, Ti, k, N, E, chunk, perm, pos, stream);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof(g_msg), "routing launch failed: %s", cudaGetErrorString(e));
    return report(ZCMOE_ECUDA);
  }
  return ZCMOE_OK;
}

}  // extern "C"
