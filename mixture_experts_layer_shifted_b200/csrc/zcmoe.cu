// C ABI of the zero-computation-expert MoE layer (declared in include/zcmoe.h).
//
// A forward pass is a fixed sequence of kernels on the caller's stream, with no
// host synchronisation and no host-visible intermediate:
//   router GEMM (+ logit offset)      -> logits [T, E] fp32
//   softmax + bias-shifted top-k      -> idx, gate [T, k]
//   integer stage (count, scan, scatter) -> counts, offsets, row blocks, perm, pos
//   row gather                        -> X_perm [P, d]
//   grouped gate/up GEMM + SwiGLU     -> H [P, inter]
//   grouped down GEMM                 -> Y [P, d]
//   combine (zero experts as identity terms) -> y [T, d]
// Every size that depends on the routing (P, row blocks) stays on the device;
// the persistent GEMM kernels read it there.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <cmath>
#include <cstdarg>
#include <mutex>
#include <new>
#include <unordered_set>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/zcmoe.h"
#include "zc_fp8.cuh"
#include "zc_internal.h"

namespace {

thread_local char g_err[512] = "";

// Live handles, so that a destroyed or foreign handle is rejected instead of
// being dereferenced.
std::mutex g_live_mu;
std::unordered_set<const void*> g_live;        // zcmoe_t
std::unordered_set<const void*> g_live_dense;  // zcmoe_dense_t

bool is_live(const void* h) {
  std::lock_guard<std::mutex> lk(g_live_mu);
  return h && g_live.count(h) != 0;
}
bool is_live_dense(const void* h) {
  std::lock_guard<std::mutex> lk(g_live_mu);
  return h && g_live_dense.count(h) != 0;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

#define ZC_CUDA(call)                                                                               \
  do {                                                                                             \
    cudaError_t e_ = (call);                                                                       \
    if (e_ != cudaSuccess) return fail(ZCMOE_ECUDA, "%s: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                                       __FILE__, __LINE__);                                       \
  } while (0)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once for the process (call_once makes
// the first lookup safe when several threads create or run layers at once).
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D tensor [outer, inner] (inner contiguous) of bf16 (esz 2) or FP8 codes
// (esz 1); box [box_outer, 128 bytes], 128-byte swizzle.
int make_tmap_esz(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer, int esz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(ZCMOE_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return fail(ZCMOE_EINVAL, "tensor base not 16-byte aligned");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * (uint64_t)esz};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esz), box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ZCMOE_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ZCMOE_OK;
}
// bf16 [outer, inner], box 32 x 32, no swizzle: a store target for 32-row x 32-column boxes
int make_tmap_store32(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(ZCMOE_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return fail(ZCMOE_EINVAL, "tensor base not 16-byte aligned");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ZCMOE_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ZCMOE_OK;
}
int make_tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  return make_tmap_esz(tm, base, inner, outer, box_outer, 2);
}
// fp32 gradient accumulator [groups][rows][cols] as a 3-D tensor, box 32 x 32 x 1,
// 128-byte swizzle: the target of the backward's TMA reduce-adds (cols a multiple of 4)
int make_tmap_acc(CUtensorMap* tm, const float* base, uint64_t cols, uint64_t rows, uint64_t groups) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(ZCMOE_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return fail(ZCMOE_EINVAL, "gradient not 16-byte aligned");
  cuuint64_t dims[3] = {cols, rows, groups};
  cuuint64_t strides[2] = {cols * 4, cols * rows * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ZCMOE_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ZCMOE_OK;
}
// bf16 [outer, inner] with a row stride of ld elements (ld >= inner, ld * 2 a multiple of 16)
int make_tmap_ld(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer, uint64_t ld) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(ZCMOE_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ZCMOE_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ZCMOE_OK;
}

template <typename T>
int dalloc(T** p, size_t n) {
  *p = nullptr;
  if (n == 0) n = 1;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), n * sizeof(T));
  if (e != cudaSuccess) {
    *p = nullptr;
    cudaGetLastError();
    return fail(ZCMOE_ENOMEM, "cudaMalloc(%zu bytes) failed: %s", n * sizeof(T), cudaGetErrorString(e));
  }
  return ZCMOE_OK;
}

}  // namespace

namespace zc {
void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }
}  // namespace zc

struct zcmoe_s {
  zcmoe_config cfg;
  int E, N, Z, k, d, inter, max_T, bf16, sms, device;
  int max_chunks, max_pairs, max_mblocks;
  zcmoe_weights w;
  // controller state
  float *bias, *b0, *offset, *eta, *integ, *eprev;
  int64_t *acc_counts, *acc_tokens;  // acc_tokens = acc_counts + E (one buffer, E+1 entries)
  int* err;
  // workspace
  float *logits, *gate;
  int32_t *idx, *pos, *counts, *offsets, *mb_off, *scal, *chunk, *perm;
  int32_t* sp_off;  // [N+1] row-block pairs per expert, prefix (the grouped GEMM's work units)
  int* sched;       // [4] unit counters of the tensor-core GEMM launches (router, gate/up, down)
  void *xperm, *H, *Y;
  // zcmoe_forward_host: x staged through two device buffers filled on an internal
  // copy stream, so the next call's upload overlaps this call's compute; y staged once
  // zcmoe_forward_host(_async): x and y staged through two device buffers each; uploads on
  // copy_stream, downloads on d2h_stream, so a call's copies overlap its neighbours' forwards
  void *stage_x, *stage_x2, *stage_y, *stage_y2;
  cudaStream_t copy_stream, d2h_stream;
  cudaEvent_t ev_in[2], ev_used[2], ev_fwd[2], ev_ydone[2];
  long long host_calls;
  // stage timing (zcmoe_profile_begin/end): ZCMOE_NUM_STAGES + 1 events per forward
  bool profiling;
  std::vector<cudaEvent_t>* events;
  // tensor maps of fixed buffers
  CUtensorMap tm_wr, tm_wr_n, tm_wg, tm_wu, tm_wd, tm_xperm, tm_h, tm_y;  // tm_wr_n: W_r in 32-row boxes
  // ZCMOE_FP8: expert weights as E4M3 codes + scale atoms (owned), padded
  // activation operands (expert e's pairs from row 128 mb_off[e] on) with their
  // scale atoms, padded expert outputs; atoms per 128 rows: gd (K = d), gi (K = inter)
  int fp8, fmt, gd, gi;  // fp8: block-scaled experts (ZCMOE_FP8, _FP4, _NVFP4); fmt 1 MXFP4, 2 NVFP4
  uint8_t *w8g, *w8u, *w8d, *sfg, *sfu, *sfd, *x8, *sx, *h8, *sh;
  float* gsc;  // NVFP4: the fp32 tensor scales of W_g [N], W_u [N], W_d [N], one per expert matrix
  void* ypad;
  CUtensorMap tm8_wg, tm8_wu, tm8_wd, tm8_x, tm8_h, tm8_y;  // tm8_y: the down GEMM's store target (ypad)
  // zcmoe_backward (allocated on its first call): padded X, dY, dH, [dG|dU], H, dX
  // rows; dg [T*k]; dl [T, dl_ld] bf16; router dx [T, d]; the router's one-group offsets
  int last_T;
  int dl_ld;
  void *b_xpad, *b_dypad, *b_dh, *b_dgu, *b_hpad, *b_dxp, *b_dl, *b_dxr;
  float* b_dg;
  int32_t* b_grp;
  // zcmoe_save_for_backward: the forward's [G | U] in padded rows; last_saved tells whether
  // the last forward wrote it
  void* b_gu;
  bool last_saved;
  // expert parallelism (zcmoe_create_ep): the handle holds FFN experts [ep_rank * n_local,
  // (ep_rank + 1) * n_local); xperm / H / Y have rows_cap rows (the routed pairs of max_T
  // tokens, or the rows received from all ranks, whichever is larger).  ep_meta (device) and
  // ep_meta_host (pinned): seg_src [nseg + 1], seg_dst [nseg], exp_off [n_local + 1],
  // mb_off [n_local + 1], sp_off [n_local + 1] of the last zcmoe_ep_experts, nseg = ep_size * n_local
  int ep_rank, ep_size, n_local;
  int64_t rows_cap;
  int32_t *ep_meta, *ep_meta_host;
  cudaEvent_t ep_meta_ev;
  bool ep_meta_pending;
  bool alive;
};

static void release(zcmoe_s* h) {
  void* ptrs[] = {h->bias,  h->b0,     h->offset, h->eta,   h->integ,   h->eprev,  h->acc_counts,
                  h->err,   h->logits, h->gate,   h->idx,   h->pos,     h->counts, h->offsets,
                  h->mb_off, h->scal,  h->chunk,  h->perm,  h->xperm,   h->H,      h->Y,  h->sp_off, h->sched,
                  h->stage_x, h->stage_x2, h->stage_y, h->stage_y2, h->w8g, h->w8u, h->w8d, h->sfg, h->sfu, h->sfd, h->gsc,
                  h->x8, h->sx, h->h8, h->sh, h->ypad, h->b_xpad, h->b_dypad, h->b_dh, h->b_dgu, h->b_hpad,
                  h->b_dxp, h->b_dl, h->b_dxr, h->b_dg, h->b_grp, h->b_gu, h->ep_meta};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  if (h->ep_meta_host) cudaFreeHost(h->ep_meta_host);
  if (h->ep_meta_ev) cudaEventDestroy(h->ep_meta_ev);
  for (int i = 0; i < 2; ++i) {
    cudaEvent_t evs[4] = {h->ev_in[i], h->ev_used[i], h->ev_fwd[i], h->ev_ydone[i]};
    for (cudaEvent_t e : evs)
      if (e) cudaEventDestroy(e);
  }
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  if (h->d2h_stream) cudaStreamDestroy(h->d2h_stream);
  if (h->events) {
    for (cudaEvent_t e : *h->events) cudaEventDestroy(e);
    delete h->events;
    h->events = nullptr;
  }
}

// ---------------------------------------------------------------- dense FFN path
// y = W_down (silu(W_gate x) * (W_up x)) through the same grouped tensor-core
// GEMM as the experts, with one group holding all T rows.
struct zcmoe_dense_s {
  int d, inter, max_T, sms;
  zcmoe_dense_weights w;
  void* H;           // [max_T, inter] bf16
  int32_t* offs;     // one group: row_off[2], mb_off[2], sp_off[2] (written per call); then the
                     // GEMMs' unit counters [2]
  int* err;          // bounded-wait error word of the dense kernels
  cudaStream_t side; // zcmoe_forward_overlap enqueues the dense FFN here
  cudaEvent_t ev_router, ev_down, ev_join;
  CUtensorMap tm_wg, tm_wu, tm_wd, tm_h;
};

static void release_dense(zcmoe_dense_s* h) {
  void* ptrs[] = {h->H, h->offs, h->err};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  cudaEvent_t evs[] = {h->ev_router, h->ev_down, h->ev_join};
  for (cudaEvent_t e : evs)
    if (e) cudaEventDestroy(e);
  if (h->side) cudaStreamDestroy(h->side);
}

// gate/up GEMM with the SwiGLU epilogue: H[:T] = silu(x W_g^T) * (x W_u^T), bf16
static int dense_gate_up(zcmoe_dense_s* h, const void* x, int T, cudaStream_t s) {
  CUtensorMap tm_x;
  int rc = make_tmap(&tm_x, x, (uint64_t)h->d, (uint64_t)T, 128);
  if (rc != ZCMOE_OK) return rc;
  ZC_CUDA(zc::launch_single_group(h->offs, h->offs + 2, T, s, h->offs + 4));
  zc::TcArgs a{};
  a.K = h->d;
  a.n_out = h->inter;
  a.nblocks = (h->inter + zc::tc_block_n(zc::kGateUp) - 1) / zc::tc_block_n(zc::kGateUp);
  a.ngroups = 1;
  a.row_off = h->offs;
  a.mb_off = h->offs + 2;
  a.sp_off = h->offs + 4;
  a.sched = h->offs + 6;
  a.pair = zc::tc_pair_for_rows(T);
  a.b_rows_per_group = h->inter;
  a.out = h->H;
  a.ldo = h->inter;
  a.err = h->err;
  const int tiles = ((T + zc::kBM - 1) / zc::kBM) * a.nblocks;
  ZC_CUDA(zc::launch_tc_gemm(zc::kGateUp, tm_x, h->tm_wg, h->tm_wu, h->tm_wu, a, tiles < h->sms ? tiles : h->sms, s));
  return ZCMOE_OK;
}

// down GEMM: y = H[:T] W_d^T, bf16
static int dense_down(zcmoe_dense_s* h, int T, void* y, cudaStream_t s) {
  zc::TcArgs b{};
  b.K = h->inter;
  b.n_out = h->d;
  b.nblocks = (h->d + zc::tc_block_n(zc::kDown) - 1) / zc::tc_block_n(zc::kDown);
  b.ngroups = 1;
  b.row_off = h->offs;
  b.mb_off = h->offs + 2;
  b.sp_off = h->offs + 4;
  b.sched = h->offs + 7;
  b.pair = zc::tc_pair_for_rows(T);
  b.b_rows_per_group = h->d;
  b.out = y;
  b.ldo = h->d;
  b.err = h->err;
  const int tiles = ((T + zc::kBM - 1) / zc::kBM) * b.nblocks;
  CUtensorMap tm_y;
  const int rc = make_tmap(&tm_y, y, (uint64_t)h->d, (uint64_t)T, 32);
  if (rc != ZCMOE_OK) return rc;
  ZC_CUDA(zc::launch_tc_gemm(zc::kDown, h->tm_h, h->tm_wd, h->tm_wd, tm_y, b, tiles < h->sms ? tiles : h->sms, s));
  return ZCMOE_OK;
}

// The dense FFN enqueued beside a MoE forward (zcmoe_forward_overlap).
struct DenseSide {
  zcmoe_dense_s* dn;
  const void* x;
  void* y;
};

extern "C" {

const char* zcmoe_last_error(void) { return g_err; }

static int create_impl(const zcmoe_config* cfg, const zcmoe_weights* w, int ep_rank, int ep_size,
                       int64_t max_recv_rows, zcmoe_t* out) {
  g_err[0] = 0;
  if (!out) return fail(ZCMOE_EINVAL, "out is NULL");
  *out = nullptr;
  if (!cfg || !w) return fail(ZCMOE_EINVAL, "cfg or weights is NULL");
  const int N = cfg->n_ffn, Z = cfg->n_zero, E = N + Z, k = cfg->top_k;
  if (ep_size < 1 || ep_rank < 0 || ep_rank >= ep_size) return fail(ZCMOE_EINVAL, "need 0 <= ep_rank < ep_size");
  if (N % ep_size) return fail(ZCMOE_EINVAL, "n_ffn must be a multiple of ep_size");
  if (ep_size > 1 && cfg->dtype != ZCMOE_BF16) return fail(ZCMOE_EUNSUPPORTED, "expert parallelism needs a bf16 layer");
  if (max_recv_rows < 0 || max_recv_rows >= (int64_t)1 << 31) return fail(ZCMOE_EINVAL, "bad max_recv_rows");
  const int NL = N / ep_size;  // FFN experts this handle holds
  if (N < 1 || Z < 0 || E > 1024) return fail(ZCMOE_EINVAL, "need 1 <= n_ffn and n_ffn + n_zero <= 1024");
  if (k < 1 || k > E || k > 32) return fail(ZCMOE_EINVAL, "need 1 <= top_k <= min(E, 32)");
  if (cfg->d < 64 || cfg->d % 64 || cfg->inter < 64 || cfg->inter % 64)
    return fail(ZCMOE_EINVAL, "d and inter must be positive multiples of 64");
  if (cfg->max_tokens < 1 || cfg->max_tokens > (1 << 20)) return fail(ZCMOE_EINVAL, "need 1 <= max_tokens <= 2^20");
  if (cfg->dtype != ZCMOE_F32 && cfg->dtype != ZCMOE_BF16 && cfg->dtype != ZCMOE_FP8 && cfg->dtype != ZCMOE_FP4 &&
      cfg->dtype != ZCMOE_NVFP4)
    return fail(ZCMOE_EINVAL, "unknown dtype");
  if (cfg->dtype == ZCMOE_FP8 && (cfg->d % 512 || cfg->inter % 128))
    return fail(ZCMOE_EINVAL, "FP8 experts need d a multiple of 512 and inter a multiple of 128");
  if ((cfg->dtype == ZCMOE_FP4 || cfg->dtype == ZCMOE_NVFP4) && (cfg->d % 512 || cfg->inter % 256))
    return fail(ZCMOE_EINVAL, "W4A4 experts need d a multiple of 512 and inter a multiple of 256");
  if (!w->w_router || !w->w_gate || !w->w_up || !w->w_down) return fail(ZCMOE_EINVAL, "a weight pointer is NULL");
  const void* wp[4] = {w->w_router, w->w_gate, w->w_up, w->w_down};
  for (const void* p : wp)
    if (reinterpret_cast<uintptr_t>(p) & 15u) return fail(ZCMOE_EINVAL, "weight pointers must be 16-byte aligned");
  if ((int64_t)cfg->max_tokens * k >= (int64_t)1 << 31) return fail(ZCMOE_EINVAL, "max_tokens * top_k too large");
  if (!std::isfinite(cfg->routed_scale)) return fail(ZCMOE_EINVAL, "routed_scale must be finite");

  int dev = 0;
  ZC_CUDA(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  ZC_CUDA(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10) return fail(ZCMOE_EUNSUPPORTED, "device %d is sm_%d%d; this library targets sm_100a", dev,
                                    prop.major, prop.minor);
  if (cfg->dtype != ZCMOE_F32 &&
      prop.sharedMemPerBlockOptin < (size_t)(zc::tc_smem_bytes() > zc::fp8_smem_bytes() ? zc::tc_smem_bytes()
                                                                                         : zc::fp8_smem_bytes()))
    return fail(ZCMOE_EUNSUPPORTED, "not enough shared memory per block");

  zcmoe_s* h = new (std::nothrow) zcmoe_s();
  if (!h) return fail(ZCMOE_ENOMEM, "host allocation failed");
  memset(h, 0, sizeof(*h));
  h->cfg = *cfg;
  h->cfg.init_bias = nullptr;
  h->cfg.logit_offset = nullptr;
  h->E = E;
  h->N = N;
  h->Z = Z;
  h->k = k;
  h->d = cfg->d;
  h->inter = cfg->inter;
  h->max_T = cfg->max_tokens;
  h->bf16 = cfg->dtype != ZCMOE_F32;  // ZCMOE_FP8 / _FP4 / _NVFP4 layers are bf16 at the interface
  h->fp8 = cfg->dtype == ZCMOE_FP8 || cfg->dtype == ZCMOE_FP4 || cfg->dtype == ZCMOE_NVFP4;
  h->fmt = cfg->dtype == ZCMOE_FP4 ? 1 : cfg->dtype == ZCMOE_NVFP4 ? 2 : 0;
  h->sms = prop.multiProcessorCount;
  h->device = dev;
  h->w = *w;
  h->max_chunks = (h->max_T + zc::kChunk - 1) / zc::kChunk;
  h->max_pairs = h->max_T * k;
  h->max_mblocks = (h->max_pairs + zc::kBM - 1) / zc::kBM + N;
  h->ep_rank = ep_rank;
  h->ep_size = ep_size;
  h->n_local = NL;
  h->rows_cap = max_recv_rows > h->max_pairs ? max_recv_rows : (int64_t)h->max_pairs;
  const size_t esz = h->bf16 ? 2 : 4;
  const size_t rcap = (size_t)h->rows_cap;

  int rc = ZCMOE_OK;
#define ZC_ALLOC(p, n)                     \
  if (rc == ZCMOE_OK) rc = dalloc(&(p), (n));
  ZC_ALLOC(h->bias, E);
  ZC_ALLOC(h->b0, E);
  if (cfg->logit_offset) ZC_ALLOC(h->offset, E);
  ZC_ALLOC(h->eta, 1);
  ZC_ALLOC(h->integ, E);
  ZC_ALLOC(h->eprev, E);
  ZC_ALLOC(h->acc_counts, E + 1);
  ZC_ALLOC(h->err, 1);
  ZC_ALLOC(h->logits, (size_t)h->max_T * E);
  ZC_ALLOC(h->gate, (size_t)h->max_pairs);
  ZC_ALLOC(h->idx, (size_t)h->max_pairs);
  ZC_ALLOC(h->pos, (size_t)h->max_pairs);
  ZC_ALLOC(h->counts, E);
  ZC_ALLOC(h->offsets, N + 1);
  ZC_ALLOC(h->mb_off, N + 1);
  ZC_ALLOC(h->sp_off, N + 1);
  ZC_ALLOC(h->sched, 4);
  ZC_ALLOC(h->scal, 4);
  ZC_ALLOC(h->chunk, (size_t)h->max_chunks * E);
  ZC_ALLOC(h->perm, (size_t)h->max_pairs);
  {
    uint8_t *xp = nullptr, *hh = nullptr, *yy = nullptr;
    // FP8 layers use the padded FP8 operands below instead
    ZC_ALLOC(xp, h->fp8 ? 0 : rcap * h->d * esz);
    ZC_ALLOC(hh, h->fp8 ? 0 : rcap * h->inter * esz);
    ZC_ALLOC(yy, h->fp8 ? 0 : rcap * h->d * esz);
    h->xperm = xp;
    h->H = hh;
    h->Y = yy;
  }
  if (ep_size > 1) ZC_ALLOC(h->ep_meta, (size_t)2 * ep_size * NL + 1 + 3 * (NL + 1));
  if (h->fp8) {
    const size_t prow = (size_t)h->max_mblocks * zc::kBM;  // padded rows
    // scale atoms per 128 rows: an atom covers 512 K elements (FP8), 128 (MXFP4) or 64 (NVFP4)
    const int akb = h->fmt == 2 ? 64 : h->fmt ? 128 : 512;
    h->gd = (h->d + akb - 1) / akb;
    h->gi = (h->inter + akb - 1) / akb;
    const size_t wn = (size_t)N * h->inter * h->d / (h->fmt ? 2 : 1);
    ZC_ALLOC(h->w8g, wn);
    ZC_ALLOC(h->w8u, wn);
    ZC_ALLOC(h->w8d, wn);
    ZC_ALLOC(h->sfg, (size_t)N * (h->inter / 128) * h->gd * zc::kAtomBytes);
    ZC_ALLOC(h->sfu, (size_t)N * (h->inter / 128) * h->gd * zc::kAtomBytes);
    ZC_ALLOC(h->sfd, (size_t)N * (h->d / 128) * h->gi * zc::kAtomBytes);
    if (h->fmt == 2) ZC_ALLOC(h->gsc, (size_t)3 * N);
    ZC_ALLOC(h->x8, prow * h->d / (h->fmt ? 2 : 1));
    ZC_ALLOC(h->sx, (size_t)h->max_mblocks * h->gd * zc::kAtomBytes);
    ZC_ALLOC(h->h8, prow * h->inter / (h->fmt ? 2 : 1));
    ZC_ALLOC(h->sh, (size_t)h->max_mblocks * h->gi * zc::kAtomBytes);
    uint8_t* yp = nullptr;
    ZC_ALLOC(yp, prow * h->d * 2);
    h->ypad = yp;
  }
#undef ZC_ALLOC
  if (rc != ZCMOE_OK) {
    release(h);
    delete h;
    return rc;
  }
  h->acc_tokens = h->acc_counts + E;
  if (ep_size > 1) {
    cudaError_t e = cudaHostAlloc(reinterpret_cast<void**>(&h->ep_meta_host),
                                  ((size_t)2 * ep_size * NL + 1 + 3 * (NL + 1)) * sizeof(int32_t), cudaHostAllocDefault);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ep_meta_ev, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      release(h);
      delete h;
      return fail(ZCMOE_ECUDA, "expert-parallel staging: %s", cudaGetErrorString(e));
    }
  }

  // initial state: bias = b0 = init_bias (or 0), eta = 1, integral/previous error = 0
  {
    float* hb = new (std::nothrow) float[E];
    if (!hb) {
      release(h);
      delete h;
      return fail(ZCMOE_ENOMEM, "host allocation failed");
    }
    for (int i = 0; i < E; ++i) hb[i] = cfg->init_bias ? cfg->init_bias[i] : 0.0f;
    const float one = 1.0f;
    cudaError_t e = cudaMemcpy(h->bias, hb, E * sizeof(float), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(h->b0, hb, E * sizeof(float), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && cfg->logit_offset)
      e = cudaMemcpy(h->offset, cfg->logit_offset, E * sizeof(float), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(h->eta, &one, sizeof(float), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(h->integ, 0, E * sizeof(float));
    if (e == cudaSuccess) e = cudaMemset(h->eprev, 0, E * sizeof(float));
    if (e == cudaSuccess) e = cudaMemset(h->acc_counts, 0, (E + 1) * sizeof(int64_t));
    if (e == cudaSuccess) e = cudaMemset(h->err, 0, sizeof(int));
    if (e == cudaSuccess && !h->fp8) e = cudaMemset(h->xperm, 0, rcap * h->d * esz);
    if (e == cudaSuccess && !h->fp8) e = cudaMemset(h->H, 0, rcap * h->inter * esz);
    if (h->fp8) {
      // padded operand rows that no pair fills read as zeros
      const size_t prow = (size_t)h->max_mblocks * zc::kBM;
      if (e == cudaSuccess) e = cudaMemset(h->x8, 0, prow * h->d / (h->fmt ? 2 : 1));
      if (e == cudaSuccess) e = cudaMemset(h->h8, 0, prow * h->inter / (h->fmt ? 2 : 1));
      if (e == cudaSuccess) e = cudaMemset(h->sx, 0, (size_t)h->max_mblocks * h->gd * zc::kAtomBytes);
      if (e == cudaSuccess) e = cudaMemset(h->sh, 0, (size_t)h->max_mblocks * h->gi * zc::kAtomBytes);
      // the expert weights, quantized into scale atoms: FP8 per [128,128], MXFP4 per [1,32], NVFP4 per [1,16]
      const int64_t ri = (int64_t)N * h->inter, rd = (int64_t)N * h->d;
      if (h->fmt == 2) {
        // one fp32 tensor scale per expert matrix, then [1,16] blocks under it
        float *gg = h->gsc, *gu = h->gsc + N, *gdn = h->gsc + 2 * N;
        if (e == cudaSuccess) e = zc::launch_nv4_global(1, w->w_gate, N, h->inter, h->d, gg, 0);
        if (e == cudaSuccess) e = zc::launch_nv4_global(1, w->w_up, N, h->inter, h->d, gu, 0);
        if (e == cudaSuccess) e = zc::launch_nv4_global(1, w->w_down, N, h->d, h->inter, gdn, 0);
        if (e == cudaSuccess)
          e = zc::launch_quant_nv4(1, w->w_gate, ri, h->d, h->w8g, h->sfg, h->gd, gg, h->inter, 1.0f, h->sms, 0);
        if (e == cudaSuccess)
          e = zc::launch_quant_nv4(1, w->w_up, ri, h->d, h->w8u, h->sfu, h->gd, gu, h->inter, 1.0f, h->sms, 0);
        if (e == cudaSuccess)
          e = zc::launch_quant_nv4(1, w->w_down, rd, h->inter, h->w8d, h->sfd, h->gi, gdn, h->d, 1.0f, h->sms, 0);
      } else if (h->fmt) {
        if (e == cudaSuccess) e = zc::launch_quant_mx4(1, w->w_gate, ri, h->d, h->w8g, h->sfg, h->gd, h->sms, 0);
        if (e == cudaSuccess) e = zc::launch_quant_mx4(1, w->w_up, ri, h->d, h->w8u, h->sfu, h->gd, h->sms, 0);
        if (e == cudaSuccess) e = zc::launch_quant_mx4(1, w->w_down, rd, h->inter, h->w8d, h->sfd, h->gi, h->sms, 0);
      } else {
        if (e == cudaSuccess) e = zc::launch_quant_tiles(1, w->w_gate, ri, h->d, h->w8g, h->sfg, h->gd, 0);
        if (e == cudaSuccess) e = zc::launch_quant_tiles(1, w->w_up, ri, h->d, h->w8u, h->sfu, h->gd, 0);
        if (e == cudaSuccess) e = zc::launch_quant_tiles(1, w->w_down, rd, h->inter, h->w8d, h->sfd, h->gi, 0);
      }
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    delete[] hb;
    if (e != cudaSuccess) {
      release(h);
      delete h;
      return fail(ZCMOE_ECUDA, "initialising state: %s", cudaGetErrorString(e));
    }
  }

  if (h->bf16) {
    const uint64_t d = h->d, inter = h->inter;
    rc = make_tmap(&h->tm_wr, w->w_router, d, (uint64_t)E, 256);
    if (rc == ZCMOE_OK) rc = make_tmap(&h->tm_wr_n, w->w_router, d, (uint64_t)E, zc::kRouterNarrowN);
    if (rc == ZCMOE_OK) rc = make_tmap(&h->tm_wg, w->w_gate, d, (uint64_t)NL * inter, 128);
    if (rc == ZCMOE_OK) rc = make_tmap(&h->tm_wu, w->w_up, d, (uint64_t)NL * inter, 128);
    if (rc == ZCMOE_OK) rc = make_tmap(&h->tm_wd, w->w_down, inter, (uint64_t)NL * d, 256);
    if (rc == ZCMOE_OK && !h->fp8) rc = make_tmap(&h->tm_xperm, h->xperm, d, (uint64_t)h->rows_cap, 128);
    if (rc == ZCMOE_OK && !h->fp8) rc = make_tmap(&h->tm_h, h->H, inter, (uint64_t)h->rows_cap, 128);
    if (rc == ZCMOE_OK && !h->fp8) rc = make_tmap(&h->tm_y, h->Y, d, (uint64_t)h->rows_cap, 32);  // down output
    if (h->fp8) {
      // codes as bytes: the K extent is d or inter bytes (FP8), half that (FP4)
      const uint64_t prow = (uint64_t)h->max_mblocks * zc::kBM;
      const uint64_t db = d / (h->fmt ? 2 : 1), ib = inter / (h->fmt ? 2 : 1);
      if (rc == ZCMOE_OK) rc = make_tmap_esz(&h->tm8_wg, h->w8g, db, (uint64_t)N * inter, 128, 1);
      if (rc == ZCMOE_OK) rc = make_tmap_esz(&h->tm8_wu, h->w8u, db, (uint64_t)N * inter, 128, 1);
      if (rc == ZCMOE_OK) rc = make_tmap_esz(&h->tm8_wd, h->w8d, ib, (uint64_t)N * d, 256, 1);
      if (rc == ZCMOE_OK) rc = make_tmap_esz(&h->tm8_x, h->x8, db, prow, 128, 1);
      if (rc == ZCMOE_OK) rc = make_tmap_esz(&h->tm8_h, h->h8, ib, prow, 128, 1);
      if (rc == ZCMOE_OK) rc = make_tmap_store32(&h->tm8_y, h->ypad, d, prow);
    }
    if (rc != ZCMOE_OK) {
      release(h);
      delete h;
      return rc;
    }
  }
  h->alive = true;
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    g_live.insert(h);
  }
  *out = h;
  return ZCMOE_OK;
}

int zcmoe_create(const zcmoe_config* cfg, const zcmoe_weights* w, zcmoe_t* out) {
  return create_impl(cfg, w, 0, 1, 0, out);
}

int zcmoe_create_ep(const zcmoe_config* cfg, const zcmoe_weights* local, int32_t ep_rank, int32_t ep_size,
                    int64_t max_recv_rows, zcmoe_t* out) {
  return create_impl(cfg, local, ep_rank, ep_size, max_recv_rows, out);
}

// 1. router logits (+ the logit offset), fp32 [T, E]
static int router_stage(zcmoe_t h, const void* x, int Ti, cudaStream_t s) {
  const int E = h->E, d = h->d;
  const int64_t T = Ti;
  if (h->bf16) {
    CUtensorMap tm_x;
    int rc = make_tmap(&tm_x, x, (uint64_t)d, (uint64_t)T, 128);
    if (rc != ZCMOE_OK) return rc;
    // a batch of a few row blocks takes 32-column tiles, so that more SMs share its
    // W_r and x bytes (the same logits either way)
    const int mblocks = (Ti + zc::kBM - 1) / zc::kBM;
    const int mode = mblocks * ((E + zc::kRouterNarrowN - 1) / zc::kRouterNarrowN) <= h->sms ? zc::kRouterNarrow
                                                                                               : zc::kRouter;
    zc::TcArgs a{};
    a.K = d;
    a.n_out = E;
    a.nblocks = (E + zc::tc_block_n(mode) - 1) / zc::tc_block_n(mode);
    a.ngroups = 1;
    a.M = Ti;
    a.out = h->logits;
    a.ldo = E;
    a.col_add = h->offset;
    a.err = h->err;
    a.sched = h->sched;
    const int tiles = mblocks * a.nblocks;
    const CUtensorMap& tm_b = mode == zc::kRouterNarrow ? h->tm_wr_n : h->tm_wr;
    ZC_CUDA(zc::launch_tc_gemm(mode, tm_x, tm_b, tm_b, tm_b, a, tiles < h->sms ? tiles : h->sms, s));
  } else {
    zc::SimtArgs a{};
    a.A = static_cast<const float*>(x);
    a.B0 = static_cast<const float*>(h->w.w_router);
    a.K = d;
    a.n_out = E;
    a.ngroups = 1;
    a.M = Ti;
    a.out = h->logits;
    a.ldo = E;
    a.col_add = h->offset;
    ZC_CUDA(zc::launch_simt_gemm(zc::kRouter, a, (Ti + zc::kBM - 1) / zc::kBM, s));
  }
  return ZCMOE_OK;
}

// 3. the integer stage: counts (into the controller's accumulators too), offsets,
// row-block offsets, the permutation of the FFN pairs, the slot positions
static int integer_stage(zcmoe_t h, int Ti, cudaStream_t s) {
  const int E = h->E, N = h->N, k = h->k;
  if (Ti <= zc::route_small_max_tokens()) {  // one launch for a small batch
    ZC_CUDA(zc::launch_route_small(h->idx, Ti, k, N, E, h->counts, h->offsets, h->mb_off, h->scal, h->acc_counts,
                                   h->acc_tokens, h->sp_off, h->perm, h->pos, s));
    return ZCMOE_OK;
  }
  const int nchunks = (Ti + zc::kChunk - 1) / zc::kChunk;
  ZC_CUDA(zc::launch_route_count(h->idx, Ti, k, E, h->chunk, s));
  ZC_CUDA(zc::launch_route_scan(h->chunk, nchunks, Ti, N, E, h->counts, h->offsets, h->mb_off, h->scal,
                                h->acc_counts, h->acc_tokens, s, h->sp_off));
  ZC_CUDA(zc::launch_route_scatter(h->idx, Ti, k, N, E, h->chunk, h->perm, h->pos, s));
  return ZCMOE_OK;
}

// The routing outputs a caller asked for in `dbg` (all but scores, which the
// top-k kernel writes itself, and expert_out), copied out of the handle's workspace.
static int copy_routing_debug(zcmoe_t h, int T, const zcmoe_debug* dbg, cudaStream_t s) {
  const int E = h->E, N = h->N, k = h->k;
  if (dbg->logits) ZC_CUDA(cudaMemcpyAsync(dbg->logits, h->logits, (size_t)T * E * 4, cudaMemcpyDeviceToDevice, s));
  if (dbg->idx) ZC_CUDA(cudaMemcpyAsync(dbg->idx, h->idx, (size_t)T * k * 4, cudaMemcpyDeviceToDevice, s));
  if (dbg->gate) ZC_CUDA(cudaMemcpyAsync(dbg->gate, h->gate, (size_t)T * k * 4, cudaMemcpyDeviceToDevice, s));
  if (dbg->counts) ZC_CUDA(cudaMemcpyAsync(dbg->counts, h->counts, (size_t)E * 4, cudaMemcpyDeviceToDevice, s));
  if (dbg->offsets)
    ZC_CUDA(cudaMemcpyAsync(dbg->offsets, h->offsets, (size_t)(N + 1) * 4, cudaMemcpyDeviceToDevice, s));
  if (dbg->perm) ZC_CUDA(cudaMemcpyAsync(dbg->perm, h->perm, (size_t)T * k * 4, cudaMemcpyDeviceToDevice, s));
  if (dbg->pos) ZC_CUDA(cudaMemcpyAsync(dbg->pos, h->pos, (size_t)T * k * 4, cudaMemcpyDeviceToDevice, s));
  return ZCMOE_OK;
}

// The forward pass; with `side`, the dense FFN's two GEMMs are forked onto its
// stream after the router GEMM and after the down GEMM, and joined back into
// `s` after the combine.
static int forward_impl(zcmoe_t h, const void* x, int64_t T, void* y, cudaStream_t s, const zcmoe_debug* dbg,
                        const DenseSide* side) {
  if (h->ep_size > 1) return fail(ZCMOE_EUNSUPPORTED, "an expert-parallel handle runs through zcmoe_ep_*");
  if (T < 0 || T > h->max_T) return fail(ZCMOE_ERANGE, "T=%lld outside [0, %d]", (long long)T, h->max_T);
  if (T == 0) return ZCMOE_OK;
  if (!x || !y) return fail(ZCMOE_EINVAL, "x or y is NULL");
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u))
    return fail(ZCMOE_EINVAL, "x and y must be 16-byte aligned");
  const size_t esz = h->bf16 ? 2 : 4;
  const size_t xbytes = (size_t)T * h->d * esz;
  const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
  if (xa < ya + xbytes && ya < xa + xbytes) return fail(ZCMOE_EINVAL, "y overlaps x");

  const int Ti = (int)T, E = h->E, N = h->N, k = h->k, d = h->d, inter = h->inter;
  h->last_T = Ti;
  // Stage boundaries: an NVTX range per stage around its enqueue on the host (profiler
  // timelines), and, while profiling, a CUDA event on the stream (per-stage device time).
  bool nvtx_open = false;
  auto mark = [&](const char* next) -> cudaError_t {
    if (nvtx_open) nvtxRangePop();
    nvtx_open = next != nullptr;
    if (next) nvtxRangePushA(next);
    if (!h->profiling) return cudaSuccess;
    cudaEvent_t ev;
    cudaError_t e = cudaEventCreate(&ev);
    if (e != cudaSuccess) return e;
    h->events->push_back(ev);
    return cudaEventRecord(ev, s);
  };
  // an early return leaves no range open
  struct RangeGuard {
    bool* open;
    ~RangeGuard() {
      if (*open) nvtxRangePop();
    }
  } range_guard{&nvtx_open};
  ZC_CUDA(mark("zcmoe.router"));

  // 1. router logits
  {
    const int rc = router_stage(h, x, Ti, s);
    if (rc != ZCMOE_OK) return rc;
  }
  ZC_CUDA(mark("zcmoe.softmax_topk"));
  if (side) {
    ZC_CUDA(cudaEventRecord(side->dn->ev_router, s));
    ZC_CUDA(cudaStreamWaitEvent(side->dn->side, side->dn->ev_router, 0));
    const int rc = dense_gate_up(side->dn, side->x, Ti, side->dn->side);
    if (rc != ZCMOE_OK) return rc;
  }
  // 2. softmax + bias-shifted top-k
  ZC_CUDA(zc::launch_softmax_topk(h->logits, h->bias, Ti, E, k, h->cfg.routed_scale, h->idx, h->gate,
                                  dbg ? dbg->scores : nullptr, h->sms, s));
  ZC_CUDA(mark("zcmoe.integer_stage"));
  // 3. integer stage
  {
    const int rc = integer_stage(h, Ti, s);
    if (rc != ZCMOE_OK) return rc;
  }
  ZC_CUDA(mark("zcmoe.gather"));
  // 4. the FFN pairs' rows in expert order, each token's row read once (FP8 / FP4 layers:
  // quantized once per token into every padded row of it)
  if (h->fp8)
    ZC_CUDA(zc::launch_scatter_quant(h->fmt, x, d, h->pos, h->idx, Ti, k, h->offsets, h->mb_off, h->x8, h->sx, h->gd,
                                     h->sms, s));
  else
    ZC_CUDA(zc::launch_scatter_rows(x, (int)(d * esz), h->pos, Ti, k, h->xperm, h->sms, s));
  ZC_CUDA(mark("zcmoe.gate_up"));
  // 5./6. expert GEMMs
  const int max_mb = (Ti * k + zc::kBM - 1) / zc::kBM + N;
  if (h->fp8) {
    zc::Fp8Args a{};
    a.fmt = h->fmt;
    a.K = d;
    a.n_out = inter;
    a.nblocks = inter / zc::fp8_block_n(zc::kGateUp);
    a.ngroups = N;
    a.row_off = h->offsets;
    a.mb_off = h->mb_off;
    a.b_rows_per_group = inter;
    a.sfa = h->sx;
    a.sfb0 = h->sfg;
    a.sfb1 = h->sfu;
    a.groups_k = h->gd;
    a.out = h->h8;
    a.ldo = inter / (h->fmt ? 2 : 1);
    a.out_sf = h->sh;
    a.out_groups = h->gi;
    a.gsc0 = h->gsc;
    a.gsc1 = h->gsc ? h->gsc + N : nullptr;
    a.err = h->err;
    int bound = max_mb * a.nblocks;
    ZC_CUDA(zc::launch_fp8_gemm(zc::kGateUp, h->tm8_x, h->tm8_wg, h->tm8_wu, h->tm8_wu, a,
                                bound < h->sms ? bound : h->sms, s));
    ZC_CUDA(mark("zcmoe.down"));
    zc::Fp8Args b{};
    b.fmt = h->fmt;
    b.K = inter;
    b.n_out = d;
    b.nblocks = (d + zc::fp8_block_n(zc::kDown) - 1) / zc::fp8_block_n(zc::kDown);
    b.ngroups = N;
    b.row_off = h->offsets;
    b.mb_off = h->mb_off;
    b.b_rows_per_group = d;
    b.sfa = h->sh;
    b.sfb0 = h->sfd;
    b.sfb1 = nullptr;
    b.groups_k = h->gi;
    b.gsc0 = h->gsc ? h->gsc + 2 * N : nullptr;
    b.out = h->ypad;
    b.ldo = d;
    b.err = h->err;
    bound = max_mb * b.nblocks;
    ZC_CUDA(zc::launch_fp8_gemm(zc::kDown, h->tm8_h, h->tm8_wd, h->tm8_wd, h->tm8_y, b, bound < h->sms ? bound : h->sms,
                                s));
  } else if (h->bf16) {
    zc::TcArgs a{};
    a.K = d;
    a.n_out = inter;
    a.nblocks = (inter + zc::tc_block_n(zc::kGateUp) - 1) / zc::tc_block_n(zc::kGateUp);
    a.ngroups = N;
    a.row_off = h->offsets;
    a.mb_off = h->mb_off;
    a.sp_off = h->sp_off;
    a.sched = h->sched + 1;
    a.pair = zc::tc_pair_for_rows((int64_t)Ti * k / E);
    a.b_rows_per_group = inter;
    a.out = h->H;
    a.ldo = inter;
    a.gu_save = h->b_gu;
    a.err = h->err;
    h->last_saved = h->b_gu != nullptr;
    int bound = max_mb * a.nblocks;
    ZC_CUDA(zc::launch_tc_gemm(zc::kGateUp, h->tm_xperm, h->tm_wg, h->tm_wu, h->tm_wu, a,
                               bound < h->sms ? bound : h->sms, s));
    ZC_CUDA(mark("zcmoe.down"));
    zc::TcArgs b{};
    b.K = inter;
    b.n_out = d;
    b.nblocks = (d + zc::tc_block_n(zc::kDown) - 1) / zc::tc_block_n(zc::kDown);
    b.ngroups = N;
    b.row_off = h->offsets;
    b.mb_off = h->mb_off;
    b.sp_off = h->sp_off;
    b.sched = h->sched + 2;
    b.pair = a.pair;
    b.b_rows_per_group = d;
    b.out = h->Y;
    b.ldo = d;
    b.err = h->err;
    bound = max_mb * b.nblocks;
    ZC_CUDA(zc::launch_tc_gemm(zc::kDown, h->tm_h, h->tm_wd, h->tm_wd, h->tm_y, b, bound < h->sms ? bound : h->sms, s));
  } else {
    zc::SimtArgs a{};
    a.A = static_cast<const float*>(h->xperm);
    a.B0 = static_cast<const float*>(h->w.w_gate);
    a.B1 = static_cast<const float*>(h->w.w_up);
    a.K = d;
    a.n_out = inter;
    a.ngroups = N;
    a.row_off = h->offsets;
    a.mb_off = h->mb_off;
    a.b_rows_per_group = inter;
    a.out = static_cast<float*>(h->H);
    a.ldo = inter;
    ZC_CUDA(zc::launch_simt_gemm(zc::kGateUp, a, max_mb, s));
    ZC_CUDA(mark("zcmoe.down"));
    zc::SimtArgs b{};
    b.A = static_cast<const float*>(h->H);
    b.B0 = static_cast<const float*>(h->w.w_down);
    b.K = inter;
    b.n_out = d;
    b.ngroups = N;
    b.row_off = h->offsets;
    b.mb_off = h->mb_off;
    b.b_rows_per_group = d;
    b.out = static_cast<float*>(h->Y);
    b.ldo = d;
    ZC_CUDA(zc::launch_simt_gemm(zc::kDown, b, max_mb, s));
  }
  ZC_CUDA(mark("zcmoe.combine"));
  if (side) {
    ZC_CUDA(cudaEventRecord(side->dn->ev_down, s));
    ZC_CUDA(cudaStreamWaitEvent(side->dn->side, side->dn->ev_down, 0));
    const int rc = dense_down(side->dn, Ti, side->y, side->dn->side);
    if (rc != ZCMOE_OK) return rc;
    ZC_CUDA(cudaEventRecord(side->dn->ev_join, side->dn->side));
  }
  // 7. combine
  if (h->fp8)
    ZC_CUDA(zc::launch_combine(1, x, h->ypad, h->idx, h->gate, h->pos, Ti, k, N, d, y, h->sms, s, h->offsets,
                               h->mb_off));
  else
    ZC_CUDA(zc::launch_combine(h->bf16, x, h->Y, h->idx, h->gate, h->pos, Ti, k, N, d, y, h->sms, s));
  ZC_CUDA(mark(nullptr));
  if (side) ZC_CUDA(cudaStreamWaitEvent(s, side->dn->ev_join, 0));

  if (dbg) {
    const int rc = copy_routing_debug(h, Ti, dbg, s);
    if (rc != ZCMOE_OK) return rc;
    if (dbg->expert_out && h->fp8)
      ZC_CUDA(zc::launch_unpad_rows(h->ypad, d * 2, h->perm, h->idx, h->offsets, h->mb_off, h->scal, dbg->expert_out,
                                    h->sms, s));
    else if (dbg->expert_out)
      ZC_CUDA(cudaMemcpyAsync(dbg->expert_out, h->Y, (size_t)T * k * d * esz, cudaMemcpyDeviceToDevice, s));
  }
  return ZCMOE_OK;
}

int zcmoe_forward(zcmoe_t h, const void* x, int64_t T, void* y, cudaStream_t s, const zcmoe_debug* dbg) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  return forward_impl(h, x, T, y, s, dbg, nullptr);
}

// ---------------------------------------------------------------- expert parallelism

int zcmoe_ep_dispatch(zcmoe_t h, const void* x, int64_t T, void* xsend, int32_t* offsets, cudaStream_t s,
                      const zcmoe_debug* dbg) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!h->bf16 || h->fp8) return fail(ZCMOE_EUNSUPPORTED, "expert parallelism needs a bf16 layer");
  if (T < 0 || T > h->max_T) return fail(ZCMOE_ERANGE, "T=%lld outside [0, %d]", (long long)T, h->max_T);
  if (!offsets) return fail(ZCMOE_EINVAL, "offsets is NULL");
  const int Ti = (int)T;
  if (T == 0) {  // x and xsend may be NULL (no rows)
    h->last_T = 0;
    ZC_CUDA(cudaMemsetAsync(offsets, 0, (size_t)(h->N + 1) * sizeof(int32_t), s));
    return ZCMOE_OK;
  }
  if (!x || !xsend) return fail(ZCMOE_EINVAL, "x or xsend is NULL");
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(xsend) & 15u))
    return fail(ZCMOE_EINVAL, "x and xsend must be 16-byte aligned");
  const size_t xb = (size_t)T * h->d * 2, sb = (size_t)T * h->k * h->d * 2;
  if (overlaps(xsend, sb, x, xb)) return fail(ZCMOE_EINVAL, "xsend overlaps x");
  h->last_T = Ti;
  int rc = router_stage(h, x, Ti, s);
  if (rc != ZCMOE_OK) return rc;
  ZC_CUDA(zc::launch_softmax_topk(h->logits, h->bias, Ti, h->E, h->k, h->cfg.routed_scale, h->idx, h->gate,
                                  dbg ? dbg->scores : nullptr, h->sms, s));
  rc = integer_stage(h, Ti, s);
  if (rc != ZCMOE_OK) return rc;
  ZC_CUDA(zc::launch_scatter_rows(x, h->d * 2, h->pos, Ti, h->k, xsend, h->sms, s));
  ZC_CUDA(cudaMemcpyAsync(offsets, h->offsets, (size_t)(h->N + 1) * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  if (dbg) return copy_routing_debug(h, Ti, dbg, s);
  return ZCMOE_OK;
}

int zcmoe_ep_experts(zcmoe_t h, const void* xrecv, const int32_t* counts, int64_t P_recv, void* yrecv,
                     cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!h->bf16 || h->fp8) return fail(ZCMOE_EUNSUPPORTED, "expert parallelism needs a bf16 layer");
  if (P_recv < 0 || P_recv > h->rows_cap)
    return fail(ZCMOE_ERANGE, "P_recv=%lld outside [0, %lld]", (long long)P_recv, (long long)h->rows_cap);
  if (!counts) return fail(ZCMOE_EINVAL, "counts is NULL");
  const int R = h->ep_size, NL = h->n_local, nseg = R * NL;
  int64_t total = 0;
  for (int i = 0; i < nseg; ++i) {
    if (counts[i] < 0) return fail(ZCMOE_EINVAL, "counts[%d] is negative", i);
    total += counts[i];
  }
  if (total != P_recv) return fail(ZCMOE_EINVAL, "counts sum to %lld, not P_recv=%lld", (long long)total,
                                   (long long)P_recv);
  if (P_recv == 0) return ZCMOE_OK;
  if (!xrecv || !yrecv) return fail(ZCMOE_EINVAL, "xrecv or yrecv is NULL");
  if ((reinterpret_cast<uintptr_t>(xrecv) & 15u) || (reinterpret_cast<uintptr_t>(yrecv) & 15u))
    return fail(ZCMOE_EINVAL, "xrecv and yrecv must be 16-byte aligned");
  const size_t rb = (size_t)P_recv * h->d * 2;
  if (overlaps(xrecv, rb, yrecv, rb)) return fail(ZCMOE_EINVAL, "yrecv overlaps xrecv");
  const int d = h->d, inter = h->inter;

  // row layout: ep_size == 1 needs no regrouping (one source: s-major is e-major)
  const int32_t* exp_off;
  const int32_t* mb_off;
  const int32_t* sp_off;
  int mb_total = 0;
  const void* a_rows = xrecv;
  void* y_rows = yrecv;
  if (R > 1) {
    if (h->ep_meta_pending) {
      ZC_CUDA(cudaEventSynchronize(h->ep_meta_ev));  // the previous upload has read the staging buffer
      h->ep_meta_pending = false;
    }
    int32_t* m = h->ep_meta_host;
    int32_t* seg_src = m;
    int32_t* seg_dst = seg_src + nseg + 1;
    int32_t* eoff = seg_dst + nseg;
    int32_t* moff = eoff + NL + 1;
    int32_t* poff = moff + NL + 1;
    seg_src[0] = 0;
    for (int i = 0; i < nseg; ++i) seg_src[i + 1] = seg_src[i] + counts[i];
    eoff[0] = 0;
    moff[0] = 0;
    poff[0] = 0;
    for (int e = 0; e < NL; ++e) {
      int cnt = 0;
      for (int r = 0; r < R; ++r) {
        seg_dst[r * NL + e] = eoff[e] + cnt;
        cnt += counts[r * NL + e];
      }
      eoff[e + 1] = eoff[e] + cnt;
      const int mb = (cnt + zc::kBM - 1) / zc::kBM;
      moff[e + 1] = moff[e] + mb;
      poff[e + 1] = poff[e] + (mb + 1) / 2;
    }
    mb_total = moff[NL];
    const size_t bytes = ((size_t)2 * nseg + 1 + 3 * (NL + 1)) * sizeof(int32_t);
    ZC_CUDA(cudaMemcpyAsync(h->ep_meta, m, bytes, cudaMemcpyHostToDevice, s));
    ZC_CUDA(cudaEventRecord(h->ep_meta_ev, s));
    h->ep_meta_pending = true;
    const int32_t* dseg_src = h->ep_meta;
    const int32_t* dseg_dst = dseg_src + nseg + 1;
    exp_off = dseg_dst + nseg;
    mb_off = exp_off + NL + 1;
    sp_off = mb_off + NL + 1;
    // rows into the e-major layout of xperm; the outputs come back through Y
    ZC_CUDA(zc::launch_ep_regroup(xrecv, h->xperm, P_recv, d * 2, dseg_src, dseg_dst, nseg, 0, h->sms, s));
    a_rows = h->xperm;
    y_rows = h->Y;
  } else {
    // one source: the counts are the expert offsets; stage them like the segments
    if (h->ep_meta_pending) {
      ZC_CUDA(cudaEventSynchronize(h->ep_meta_ev));
      h->ep_meta_pending = false;
    }
    if (!h->ep_meta) {
      int rc = dalloc(&h->ep_meta, (size_t)3 * (NL + 1));
      if (rc != ZCMOE_OK) return rc;
      cudaError_t e = cudaHostAlloc(reinterpret_cast<void**>(&h->ep_meta_host), (size_t)3 * (NL + 1) * sizeof(int32_t),
                                    cudaHostAllocDefault);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ep_meta_ev, cudaEventDisableTiming);
      if (e != cudaSuccess) return fail(ZCMOE_ECUDA, "expert-parallel staging: %s", cudaGetErrorString(e));
    }
    int32_t* eoff = h->ep_meta_host;
    int32_t* moff = eoff + NL + 1;
    int32_t* poff = moff + NL + 1;
    eoff[0] = 0;
    moff[0] = 0;
    poff[0] = 0;
    for (int e = 0; e < NL; ++e) {
      eoff[e + 1] = eoff[e] + counts[e];
      const int mb = (counts[e] + zc::kBM - 1) / zc::kBM;
      moff[e + 1] = moff[e] + mb;
      poff[e + 1] = poff[e] + (mb + 1) / 2;
    }
    mb_total = moff[NL];
    ZC_CUDA(cudaMemcpyAsync(h->ep_meta, eoff, (size_t)3 * (NL + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, s));
    ZC_CUDA(cudaEventRecord(h->ep_meta_ev, s));
    h->ep_meta_pending = true;
    exp_off = h->ep_meta;
    mb_off = exp_off + NL + 1;
    sp_off = mb_off + NL + 1;
  }
  CUtensorMap tm_a, tm_h;
  int rc = make_tmap(&tm_a, a_rows, (uint64_t)d, (uint64_t)P_recv, 128);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_h, h->H, (uint64_t)inter, (uint64_t)P_recv, 128);
  if (rc != ZCMOE_OK) return rc;
  // the local experts' grouped GEMMs (the forward's kernels, over the received rows)
  zc::TcArgs a{};
  a.K = d;
  a.n_out = inter;
  a.nblocks = (inter + zc::tc_block_n(zc::kGateUp) - 1) / zc::tc_block_n(zc::kGateUp);
  a.ngroups = NL;
  a.row_off = exp_off;
  a.mb_off = mb_off;
  a.sp_off = sp_off;
  a.sched = h->sched + 1;
  a.pair = zc::tc_pair_for_rows(P_recv / NL);
  a.b_rows_per_group = inter;
  a.out = h->H;
  a.ldo = inter;
  a.err = h->err;
  int bound = mb_total * a.nblocks;
  ZC_CUDA(zc::launch_tc_gemm(zc::kGateUp, tm_a, h->tm_wg, h->tm_wu, h->tm_wu, a, bound < h->sms ? bound : h->sms, s));
  zc::TcArgs b{};
  b.K = inter;
  b.n_out = d;
  b.nblocks = (d + zc::tc_block_n(zc::kDown) - 1) / zc::tc_block_n(zc::kDown);
  b.ngroups = NL;
  b.row_off = exp_off;
  b.mb_off = mb_off;
  b.sp_off = sp_off;
  b.sched = h->sched + 2;
  b.pair = a.pair;
  b.b_rows_per_group = d;
  b.out = y_rows;
  b.ldo = d;
  b.err = h->err;
  bound = mb_total * b.nblocks;
  CUtensorMap tm_yr;
  rc = make_tmap(&tm_yr, y_rows, (uint64_t)d, (uint64_t)P_recv, 32);
  if (rc != ZCMOE_OK) return rc;
  ZC_CUDA(zc::launch_tc_gemm(zc::kDown, tm_h, h->tm_wd, h->tm_wd, tm_yr, b, bound < h->sms ? bound : h->sms, s));
  if (R > 1) {
    const int32_t* dseg_src = h->ep_meta;
    ZC_CUDA(zc::launch_ep_regroup(h->Y, yrecv, P_recv, d * 2, dseg_src, dseg_src + nseg + 1, nseg, 1, h->sms, s));
  }
  return ZCMOE_OK;
}

int zcmoe_ep_combine(zcmoe_t h, const void* x, const void* yback, int64_t T, void* y, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!h->bf16 || h->fp8) return fail(ZCMOE_EUNSUPPORTED, "expert parallelism needs a bf16 layer");
  if (T < 0 || T > h->max_T) return fail(ZCMOE_ERANGE, "T=%lld outside [0, %d]", (long long)T, h->max_T);
  if (T != h->last_T) return fail(ZCMOE_EINVAL, "T=%lld differs from the last dispatch's %d", (long long)T, h->last_T);
  if (T == 0) return ZCMOE_OK;
  if (!x || !y || !yback) return fail(ZCMOE_EINVAL, "x, yback or y is NULL");
  const void* ps[3] = {x, yback, y};
  for (const void* p : ps)
    if (reinterpret_cast<uintptr_t>(p) & 15u) return fail(ZCMOE_EINVAL, "x, yback and y must be 16-byte aligned");
  const size_t xb = (size_t)T * h->d * 2;
  if (overlaps(y, xb, x, xb)) return fail(ZCMOE_EINVAL, "y overlaps x");
  ZC_CUDA(zc::launch_combine(1, x, yback, h->idx, h->gate, h->pos, (int)T, h->k, h->N, h->d, y, h->sms, s));
  return ZCMOE_OK;
}

// Call i uses staging buffers i % 2.  Upload (copy_stream, after forward i-2 has read the
// buffer) -> forward on `s` (after the upload and after download i-2 has read the y buffer)
// -> download (d2h_stream, after the forward).  At the end of the call `s` waits for
// download i-1 (async form) or download i (zcmoe_forward_host): in the async form, forward i
// runs while download i-1 and upload i+1 move.
static int forward_host_impl(zcmoe_t h, const void* x_host, int64_t T, void* y_host, cudaStream_t s, bool async) {
  if (T < 0 || T > h->max_T) return fail(ZCMOE_ERANGE, "T=%lld outside [0, %d]", (long long)T, h->max_T);
  if (T == 0) return ZCMOE_OK;
  if (!x_host || !y_host) return fail(ZCMOE_EINVAL, "x or y is NULL");
  const size_t bytes_max = (size_t)h->max_T * h->d * (h->bf16 ? 2 : 4);
  if (!h->stage_x) {
    uint8_t *a = nullptr, *a2 = nullptr, *b = nullptr, *b2 = nullptr;
    int rc = dalloc(&a, bytes_max);
    if (rc == ZCMOE_OK) rc = dalloc(&a2, bytes_max);
    if (rc == ZCMOE_OK) rc = dalloc(&b, bytes_max);
    if (rc == ZCMOE_OK) rc = dalloc(&b2, bytes_max);
    cudaError_t e = cudaSuccess;
    if (rc == ZCMOE_OK) e = cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking);
    if (rc == ZCMOE_OK && e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->d2h_stream, cudaStreamNonBlocking);
    for (int i = 0; i < 2 && rc == ZCMOE_OK && e == cudaSuccess; ++i) {
      cudaEvent_t* evs[4] = {&h->ev_in[i], &h->ev_used[i], &h->ev_fwd[i], &h->ev_ydone[i]};
      for (cudaEvent_t* ev : evs)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    }
    if (rc != ZCMOE_OK || e != cudaSuccess) {
      uint8_t* bufs[4] = {a, a2, b, b2};
      for (uint8_t* p : bufs)
        if (p) cudaFree(p);
      for (int i = 0; i < 2; ++i) {
        cudaEvent_t* evs[4] = {&h->ev_in[i], &h->ev_used[i], &h->ev_fwd[i], &h->ev_ydone[i]};
        for (cudaEvent_t* ev : evs) {
          if (*ev) cudaEventDestroy(*ev);
          *ev = nullptr;
        }
      }
      if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
      if (h->d2h_stream) cudaStreamDestroy(h->d2h_stream);
      h->copy_stream = h->d2h_stream = nullptr;
      if (rc != ZCMOE_OK) return rc;
      return fail(ZCMOE_ECUDA, "creating the copy streams: %s", cudaGetErrorString(e));
    }
    h->stage_x = a;
    h->stage_x2 = a2;
    h->stage_y = b;
    h->stage_y2 = b2;
  }
  const size_t bytes = (size_t)T * h->d * (h->bf16 ? 2 : 4);
  const int buf = (int)(h->host_calls & 1);
  void* sx = buf ? h->stage_x2 : h->stage_x;
  void* sy = buf ? h->stage_y2 : h->stage_y;
  if (h->host_calls >= 2) ZC_CUDA(cudaStreamWaitEvent(h->copy_stream, h->ev_used[buf], 0));
  ZC_CUDA(cudaMemcpyAsync(sx, x_host, bytes, cudaMemcpyHostToDevice, h->copy_stream));
  ZC_CUDA(cudaEventRecord(h->ev_in[buf], h->copy_stream));
  ZC_CUDA(cudaStreamWaitEvent(s, h->ev_in[buf], 0));
  if (h->host_calls >= 2) ZC_CUDA(cudaStreamWaitEvent(s, h->ev_ydone[buf], 0));
  int rc = zcmoe_forward(h, sx, T, sy, s, nullptr);
  if (rc != ZCMOE_OK) return rc;
  ZC_CUDA(cudaEventRecord(h->ev_used[buf], s));
  ZC_CUDA(cudaEventRecord(h->ev_fwd[buf], s));
  ZC_CUDA(cudaStreamWaitEvent(h->d2h_stream, h->ev_fwd[buf], 0));
  ZC_CUDA(cudaMemcpyAsync(y_host, sy, bytes, cudaMemcpyDeviceToHost, h->d2h_stream));
  ZC_CUDA(cudaEventRecord(h->ev_ydone[buf], h->d2h_stream));
  if (!async) ZC_CUDA(cudaStreamWaitEvent(s, h->ev_ydone[buf], 0));
  else if (h->host_calls >= 1) ZC_CUDA(cudaStreamWaitEvent(s, h->ev_ydone[buf ^ 1], 0));
  ++h->host_calls;
  return ZCMOE_OK;
}

int zcmoe_forward_host(zcmoe_t h, const void* x_host, int64_t T, void* y_host, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  return forward_host_impl(h, x_host, T, y_host, s, false);
}

int zcmoe_forward_host_async(zcmoe_t h, const void* x_host, int64_t T, void* y_host, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  return forward_host_impl(h, x_host, T, y_host, s, true);
}

int zcmoe_forward_host_flush(zcmoe_t h, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (h->host_calls == 0) return ZCMOE_OK;
  ZC_CUDA(cudaStreamWaitEvent(s, h->ev_ydone[(int)((h->host_calls - 1) & 1)], 0));
  return ZCMOE_OK;
}

int zcmoe_update_bias(zcmoe_t h, const zcmoe_gains* g, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!g) return fail(ZCMOE_EINVAL, "gains is NULL");
  if (!std::isfinite(g->kp) || !std::isfinite(g->ki) || !std::isfinite(g->kd) || !std::isfinite(g->decay))
    return fail(ZCMOE_EINVAL, "kp, ki, kd and decay must be finite");
  if (!(g->target_ffn_per_token >= 0.0f && g->target_ffn_per_token <= (float)h->k))
    return fail(ZCMOE_EINVAL, "target_ffn_per_token must lie in [0, top_k]");
  if (h->Z == 0 && g->target_ffn_per_token != (float)h->k)
    return fail(ZCMOE_EINVAL, "without zero experts the FFN target must equal top_k");
  ZC_CUDA(zc::launch_update_bias(h->acc_counts, h->acc_tokens, h->N, h->Z, h->k, g->kp, g->ki, g->kd, g->decay,
                                 g->target_ffn_per_token, h->b0, h->eta, h->integ, h->eprev, h->bias, s));
  return ZCMOE_OK;
}

int zcmoe_read_counts(zcmoe_t h, int64_t* dst, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!dst) return fail(ZCMOE_EINVAL, "dst is NULL");
  ZC_CUDA(cudaMemcpyAsync(dst, h->acc_counts, (size_t)(h->E + 1) * sizeof(int64_t), cudaMemcpyDeviceToDevice, s));
  return ZCMOE_OK;
}

int zcmoe_write_counts(zcmoe_t h, const int64_t* src, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!src) return fail(ZCMOE_EINVAL, "src is NULL");
  ZC_CUDA(cudaMemcpyAsync(h->acc_counts, src, (size_t)(h->E + 1) * sizeof(int64_t), cudaMemcpyDeviceToDevice, s));
  return ZCMOE_OK;
}

int zcmoe_get_state(zcmoe_t h, float* bias, int64_t* counts, int64_t* tokens, float* eta) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  ZC_CUDA(cudaDeviceSynchronize());
  if (bias) ZC_CUDA(cudaMemcpy(bias, h->bias, h->E * sizeof(float), cudaMemcpyDeviceToHost));
  if (counts) ZC_CUDA(cudaMemcpy(counts, h->acc_counts, h->E * sizeof(int64_t), cudaMemcpyDeviceToHost));
  if (tokens) ZC_CUDA(cudaMemcpy(tokens, h->acc_tokens, sizeof(int64_t), cudaMemcpyDeviceToHost));
  if (eta) ZC_CUDA(cudaMemcpy(eta, h->eta, sizeof(float), cudaMemcpyDeviceToHost));
  return ZCMOE_OK;
}

int zcmoe_set_bias(zcmoe_t h, const float* bias) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!bias) return fail(ZCMOE_EINVAL, "bias is NULL");
  ZC_CUDA(cudaDeviceSynchronize());
  ZC_CUDA(cudaMemcpy(h->bias, bias, h->E * sizeof(float), cudaMemcpyHostToDevice));
  return ZCMOE_OK;
}

int zcmoe_get_controller(zcmoe_t h, float* bias, float* integ, float* eprev, float* eta, int64_t* counts,
                         int64_t* tokens) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  ZC_CUDA(cudaDeviceSynchronize());
  const size_t fE = (size_t)h->E * sizeof(float);
  if (bias) ZC_CUDA(cudaMemcpy(bias, h->bias, fE, cudaMemcpyDeviceToHost));
  if (integ) ZC_CUDA(cudaMemcpy(integ, h->integ, fE, cudaMemcpyDeviceToHost));
  if (eprev) ZC_CUDA(cudaMemcpy(eprev, h->eprev, fE, cudaMemcpyDeviceToHost));
  if (eta) ZC_CUDA(cudaMemcpy(eta, h->eta, sizeof(float), cudaMemcpyDeviceToHost));
  if (counts) ZC_CUDA(cudaMemcpy(counts, h->acc_counts, (size_t)h->E * sizeof(int64_t), cudaMemcpyDeviceToHost));
  if (tokens) ZC_CUDA(cudaMemcpy(tokens, h->acc_tokens, sizeof(int64_t), cudaMemcpyDeviceToHost));
  return ZCMOE_OK;
}

int zcmoe_set_controller(zcmoe_t h, const float* bias, const float* integ, const float* eprev, const float* eta,
                         const int64_t* counts, const int64_t* tokens) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!bias || !integ || !eprev || !eta || !counts || !tokens) return fail(ZCMOE_EINVAL, "a state pointer is NULL");
  if (!std::isfinite(*eta)) return fail(ZCMOE_EINVAL, "eta must be finite");
  if (*tokens < 0) return fail(ZCMOE_EINVAL, "tokens must be >= 0");
  for (int i = 0; i < h->E; ++i)
    if (counts[i] < 0) return fail(ZCMOE_EINVAL, "counts must be >= 0 (expert %d)", i);
  ZC_CUDA(cudaDeviceSynchronize());
  const size_t fE = (size_t)h->E * sizeof(float);
  ZC_CUDA(cudaMemcpy(h->bias, bias, fE, cudaMemcpyHostToDevice));
  ZC_CUDA(cudaMemcpy(h->integ, integ, fE, cudaMemcpyHostToDevice));
  ZC_CUDA(cudaMemcpy(h->eprev, eprev, fE, cudaMemcpyHostToDevice));
  ZC_CUDA(cudaMemcpy(h->eta, eta, sizeof(float), cudaMemcpyHostToDevice));
  ZC_CUDA(cudaMemcpy(h->acc_counts, counts, (size_t)h->E * sizeof(int64_t), cudaMemcpyHostToDevice));
  ZC_CUDA(cudaMemcpy(h->acc_tokens, tokens, sizeof(int64_t), cudaMemcpyHostToDevice));
  return ZCMOE_OK;
}

int zcmoe_check(zcmoe_t h) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  ZC_CUDA(cudaDeviceSynchronize());
  int code = 0;
  ZC_CUDA(cudaMemcpy(&code, h->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (code) {
    ZC_CUDA(cudaMemset(h->err, 0, sizeof(int)));
    return fail(ZCMOE_ETIMEOUT, "a device-side wait timed out (site %d)", code);
  }
  return ZCMOE_OK;
}

int zcmoe_profile_begin(zcmoe_t h) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!h->events) h->events = new (std::nothrow) std::vector<cudaEvent_t>();
  if (!h->events) return fail(ZCMOE_ENOMEM, "host allocation failed");
  for (cudaEvent_t e : *h->events) cudaEventDestroy(e);
  h->events->clear();
  h->profiling = true;
  return ZCMOE_OK;
}

int zcmoe_profile_end(zcmoe_t h, float* ms, int32_t* n_forwards) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!h->profiling || !h->events) return fail(ZCMOE_EINVAL, "profiling was not started");
  h->profiling = false;
  ZC_CUDA(cudaDeviceSynchronize());
  const size_t per = ZCMOE_NUM_STAGES + 1;
  const size_t n = h->events->size() / per;
  for (int i = 0; i < ZCMOE_NUM_STAGES; ++i) ms[i] = 0.0f;
  for (size_t f = 0; f < n; ++f) {
    for (int i = 0; i < ZCMOE_NUM_STAGES; ++i) {
      float t = 0.0f;
      ZC_CUDA(cudaEventElapsedTime(&t, (*h->events)[f * per + i], (*h->events)[f * per + i + 1]));
      ms[i] += t;
    }
  }
  if (n_forwards) *n_forwards = (int32_t)n;
  for (cudaEvent_t e : *h->events) cudaEventDestroy(e);
  h->events->clear();
  return ZCMOE_OK;
}

int zcmoe_selftest_wait(zcmoe_t h, int64_t limit_ns, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (limit_ns < 1000 || limit_ns > 1000000000LL) return fail(ZCMOE_EINVAL, "limit_ns must lie in [1e3, 1e9]");
  ZC_CUDA(zc::launch_selftest_wait(h->err, (uint64_t)limit_ns, s));
  return ZCMOE_OK;
}

int zcmoe_destroy(zcmoe_t h) {
  g_err[0] = 0;
  if (!h) return ZCMOE_OK;
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    if (!g_live.erase(h)) return fail(ZCMOE_EINVAL, "invalid or already destroyed handle");
  }
  h->alive = false;
  cudaDeviceSynchronize();
  release(h);
  delete h;
  return ZCMOE_OK;
}

int zcmoe_save_for_backward(zcmoe_t h, int32_t on) {
  g_err[0] = 0;
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!h->bf16 || h->fp8) return fail(ZCMOE_EUNSUPPORTED, "training mode needs a bf16 layer");
  if (h->ep_size > 1) return fail(ZCMOE_EUNSUPPORTED, "training mode needs a layer that holds all experts");
  if (!on) {
    if (h->b_gu) {
      ZC_CUDA(cudaDeviceSynchronize());
      cudaFree(h->b_gu);
      h->b_gu = nullptr;
    }
    h->last_saved = false;
    return ZCMOE_OK;
  }
  if (h->b_gu) return ZCMOE_OK;
  uint8_t* p = nullptr;
  const int rc = dalloc(&p, (size_t)h->max_mblocks * zc::kBM * h->inter * 4);
  if (rc != ZCMOE_OK) return rc;
  h->b_gu = p;
  return ZCMOE_OK;
}

int zcmoe_backward_ex(zcmoe_t h, const void* x, const void* dy, int64_t T, void* dx, float* g_router, float* g_gate,
                      float* g_up, float* g_down, uint32_t flags, cudaStream_t s) {
  g_err[0] = 0;
  if (flags & ~(uint32_t)ZCMOE_GRAD_OVERWRITE) return fail(ZCMOE_EINVAL, "unknown flags 0x%x", flags);
  if (!is_live(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!h->bf16 || h->fp8) return fail(ZCMOE_EUNSUPPORTED, "the backward pass needs a bf16 layer");
  if (h->ep_size > 1) return fail(ZCMOE_EUNSUPPORTED, "the backward pass needs a layer that holds all experts");
  if (T < 0 || T > h->max_T) return fail(ZCMOE_ERANGE, "T=%lld outside [0, %d]", (long long)T, h->max_T);
  if (T == 0) return ZCMOE_OK;
  if (T != h->last_T) return fail(ZCMOE_EINVAL, "T=%lld differs from the last forward's %d", (long long)T, h->last_T);
  if (!x || !dy || !dx) return fail(ZCMOE_EINVAL, "x, dy or dx is NULL");
  const void* bufs[3] = {x, dy, dx};
  for (const void* p : bufs)
    if (reinterpret_cast<uintptr_t>(p) & 15u) return fail(ZCMOE_EINVAL, "x, dy and dx must be 16-byte aligned");
  const size_t nb = (size_t)T * h->d * 2;
  if (overlaps(dx, nb, x, nb) || overlaps(dx, nb, dy, nb)) return fail(ZCMOE_EINVAL, "dx overlaps x or dy");
  if (h->d > 24576) return fail(ZCMOE_EUNSUPPORTED, "the backward pass supports d <= 24576");
  const int Ti = (int)T, E = h->E, N = h->N, k = h->k, d = h->d, inter = h->inter;
  const size_t prow = (size_t)h->max_mblocks * zc::kBM;
  if (!h->b_xpad) {
    h->dl_ld = (E + 63) / 64 * 64;
    int rc = ZCMOE_OK;
    uint8_t *a = nullptr, *b = nullptr, *c = nullptr, *e2 = nullptr, *f = nullptr, *g = nullptr, *l = nullptr,
            *r = nullptr;
    rc = dalloc(&a, prow * d * 2);
    if (rc == ZCMOE_OK) rc = dalloc(&b, prow * d * 2);
    if (rc == ZCMOE_OK) rc = dalloc(&c, prow * inter * 2);
    if (rc == ZCMOE_OK) rc = dalloc(&e2, prow * inter * 4);
    if (rc == ZCMOE_OK) rc = dalloc(&f, prow * inter * 2);
    if (rc == ZCMOE_OK) rc = dalloc(&g, prow * d * 2);
    if (rc == ZCMOE_OK) rc = dalloc(&l, (size_t)h->max_T * h->dl_ld * 2);
    if (rc == ZCMOE_OK) rc = dalloc(&r, (size_t)h->max_T * d * 2);
    if (rc == ZCMOE_OK) rc = dalloc(&h->b_dg, (size_t)h->max_pairs);
    if (rc == ZCMOE_OK) rc = dalloc(&h->b_grp, 4);
    h->b_xpad = a;
    h->b_dypad = b;
    h->b_dh = c;
    h->b_dgu = e2;
    h->b_hpad = f;
    h->b_dxp = g;
    h->b_dl = l;
    h->b_dxr = r;
    if (rc != ZCMOE_OK) {
      void* ps[] = {h->b_xpad, h->b_dypad, h->b_dh, h->b_dgu, h->b_hpad, h->b_dxp, h->b_dl, h->b_dxr, h->b_dg, h->b_grp};
      for (void* p : ps)
        if (p) cudaFree(p);
      h->b_xpad = h->b_dypad = h->b_dh = h->b_dgu = h->b_hpad = h->b_dxp = h->b_dl = h->b_dxr = nullptr;
      h->b_dg = nullptr;
      h->b_grp = nullptr;
      return rc;
    }
  }
  const uint64_t P = prow;
  CUtensorMap tm_dy_k, tm_wd_mn, tm_x_k, tm_dgu_k, tm_wg_mn, tm_wu_mn, tm_dl_k, tm_wr_mn;
  CUtensorMap tm_dy_mn, tm_h_mn, tm_dgu_mn, tm_x_mn, tm_dl_mn, tm_xin_mn;
  int rc = make_tmap(&tm_dy_k, h->b_dypad, d, P, 128);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_wd_mn, h->w.w_down, inter, (uint64_t)N * d, 64);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_x_k, h->b_xpad, d, P, 128);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_dgu_k, h->b_dgu, 2 * (uint64_t)inter, P, 128);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_wg_mn, h->w.w_gate, d, (uint64_t)N * inter, 64);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_wu_mn, h->w.w_up, d, (uint64_t)N * inter, 64);
  if (rc == ZCMOE_OK) rc = make_tmap_ld(&tm_dl_k, h->b_dl, E, T, 128, h->dl_ld);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_wr_mn, h->w.w_router, d, E, 64);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_dy_mn, h->b_dypad, d, P, 64);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_h_mn, h->b_hpad, inter, P, 64);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_dgu_mn, h->b_dgu, 2 * (uint64_t)inter, P, 64);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_x_mn, h->b_xpad, d, P, 64);
  if (rc == ZCMOE_OK) rc = make_tmap_ld(&tm_dl_mn, h->b_dl, E, T, 64, h->dl_ld);
  if (rc == ZCMOE_OK) rc = make_tmap(&tm_xin_mn, x, d, T, 64);
  if (rc != ZCMOE_OK) return rc;
  const int max_mb = (Ti * k + zc::kBM - 1) / zc::kBM + N;
  auto grid_for = [&](int64_t tiles) { return (int)(tiles < h->sms ? (tiles < 1 ? 1 : tiles) : h->sms); };
  auto rows_args = [&]() {
    zc::BwdArgs a{};
    a.ngroups = N;
    a.row_off = h->offsets;
    a.mb_off = h->mb_off;
    a.k_split = 0x7fffffff;
    a.err = h->err;
    return a;
  };

  // routing-side backward and the padded operands
  ZC_CUDA(zc::launch_single_group(h->b_grp, h->b_grp + 2, Ti, s));
  ZC_CUDA(zc::launch_gather_pad(x, d, h->perm, k, h->offsets, h->mb_off, N, h->b_xpad, h->b_dypad, h->sms, s));
  ZC_CUDA(zc::launch_combine_bwd(x, dy, h->Y, h->gate, h->pos, h->idx, h->offsets, h->mb_off, Ti, k, d, h->b_dypad,
                                 h->b_dg, s));
  ZC_CUDA(zc::launch_router_bwd(h->logits, Ti, E, k, h->cfg.routed_scale, h->idx, h->b_dg,
                                static_cast<__nv_bfloat16*>(h->b_dl), h->dl_ld, h->sms, s));
  if (h->last_saved) {
    // dH = dY W_d with the SwiGLU backward in its epilogue, on the forward's G and U
    zc::BwdArgs a = rows_args();
    a.K = d;
    a.n_out = inter;
    a.nblocks = (inter + 255) / 256;
    a.b_row_per_group = d;
    a.gu = static_cast<const __nv_bfloat16*>(h->b_gu);
    a.dgu = static_cast<__nv_bfloat16*>(h->b_dgu);
    a.hpad = static_cast<__nv_bfloat16*>(h->b_hpad);
    a.inter = inter;
    CUtensorMap tm_dgu_st, tm_h_st;  // store targets: [dG | dU] (as c) and H (as the unused second B)
    if ((rc = make_tmap_store32(&tm_dgu_st, h->b_dgu, 2 * (uint64_t)inter, P)) != ZCMOE_OK) return rc;
    if ((rc = make_tmap_store32(&tm_h_st, h->b_hpad, (uint64_t)inter, P)) != ZCMOE_OK) return rc;
    ZC_CUDA(zc::launch_bwd_gemm(zc::kBwdDhSwiglu, tm_dy_k, tm_wd_mn, tm_h_st, tm_dgu_st, a,
                                grid_for((int64_t)max_mb * a.nblocks), s));
  }
  // dH = dY W_d
  if (!h->last_saved) {
    zc::BwdArgs a = rows_args();
    a.K = d;
    a.n_out = inter;
    a.nblocks = (inter + 255) / 256;
    a.b_row_per_group = d;
    a.out = h->b_dh;
    a.ldo = inter;
    CUtensorMap tm_dh_st;
    if ((rc = make_tmap(&tm_dh_st, h->b_dh, (uint64_t)inter, P, 32)) != ZCMOE_OK) return rc;
    ZC_CUDA(zc::launch_bwd_gemm(zc::kBwdRowsMnB, tm_dy_k, tm_wd_mn, tm_wd_mn, tm_dh_st, a,
                                grid_for((int64_t)max_mb * a.nblocks), s));
  }
  // [G|U] recomputed from X; SwiGLU backward -> dG, dU; H
  if (!h->last_saved) {
    zc::BwdArgs a = rows_args();
    a.K = d;
    a.n_out = inter;
    a.nblocks = (inter + 127) / 128;
    a.b_row_per_group = inter;
    a.dh = static_cast<const __nv_bfloat16*>(h->b_dh);
    a.dgu = static_cast<__nv_bfloat16*>(h->b_dgu);
    a.hpad = static_cast<__nv_bfloat16*>(h->b_hpad);
    a.inter = inter;
    ZC_CUDA(zc::launch_bwd_gemm(zc::kBwdSwiglu, tm_x_k, h->tm_wg, h->tm_wu, tm_x_k, a, grid_for((int64_t)max_mb * a.nblocks),
                                s));
  }
  // dX = [dG|dU] [W_g; W_u]
  {
    zc::BwdArgs a = rows_args();
    a.K = 2 * inter;
    a.k_split = inter;
    a.n_out = d;
    a.nblocks = (d + 255) / 256;
    a.b_row_per_group = inter;
    a.out = h->b_dxp;
    a.ldo = d;
    CUtensorMap tm_dxp_st;
    if ((rc = make_tmap(&tm_dxp_st, h->b_dxp, (uint64_t)d, P, 32)) != ZCMOE_OK) return rc;
    ZC_CUDA(zc::launch_bwd_gemm(zc::kBwdRowsMnB, tm_dgu_k, tm_wg_mn, tm_wu_mn, tm_dxp_st, a,
                                grid_for((int64_t)max_mb * a.nblocks), s));
  }
  // router: dx_router = dl W_r
  {
    zc::BwdArgs a{};
    a.ngroups = 1;
    a.row_off = h->b_grp;
    a.mb_off = h->b_grp + 2;
    a.k_split = 0x7fffffff;
    a.err = h->err;
    a.K = h->dl_ld;
    a.n_out = d;
    a.nblocks = (d + 255) / 256;
    a.b_row_per_group = 0;
    a.out = h->b_dxr;
    a.ldo = d;
    CUtensorMap tm_dxr_st;
    if ((rc = make_tmap(&tm_dxr_st, h->b_dxr, (uint64_t)d, (uint64_t)T, 32)) != ZCMOE_OK) return rc;
    ZC_CUDA(zc::launch_bwd_gemm(zc::kBwdRowsMnB, tm_dl_k, tm_wr_mn, tm_wr_mn, tm_dxr_st, a,
                                grid_for((int64_t)((Ti + 127) / 128) * a.nblocks), s));
  }
  // dx: the deterministic ScatterAdd
  ZC_CUDA(zc::launch_final_dx(dy, h->b_dxp, h->b_dxr, h->gate, h->pos, h->idx, h->offsets, h->mb_off, Ti, k, d, dx, s));
  // weight gradients, added into the fp32 accumulators in the GEMM epilogue
  // acc2 (optional): a second accumulator of the same shape for A's next m_out columns, so that
  // one launch reads B once for both (dW_g and dW_u over [dG | dU] and X)
  auto wgrad = [&](const CUtensorMap& A, const CUtensorMap& B, int a_col0, int m_out, int n_out, float* acc,
                   int64_t stride, int groups, const int32_t* row_off, const int32_t* mb_off,
                   float* acc2 = nullptr) -> int {
    zc::BwdArgs a{};
    a.ngroups = groups;
    a.row_off = row_off;
    a.mb_off = mb_off;
    a.a_col0 = a_col0;
    a.m_out = acc2 ? 2 * m_out : m_out;
    a.m_split = acc2 ? m_out : 0;
    a.mblocks = (a.m_out + 127) / 128;
    a.n_out = n_out;
    a.nblocks = (n_out + 255) / 256;
    a.acc = acc;
    a.overwrite = (flags & ZCMOE_GRAD_OVERWRITE) ? 1 : 0;
    a.acc_ld = n_out;
    a.acc_group_stride = stride;
    a.err = h->err;
    CUtensorMap tmc, tmc2;
    int rc2 = make_tmap_acc(&tmc, acc, (uint64_t)n_out, (uint64_t)m_out, (uint64_t)groups);
    if (rc2 == ZCMOE_OK && acc2) rc2 = make_tmap_acc(&tmc2, acc2, (uint64_t)n_out, (uint64_t)m_out, (uint64_t)groups);
    if (rc2 != ZCMOE_OK) return rc2;
    ZC_CUDA(zc::launch_bwd_gemm(zc::kBwdWgrad, A, B, acc2 ? tmc2 : B, tmc, a,
                                grid_for((int64_t)groups * a.mblocks * a.nblocks), s));
    return ZCMOE_OK;
  };
  if (g_down && (rc = wgrad(tm_dy_mn, tm_h_mn, 0, d, inter, g_down, (int64_t)d * inter, N, h->offsets, h->mb_off)))
    return rc;
  if (g_gate && g_up) {  // both from one launch over [dG | dU]: X is read once
    if ((rc = wgrad(tm_dgu_mn, tm_x_mn, 0, inter, d, g_gate, (int64_t)inter * d, N, h->offsets, h->mb_off, g_up)))
      return rc;
  } else {
    if (g_gate && (rc = wgrad(tm_dgu_mn, tm_x_mn, 0, inter, d, g_gate, (int64_t)inter * d, N, h->offsets, h->mb_off)))
      return rc;
    if (g_up && (rc = wgrad(tm_dgu_mn, tm_x_mn, inter, inter, d, g_up, (int64_t)inter * d, N, h->offsets, h->mb_off)))
      return rc;
  }
  if (g_router && (rc = wgrad(tm_dl_mn, tm_xin_mn, 0, E, d, g_router, 0, 1, h->b_grp, h->b_grp + 2))) return rc;
  return ZCMOE_OK;
}

int zcmoe_backward(zcmoe_t h, const void* x, const void* dy, int64_t T, void* dx, float* g_router, float* g_gate,
                   float* g_up, float* g_down, cudaStream_t s) {
  return zcmoe_backward_ex(h, x, dy, T, dx, g_router, g_gate, g_up, g_down, 0u, s);
}

int zcmoe_quantize_e4m3(const void* src, int32_t src_dtype, int64_t rows, int64_t cols, int32_t block_rows,
                        uint8_t* codes, uint8_t* scales, cudaStream_t s) {
  g_err[0] = 0;
  if (src_dtype != ZCMOE_BF16 && src_dtype != ZCMOE_F32) return fail(ZCMOE_EINVAL, "src_dtype must be BF16 or F32");
  if (block_rows != 1 && block_rows != 128) return fail(ZCMOE_EINVAL, "block_rows must be 1 or 128");
  if (rows < 0 || cols <= 0 || cols % 128 || cols > (1 << 30)) return fail(ZCMOE_EINVAL, "bad rows / cols");
  if (rows == 0) return ZCMOE_OK;
  if (block_rows == 128 && (rows + 127) / 128 > 65535) return fail(ZCMOE_ERANGE, "too many row blocks");
  if (!src || !codes || !scales) return fail(ZCMOE_EINVAL, "a pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(codes) & 15u))
    return fail(ZCMOE_EINVAL, "src and codes must be 16-byte aligned");
  int dev = 0, sms = 0;
  ZC_CUDA(cudaGetDevice(&dev));
  ZC_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int bf16 = src_dtype == ZCMOE_BF16;
  if (block_rows == 1)
    ZC_CUDA(zc::launch_quant_rows(bf16, src, rows, (int)cols, codes, scales, 0, sms, s));
  else
    ZC_CUDA(zc::launch_quant_tiles(bf16, src, rows, (int)cols, codes, scales, 0, s));
  return ZCMOE_OK;
}

int zcmoe_quantize_mx4(const void* src, int32_t src_dtype, int64_t rows, int64_t cols, uint8_t* codes,
                       uint8_t* scales, cudaStream_t s) {
  g_err[0] = 0;
  if (src_dtype != ZCMOE_BF16 && src_dtype != ZCMOE_F32) return fail(ZCMOE_EINVAL, "src_dtype must be BF16 or F32");
  if (rows < 0 || cols <= 0 || cols % 256 || cols > (1 << 30)) return fail(ZCMOE_EINVAL, "bad rows / cols");
  if (rows == 0) return ZCMOE_OK;
  if (!src || !codes || !scales) return fail(ZCMOE_EINVAL, "a pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(codes) & 15u))
    return fail(ZCMOE_EINVAL, "src and codes must be 16-byte aligned");
  int dev = 0, sms = 0;
  ZC_CUDA(cudaGetDevice(&dev));
  ZC_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  ZC_CUDA(zc::launch_quant_mx4(src_dtype == ZCMOE_BF16, src, rows, (int)cols, codes, scales, 0, sms, s));
  return ZCMOE_OK;
}

int zcmoe_quantize_nv4(const void* src, int32_t src_dtype, int64_t rows, int64_t cols, float global_scale,
                       uint8_t* codes, uint8_t* scales, float* global_out, cudaStream_t s) {
  g_err[0] = 0;
  if (src_dtype != ZCMOE_BF16 && src_dtype != ZCMOE_F32) return fail(ZCMOE_EINVAL, "src_dtype must be BF16 or F32");
  if (rows < 0 || cols <= 0 || cols % 256 || cols > (1 << 30)) return fail(ZCMOE_EINVAL, "bad rows / cols");
  if (!(std::isfinite(global_scale) && global_scale >= 0.0f))
    return fail(ZCMOE_EINVAL, "global_scale must be finite and >= 0 (0: derived from the tensor)");
  if (global_scale == 0.0f && !global_out) return fail(ZCMOE_EINVAL, "global_out is NULL (needed when global_scale is 0)");
  if (rows == 0) return ZCMOE_OK;
  if (!src || !codes || !scales) return fail(ZCMOE_EINVAL, "a pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(codes) & 15u) ||
      (reinterpret_cast<uintptr_t>(global_out) & 3u))
    return fail(ZCMOE_EINVAL, "src and codes must be 16-byte aligned, global_out 4-byte aligned");
  int dev = 0, sms = 0;
  ZC_CUDA(cudaGetDevice(&dev));
  ZC_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int bf16 = src_dtype == ZCMOE_BF16;
  if (global_scale == 0.0f) {
    ZC_CUDA(zc::launch_nv4_global(bf16, src, 1, rows, (int)cols, global_out, s));
    ZC_CUDA(zc::launch_quant_nv4(bf16, src, rows, (int)cols, codes, scales, 0, global_out, rows, 1.0f, sms, s));
  } else {
    ZC_CUDA(zc::launch_quant_nv4(bf16, src, rows, (int)cols, codes, scales, 0, nullptr, 1, global_scale, sms, s));
  }
  return ZCMOE_OK;
}

// ---------------------------------------------------------------- dense FFN path and the overlap

int zcmoe_dense_create(const zcmoe_dense_config* cfg, const zcmoe_dense_weights* w, zcmoe_dense_t* out) {
  g_err[0] = 0;
  if (!out) return fail(ZCMOE_EINVAL, "out is NULL");
  *out = nullptr;
  if (!cfg || !w) return fail(ZCMOE_EINVAL, "cfg or weights is NULL");
  if (cfg->d < 64 || cfg->d % 64 || cfg->inter < 64 || cfg->inter % 64)
    return fail(ZCMOE_EINVAL, "d and inter must be positive multiples of 64");
  if (cfg->max_tokens < 1 || cfg->max_tokens > (1 << 20)) return fail(ZCMOE_EINVAL, "need 1 <= max_tokens <= 2^20");
  if (!w->w_gate || !w->w_up || !w->w_down) return fail(ZCMOE_EINVAL, "a weight pointer is NULL");
  const void* wp[3] = {w->w_gate, w->w_up, w->w_down};
  for (const void* p : wp)
    if (reinterpret_cast<uintptr_t>(p) & 15u) return fail(ZCMOE_EINVAL, "weight pointers must be 16-byte aligned");

  int dev = 0;
  ZC_CUDA(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  ZC_CUDA(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10) return fail(ZCMOE_EUNSUPPORTED, "device %d is sm_%d%d; this library targets sm_100a", dev,
                                    prop.major, prop.minor);
  if (prop.sharedMemPerBlockOptin < (size_t)zc::tc_smem_bytes())
    return fail(ZCMOE_EUNSUPPORTED, "not enough shared memory per block");

  zcmoe_dense_s* h = new (std::nothrow) zcmoe_dense_s();
  if (!h) return fail(ZCMOE_ENOMEM, "host allocation failed");
  memset(h, 0, sizeof(*h));
  h->d = cfg->d;
  h->inter = cfg->inter;
  h->max_T = cfg->max_tokens;
  h->sms = prop.multiProcessorCount;
  h->w = *w;
  const size_t hbytes = (size_t)h->max_T * h->inter * 2;
  uint8_t* hh = nullptr;
  int rc = dalloc(&hh, hbytes);
  h->H = hh;
  if (rc == ZCMOE_OK) rc = dalloc(&h->offs, 8);
  if (rc == ZCMOE_OK) rc = dalloc(&h->err, 1);
  if (rc == ZCMOE_OK) {
    cudaError_t e = cudaMemset(h->H, 0, hbytes);
    if (e == cudaSuccess) e = cudaMemset(h->offs, 0, 8 * sizeof(int32_t));
    if (e == cudaSuccess) e = cudaMemset(h->err, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_router, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_down, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) rc = fail(ZCMOE_ECUDA, "initialising the dense handle: %s", cudaGetErrorString(e));
  }
  if (rc == ZCMOE_OK) rc = make_tmap(&h->tm_wg, w->w_gate, (uint64_t)h->d, (uint64_t)h->inter, 128);
  if (rc == ZCMOE_OK) rc = make_tmap(&h->tm_wu, w->w_up, (uint64_t)h->d, (uint64_t)h->inter, 128);
  if (rc == ZCMOE_OK) rc = make_tmap(&h->tm_wd, w->w_down, (uint64_t)h->inter, (uint64_t)h->d, 256);
  if (rc == ZCMOE_OK) rc = make_tmap(&h->tm_h, h->H, (uint64_t)h->inter, (uint64_t)h->max_T, 128);
  if (rc != ZCMOE_OK) {
    release_dense(h);
    delete h;
    return rc;
  }
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    g_live_dense.insert(h);
  }
  *out = h;
  return ZCMOE_OK;
}

int zcmoe_dense_forward(zcmoe_dense_t h, const void* x, int64_t T, void* y, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live_dense(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed dense handle");
  if (T < 0 || T > h->max_T) return fail(ZCMOE_ERANGE, "T=%lld outside [0, %d]", (long long)T, h->max_T);
  if (T == 0) return ZCMOE_OK;
  if (!x || !y) return fail(ZCMOE_EINVAL, "x or y is NULL");
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u))
    return fail(ZCMOE_EINVAL, "x and y must be 16-byte aligned");
  const size_t nb = (size_t)T * h->d * 2;
  if (overlaps(x, nb, y, nb)) return fail(ZCMOE_EINVAL, "y overlaps x");
  const int rc = dense_gate_up(h, x, (int)T, s);
  if (rc != ZCMOE_OK) return rc;
  return dense_down(h, (int)T, y, s);
}

int zcmoe_forward_overlap(zcmoe_t moe, zcmoe_dense_t dense, const void* x_moe, const void* x_dense, int64_t T,
                          void* y_moe, void* y_dense, cudaStream_t s) {
  g_err[0] = 0;
  if (!is_live(moe)) return fail(ZCMOE_EINVAL, "invalid or destroyed handle");
  if (!is_live_dense(dense)) return fail(ZCMOE_EINVAL, "invalid or destroyed dense handle");
  if (!moe->bf16) return fail(ZCMOE_EUNSUPPORTED, "the overlap needs a bf16 MoE handle");
  if (moe->d != dense->d) return fail(ZCMOE_EINVAL, "hidden sizes differ (%d vs %d)", moe->d, dense->d);
  if (T < 0 || T > moe->max_T || T > dense->max_T)
    return fail(ZCMOE_ERANGE, "T=%lld outside [0, %d]", (long long)T,
                moe->max_T < dense->max_T ? moe->max_T : dense->max_T);
  if (T == 0) return ZCMOE_OK;
  if (!x_moe || !x_dense || !y_moe || !y_dense) return fail(ZCMOE_EINVAL, "a buffer is NULL");
  const void* bufs[4] = {x_moe, x_dense, y_moe, y_dense};
  for (const void* p : bufs)
    if (reinterpret_cast<uintptr_t>(p) & 15u) return fail(ZCMOE_EINVAL, "buffers must be 16-byte aligned");
  const size_t nb = (size_t)T * moe->d * 2;
  if (overlaps(y_moe, nb, y_dense, nb) || overlaps(y_moe, nb, x_moe, nb) || overlaps(y_moe, nb, x_dense, nb) ||
      overlaps(y_dense, nb, x_moe, nb) || overlaps(y_dense, nb, x_dense, nb))
    return fail(ZCMOE_EINVAL, "an output overlaps another buffer");
  const DenseSide side{dense, x_dense, y_dense};
  const int rc = forward_impl(moe, x_moe, T, y_moe, s, nullptr, &side);
  if (rc != ZCMOE_OK) {
    // best effort: leave no work of the side stream unjoined
    if (cudaEventRecord(dense->ev_join, dense->side) == cudaSuccess) cudaStreamWaitEvent(s, dense->ev_join, 0);
    cudaGetLastError();
  }
  return rc;
}

int zcmoe_dense_check(zcmoe_dense_t h) {
  g_err[0] = 0;
  if (!is_live_dense(h)) return fail(ZCMOE_EINVAL, "invalid or destroyed dense handle");
  ZC_CUDA(cudaDeviceSynchronize());
  int code = 0;
  ZC_CUDA(cudaMemcpy(&code, h->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (code) {
    ZC_CUDA(cudaMemset(h->err, 0, sizeof(int)));
    return fail(ZCMOE_ETIMEOUT, "a device-side wait timed out (site %d)", code);
  }
  return ZCMOE_OK;
}

int zcmoe_dense_destroy(zcmoe_dense_t h) {
  g_err[0] = 0;
  if (!h) return ZCMOE_OK;
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    if (!g_live_dense.erase(h)) return fail(ZCMOE_EINVAL, "invalid or already destroyed dense handle");
  }
  cudaDeviceSynchronize();
  release_dense(h);
  delete h;
  return ZCMOE_OK;
}

}  // extern "C"
