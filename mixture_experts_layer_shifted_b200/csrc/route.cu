// Routing, integer stage, row gather, combine and bias controller kernels.
//
// Sources (page title, section):
//  - LongCat-Flash technical summary (zhangjingwei.cn), 二 架構, part 1
//    "零計算專家": zero experts return the input at no cost; an expert-specific
//    bias shifts the routing scores; a PID controller keeps the FFN/zero
//    selection ratio near a target.
//  - LongCat-Flash tech-report thread (web3.cnouyi.fund): DeepSeek-V3-like
//    auxiliary-loss-free bias (selection only) with a decay schedule.
//  - LongCat-Flash-Lite N-gram article (onthewifi.com), part 02: the router is a
//    fused softmax + top-k + scaling step.
//
// The routing of a token (softmax, bias-shifted top-k, gates) and its written
// fp32 rule live in zc_route.cuh.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_internal.h"
#include "zc_ptx.cuh"
#include "zc_route.cuh"

namespace zc {
namespace {

// One warp per token (route_token in zc_route.cuh); the stand-alone routing kernel,
// for layers whose router logits come from elsewhere (fp32 layers, zcmoe_route_noalloc).
template <int EPL>
__global__ void __launch_bounds__(256, 3) k_softmax_topk(const float* __restrict__ logits, const float* __restrict__ bias,
                                                         int T, int E, int k, float scale, int32_t* __restrict__ idx,
                                                         float* __restrict__ gate, float* __restrict__ scores) {
  __shared__ uint32_t slots[8][96];  // per warp: the candidates' keys, ids and scores
  const int lane = threadIdx.x & 31;
  const int warp = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
  for (int t = warp; t < T; t += nwarps)
    route_token<EPL>(logits + (int64_t)t * E, bias, E, k, scale, idx + (int64_t)t * k, gate + (int64_t)t * k,
                     scores ? scores + (int64_t)t * E : nullptr, lane, slots[threadIdx.x >> 5]);
}

// Router backward, one warp per token: the scores s are recomputed from the
// saved logits exactly as k_softmax_topk computes them; ds_e = scale * dg of the
// slot that picked e (0 for experts not picked); dl = s * (ds - <s, ds>), bf16
// into dl [T, ld].  The bias only selected and gets no gradient.
template <int EPL>
__global__ void __launch_bounds__(256) k_router_bwd(const float* __restrict__ logits, int T, int E, int k,
                                                    float scale, const int32_t* __restrict__ idx,
                                                    const float* __restrict__ dg, __nv_bfloat16* __restrict__ dl,
                                                    int ld) {
  const int lane = threadIdx.x & 31;
  const int warp = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
  for (int t = warp; t < T; t += nwarps) {
    const float* lt = logits + (int64_t)t * E;
    float l[EPL];
    float m = -__int_as_float(0x7f800000);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      l[i] = e < E ? lt[e] : -__int_as_float(0x7f800000);
      m = fmaxf(m, l[i]);
    }
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, w));
    float u[EPL];
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      u[i] = 0.0f;
      if (e < E) {
        u[i] = zexp(__fsub_rn(l[i], m));
        acc = __fadd_rn(acc, u[i]);
      }
    }
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, w));
    float ds[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      u[i] = __fdiv_rn(u[i], acc);
      ds[i] = 0.0f;
    }
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)t * k + j];
      if ((e & 31) == lane) {
        const float v = scale * dg[(int64_t)t * k + j];
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          if (i == (e >> 5)) ds[i] = v;
      }
    }
    float dot = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) dot = fmaf(u[i], ds[i], dot);
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, w);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < ld) dl[(int64_t)t * ld + e] = __float2bfloat16_rn(e < E ? u[i] * (ds[i] - dot) : 0.0f);
    }
  }
}

// Integer stage, part 1: per block of 256 tokens, one 32-bit token mask per
// (warp, expert) in shared memory; writes the block's per-expert counts.
__global__ void __launch_bounds__(kChunk) k_route_count(const int32_t* __restrict__ idx, int T, int k, int E,
                                                        int32_t* __restrict__ chunk_cnt) {
  extern __shared__ uint32_t smask[];  // [8][E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 8 * E; i += kChunk) smask[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kChunk + tid;
  if (t < T)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)t * k + j];
      if ((unsigned)e < (unsigned)E) atomicOr(&smask[warp * E + e], 1u << lane);  // an id out of range is skipped
    }
  __syncthreads();
  for (int e = tid; e < E; e += kChunk) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) c += __popc(smask[w * E + e]);
    chunk_cnt[(int64_t)blockIdx.x * E + e] = c;
  }
}

// Block-wide exclusive scan of two ints (1024 threads).
__device__ __forceinline__ int2 block_exclusive_scan2(int2 v, int2* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int2 inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, inc.x, o);
    const int b = __shfl_up_sync(0xffffffffu, inc.y, o);
    if (lane >= o) {
      inc.x += a;
      inc.y += b;
    }
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int2 w = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : make_int2(0, 0);
    int2 wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, wi.x, o);
      const int b = __shfl_up_sync(0xffffffffu, wi.y, o);
      if (lane >= o) {
        wi.x += a;
        wi.y += b;
      }
    }
    warp_tot[lane] = make_int2(wi.x - w.x, wi.y - w.y);
  }
  __syncthreads();
  const int2 base = warp_tot[warp];
  return make_int2(base.x + inc.x - v.x, base.y + inc.y - v.y);
}

// Integer stage, part 2 (one block of 1024 threads, thread = expert): totals,
// controller accumulation, exclusive scans over FFN experts of the counts, of
// their 128-row block counts and (sp_off, when asked) of their row-block pairs
// ceil(blocks / 2), and the first permuted row of every (token block, expert)
// pair, written over chunk_cnt.
__global__ void __launch_bounds__(1024) k_route_scan(int32_t* __restrict__ chunk_cnt, int nchunks, int T, int N, int E,
                                                     int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                     int32_t* __restrict__ mb_off, int32_t* __restrict__ scal,
                                                     int64_t* __restrict__ acc_counts, int64_t* __restrict__ acc_tokens,
                                                     int32_t* __restrict__ sp_off) {
  __shared__ int2 warp_tot[32];
  __shared__ int2 warp_tot2[32];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
#pragma unroll 8
    for (int c = 0; c < nchunks; ++c) total += chunk_cnt[(int64_t)c * E + e];
    counts[e] = total;
    acc_counts[e] += total;
  }
  const int2 v = (e < N) ? make_int2(total, (total + kBM - 1) / kBM) : make_int2(0, 0);
  const int2 ex = block_exclusive_scan2(v, warp_tot);
  const int2 v2 = make_int2((v.y + 1) / 2, 0);
  const int2 ex2 = sp_off ? block_exclusive_scan2(v2, warp_tot2) : make_int2(0, 0);
  if (e < N) {
    offsets[e] = ex.x;
    mb_off[e] = ex.y;
    if (sp_off) sp_off[e] = ex2.x;
    if (e == N - 1) {
      offsets[N] = ex.x + v.x;
      mb_off[N] = ex.y + v.y;
      if (sp_off) sp_off[N] = ex2.x + v2.x;
      scal[0] = ex.x + v.x;
      scal[1] = ex.y + v.y;
    }
    int run = ex.x;
    for (int c = 0; c < nchunks; ++c) {
      const int64_t i = (int64_t)c * E + e;
      const int cc = chunk_cnt[i];
      chunk_cnt[i] = run;
      run += cc;
    }
  }
  if (e == 0) *acc_tokens += T;
}

// Integer stage of a small batch (T <= 1024, decode) in one block of 1024 threads, one
// token per thread: the work of the three kernels above in one launch.  One 32-bit token
// mask per (warp, expert) covers the whole batch, so the counts, the offsets and the
// order (ascending token within each expert) are the same.
constexpr int kSmallT = 1024;
__global__ void __launch_bounds__(1024) k_route_small(const int32_t* __restrict__ idx, int T, int k, int N, int E,
                                                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                      int32_t* __restrict__ mb_off, int32_t* __restrict__ scal,
                                                      int64_t* __restrict__ acc_counts,
                                                      int64_t* __restrict__ acc_tokens, int32_t* __restrict__ sp_off,
                                                      int32_t* __restrict__ perm, int32_t* __restrict__ pos) {
  extern __shared__ uint32_t smask[];  // [32][E]
  __shared__ int2 warp_tot[32];
  __shared__ int2 warp_tot2[32];
  __shared__ int32_t base[1024];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 32 * E; i += 1024) smask[i] = 0u;
  __syncthreads();
  if (tid < T)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)tid * k + j];
      if ((unsigned)e < (unsigned)E) atomicOr(&smask[warp * E + e], 1u << lane);  // an id out of range is skipped
    }
  __syncthreads();
  const int e = tid;  // thread = expert
  int total = 0;
  if (e < E) {
#pragma unroll 8
    for (int w = 0; w < 32; ++w) total += __popc(smask[w * E + e]);
    counts[e] = total;
    acc_counts[e] += total;
  }
  const int2 v = (e < N) ? make_int2(total, (total + kBM - 1) / kBM) : make_int2(0, 0);
  const int2 ex = block_exclusive_scan2(v, warp_tot);
  const int2 v2 = make_int2((v.y + 1) / 2, 0);
  const int2 ex2 = sp_off ? block_exclusive_scan2(v2, warp_tot2) : make_int2(0, 0);
  if (e < N) {
    offsets[e] = ex.x;
    mb_off[e] = ex.y;
    base[e] = ex.x;
    if (sp_off) sp_off[e] = ex2.x;
    if (e == N - 1) {
      offsets[N] = ex.x + v.x;
      mb_off[N] = ex.y + v.y;
      if (sp_off) sp_off[N] = ex2.x + v2.x;
      scal[0] = ex.x + v.x;
      scal[1] = ex.y + v.y;
    }
  }
  if (e == 0) *acc_tokens += T;
  __syncthreads();
  if (tid >= T) return;
  for (int j = 0; j < k; ++j) {
    const int64_t pair = (int64_t)tid * k + j;
    const int ej = idx[pair];
    if ((unsigned)ej < (unsigned)N) {
      int r = base[ej];
      for (int w = 0; w < warp; ++w) r += __popc(smask[w * E + ej]);
      r += __popc(smask[warp * E + ej] & ((1u << lane) - 1u));
      pos[pair] = r;
      perm[r] = (int32_t)pair;
    } else {
      pos[pair] = -1;
    }
  }
}

// Integer stage, part 3: the permuted row of every FFN pair.  Within a 256-token
// block the rank of (t, e) is the number of earlier tokens of the block that
// chose e (earlier warps' masks, then the lower lanes of its own warp's mask),
// so the order is ascending token within each expert.
__global__ void __launch_bounds__(kChunk) k_route_scatter(const int32_t* __restrict__ idx, int T, int k, int N, int E,
                                                          const int32_t* __restrict__ chunk_base,
                                                          int32_t* __restrict__ perm, int32_t* __restrict__ pos) {
  extern __shared__ uint32_t smask[];  // [8][E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 8 * E; i += kChunk) smask[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kChunk + tid;
  if (t < T)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)t * k + j];
      if ((unsigned)e < (unsigned)E) atomicOr(&smask[warp * E + e], 1u << lane);
    }
  __syncthreads();
  if (t >= T) return;
  for (int j = 0; j < k; ++j) {
    const int64_t pair = (int64_t)t * k + j;
    const int e = idx[pair];
    if ((unsigned)e < (unsigned)N) {
      int r = chunk_base[(int64_t)blockIdx.x * E + e];
      for (int w = 0; w < warp; ++w) r += __popc(smask[w * E + e]);
      r += __popc(smask[warp * E + e] & ((1u << lane) - 1u));
      pos[pair] = r;
      perm[r] = (int32_t)pair;
    } else {
      pos[pair] = -1;
    }
  }
}

// X_perm[pos[t, j]] = x[t] for every FFN slot of every token: the FFN pairs' rows in
// expert order, written from the token side.  A warp takes one (token, 2 KB column chunk)
// item at a time: it reads the chunk once, four 16-byte vectors per lane, and writes it to
// all of the token's FFN rows.  (Reading per pair instead -- X_perm[p] = x[token of p], one
// warp per row -- fetched each token's row up to k times, about twice its bytes from DRAM, and
// took 0.50 against 0.36-0.39 ms at prefill_560b.)
__global__ void __launch_bounds__(256) k_scatter_rows(const uint4* __restrict__ x, int row_vecs,
                                                      const int32_t* __restrict__ pos, int T, int k,
                                                      uint4* __restrict__ xperm) {
  const int lane = threadIdx.x & 31;
  const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
  const int nchunks = (row_vecs + 127) / 128;
  const int64_t items = (int64_t)T * nchunks;
  for (int64_t it = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
    const int t = (int)(it / nchunks);
    const int v0 = (int)(it - (int64_t)t * nchunks) * 128;
    const int my_p = lane < k ? pos[(int64_t)t * k + lane] : -1;  // slot `lane`'s FFN row (-1: zero expert)
    const uint4* src = x + (int64_t)t * row_vecs;
    uint4 a[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + 32 * u + lane;
      if (v < row_vecs) a[u] = src[v];
    }
    for (int j = 0; j < k; ++j) {
      const int p = __shfl_sync(0xffffffffu, my_p, j);
      if (p < 0) continue;
      uint4* dst = xperm + (int64_t)p * row_vecs;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + 32 * u + lane;
        if (v < row_vecs) dst[v] = a[u];
      }
    }
  }
}

// Combine / unpermute (zero experts folded in as identity terms):
//   y_t = zsum_t * x_t + sum over FFN slots j (in slot order) of g_tj * Y[pos_tj],
// fp32 accumulation, one rounding to the output type.  A gather per token, no atomics.
template <typename TIO>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void load(const __nv_bfloat16* p, float* f) {
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float* f) {
    uint4 r;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = r;
  }
};
template <>
struct Vec<float> {
  static constexpr int kN = 4;
  __device__ static void load(const float* p, float* f) {
    const float4 r = *reinterpret_cast<const float4*>(p);
    f[0] = r.x;
    f[1] = r.y;
    f[2] = r.z;
    f[3] = r.w;
  }
  __device__ static void store(float* p, const float* f) { *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]); }
};

// Large batches: one block per token, its threads striding over the row's vectors, one
// slot's load at a time (G = 1) -- many resident blocks keep the most loads in flight
// (~91% of the HBM copy rate measured on B200).  Smaller batches: one block per (token,
// 128 vectors); and when even those blocks are few (decode), G = 8 slots' loads issued
// together before their products are added, so that a thread's loads do not wait one
// after another.  The products are added in slot order either way, so the result is the
// same.  (At 2048 tokens the G = 8 form took twice the time of the one-block-per-token form,
// 118 against 56 us, hence the thresholds.)
// With offsets / mb_off (FP8 layers), Y holds expert e's pairs from padded row
// 128 mb_off[e] on, so a pair's row is pos - offsets[e] + 128 mb_off[e].
template <typename TIO, int G>
__global__ void __launch_bounds__(128) k_combine(const TIO* __restrict__ x, const TIO* __restrict__ Y,
                                                 const float* __restrict__ gate, const int32_t* __restrict__ pos, int T,
                                                 int k, int d, TIO* __restrict__ y, const int32_t* __restrict__ idx,
                                                 const int32_t* __restrict__ offsets,
                                                 const int32_t* __restrict__ mb_off) {
  constexpr int V = Vec<TIO>::kN;
  __shared__ float sg[32];
  __shared__ int32_t sp[32];
  __shared__ float szsum;
  const int nv = d / V;
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    sg[threadIdx.x] = gate[(int64_t)t * k + threadIdx.x];
    int p = pos[(int64_t)t * k + threadIdx.x];
    if (offsets && p >= 0) {
      const int e = idx[(int64_t)t * k + threadIdx.x];
      p = p - offsets[e] + 128 * mb_off[e];
    }
    sp[threadIdx.x] = p;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float z = 0.0f;
    for (int j = 0; j < k; ++j)
      if (sp[j] < 0) z = __fadd_rn(z, sg[j]);
    szsum = z;
  }
  __syncthreads();
  const float zsum = szsum;
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < nv; v += gridDim.y * blockDim.x) {
    float acc[V], a[V];
    Vec<TIO>::load(x + (int64_t)t * d + v * V, a);
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = __fmul_rn(zsum, a[i]);
    for (int j0 = 0; j0 < k; j0 += G) {
      float b[G][V];
#pragma unroll
      for (int jj = 0; jj < G; ++jj) {
        const int j = j0 + jj;
        if (j < k && sp[j] >= 0) Vec<TIO>::load(Y + (int64_t)sp[j] * d + v * V, b[jj]);
      }
#pragma unroll
      for (int jj = 0; jj < G; ++jj) {
        const int j = j0 + jj;
        if (j < k && sp[j] >= 0) {
          const float g = sg[j];
#pragma unroll
          for (int i = 0; i < V; ++i) acc[i] = __fmaf_rn(g, b[jj][i], acc[i]);
        }
      }
    }
    Vec<TIO>::store(y + (int64_t)t * d + v * V, acc);
  }
}

// Bias controller step; one block, thread = expert.  Every operation rounds
// once and none is fused, in the order of the rule in the header.
__global__ void __launch_bounds__(1024) k_update_bias(int64_t* __restrict__ counts, int64_t* __restrict__ tokens, int N,
                                                      int Z, int k, float kp, float ki, float kd, float decay,
                                                      float target, const float* __restrict__ b0,
                                                      float* __restrict__ eta, float* __restrict__ integ,
                                                      float* __restrict__ eprev, float* __restrict__ bias) {
  const int64_t tok = *tokens;
  const float eta0 = *eta;
  __syncthreads();
  if (tok <= 0) return;
  const int E = N + Z;
  const float tf = __ll2float_rn(tok);
  const float tau_f = __fdiv_rn(target, __int2float_rn(N));
  const float tau_z = Z > 0 ? __fdiv_rn(__fsub_rn(__int2float_rn(k), target), __int2float_rn(Z)) : 0.0f;
  const float et = __fmul_rn(eta0, decay);
  const float kpe = __fmul_rn(kp, et);
  const float kde = __fmul_rn(kd, et);
  for (int i = threadIdx.x; i < E; i += blockDim.x) {
    const float load = __fdiv_rn(__ll2float_rn(counts[i]), tf);
    const float tau = i < N ? tau_f : tau_z;
    const float err = __fsub_rn(tau, load);
    const float step = __fmul_rn(et, err);
    const float in = __fadd_rn(integ[i], step);
    integ[i] = in;
    const float p = __fmul_rn(kpe, err);
    const float q = __fmul_rn(ki, in);
    const float dd = __fmul_rn(kde, __fsub_rn(err, eprev[i]));
    bias[i] = __fadd_rn(__fadd_rn(__fadd_rn(p, q), dd), b0[i]);
    eprev[i] = err;
    counts[i] = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    *eta = et;
    *tokens = 0;
  }
}

// Self-test of the bounded-wait path used by every pipelined kernel: waits on an
// mbarrier that nothing arrives at, gives up after limit_ns, records site 99.
__global__ void k_selftest_wait(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, err, 99, limit_ns);
}

int grid_cap(int want, int cap) { return want < 1 ? 1 : (want < cap ? want : cap); }

// One group holding all T rows (the dense FFN through the grouped GEMM):
// row_off = {0, T}, mb_off = {0, ceil(T / 128)}, sp_off (if given) = {0, ceil(mb / 2)}.
__global__ void k_single_group(int32_t* row_off, int32_t* mb_off, int32_t* sp_off, int T) {
  if (threadIdx.x == 0) {
    const int mb = (T + kBM - 1) / kBM;
    row_off[0] = 0;
    row_off[1] = T;
    mb_off[0] = 0;
    mb_off[1] = mb;
    if (sp_off) {
      sp_off[0] = 0;
      sp_off[1] = (mb + 1) / 2;
    }
  }
}

}  // namespace

cudaError_t launch_softmax_topk(const float* logits, const float* bias, int T, int E, int k, float scale, int32_t* idx,
                                float* gate, float* scores, int sms, cudaStream_t s) {
  const int grid = grid_cap((T + 7) / 8, sms * 16);
  const int epl = (E + 31) / 32;
#define ZC_TOPK(n)                                                                                   \
  case n:                                                                                            \
    k_softmax_topk<n><<<grid, 256, 0, s>>>(logits, bias, T, E, k, scale, idx, gate, scores); \
    break;
  switch (epl) {
    ZC_TOPK(1) ZC_TOPK(2) ZC_TOPK(3) ZC_TOPK(4) ZC_TOPK(5) ZC_TOPK(6) ZC_TOPK(7) ZC_TOPK(8)
    ZC_TOPK(9) ZC_TOPK(10) ZC_TOPK(11) ZC_TOPK(12) ZC_TOPK(13) ZC_TOPK(14) ZC_TOPK(15) ZC_TOPK(16)
    ZC_TOPK(17) ZC_TOPK(18) ZC_TOPK(19) ZC_TOPK(20) ZC_TOPK(21) ZC_TOPK(22) ZC_TOPK(23) ZC_TOPK(24)
    ZC_TOPK(25) ZC_TOPK(26) ZC_TOPK(27) ZC_TOPK(28) ZC_TOPK(29) ZC_TOPK(30) ZC_TOPK(31) ZC_TOPK(32)
    default:
      return cudaErrorInvalidValue;
  }
#undef ZC_TOPK
  return cudaGetLastError();
}

cudaError_t launch_route_count(const int32_t* idx, int T, int k, int E, int32_t* chunk_cnt, cudaStream_t s) {
  const int nchunks = (T + kChunk - 1) / kChunk;
  k_route_count<<<nchunks, kChunk, 8 * E * sizeof(uint32_t), s>>>(idx, T, k, E, chunk_cnt);
  return cudaGetLastError();
}

cudaError_t launch_route_scan(int32_t* chunk_cnt, int nchunks, int T, int N, int E, int32_t* counts, int32_t* offsets,
                              int32_t* mb_off, int32_t* scal, int64_t* acc_counts, int64_t* acc_tokens, cudaStream_t s,
                              int32_t* sp_off) {
  k_route_scan<<<1, 1024, 0, s>>>(chunk_cnt, nchunks, T, N, E, counts, offsets, mb_off, scal, acc_counts, acc_tokens,
                                  sp_off);
  return cudaGetLastError();
}

int route_small_max_tokens() { return kSmallT; }

cudaError_t launch_route_small(const int32_t* idx, int T, int k, int N, int E, int32_t* counts, int32_t* offsets,
                               int32_t* mb_off, int32_t* scal, int64_t* acc_counts, int64_t* acc_tokens,
                               int32_t* sp_off, int32_t* perm, int32_t* pos, cudaStream_t s) {
  if (T < 1 || T > kSmallT || E > 1024) return cudaErrorInvalidValue;
  static SmemAttr attr{};
  const cudaError_t e = ensure_smem_attr(attr, k_route_small, 32 * 1024 * (int)sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  k_route_small<<<1, 1024, 32 * E * sizeof(uint32_t), s>>>(idx, T, k, N, E, counts, offsets, mb_off, scal, acc_counts,
                                                          acc_tokens, sp_off, perm, pos);
  return cudaGetLastError();
}

cudaError_t launch_route_scatter(const int32_t* idx, int T, int k, int N, int E, const int32_t* chunk_base,
                                 int32_t* perm, int32_t* pos, cudaStream_t s) {
  const int nchunks = (T + kChunk - 1) / kChunk;
  k_route_scatter<<<nchunks, kChunk, 8 * E * sizeof(uint32_t), s>>>(idx, T, k, N, E, chunk_base, perm, pos);
  return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const void* x, int row_bytes, const int32_t* pos, int T, int k, void* xperm, int sms,
                                cudaStream_t s) {
  const int64_t items = (int64_t)T * ((row_bytes / 16 + 127) / 128);  // one warp per (token, 2 KB chunk)
  int64_t blocks = (items + 7) / 8;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  if (blocks < 1) blocks = 1;
  k_scatter_rows<<<(int)blocks, 256, 0, s>>>(static_cast<const uint4*>(x), row_bytes / 16, pos, T, k,
                                             static_cast<uint4*>(xperm));
  return cudaGetLastError();
}

cudaError_t launch_combine(int bf16, const void* x, const void* Y, const int32_t* idx, const float* gate,
                           const int32_t* pos, int T, int k, int N, int d, void* y, int sms, cudaStream_t s,
                           const int32_t* offsets, const int32_t* mb_off) {
  (void)N;
  const int nv = d / (bf16 ? 8 : 4);
  const int split = (nv + 127) / 128;
  const bool wide = T < sms * 8;                                 // < 8 token blocks per SM: split the rows
  const bool small = wide && (int64_t)T * split <= (int64_t)sms * 8;  // still < 8 blocks per SM: G = 8
  const dim3 grid((unsigned)T, wide ? (unsigned)split : 1u);
  if (bf16) {
    auto x_ = static_cast<const __nv_bfloat16*>(x);
    auto Y_ = static_cast<const __nv_bfloat16*>(Y);
    auto y_ = static_cast<__nv_bfloat16*>(y);
    if (small) k_combine<__nv_bfloat16, 8><<<grid, 128, 0, s>>>(x_, Y_, gate, pos, T, k, d, y_, idx, offsets, mb_off);
    else k_combine<__nv_bfloat16, 1><<<grid, 128, 0, s>>>(x_, Y_, gate, pos, T, k, d, y_, idx, offsets, mb_off);
  } else {
    auto x_ = static_cast<const float*>(x);
    auto Y_ = static_cast<const float*>(Y);
    auto y_ = static_cast<float*>(y);
    if (small) k_combine<float, 8><<<grid, 128, 0, s>>>(x_, Y_, gate, pos, T, k, d, y_, idx, offsets, mb_off);
    else k_combine<float, 1><<<grid, 128, 0, s>>>(x_, Y_, gate, pos, T, k, d, y_, idx, offsets, mb_off);
  }
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(int* err, uint64_t limit_ns, cudaStream_t s) {
  k_selftest_wait<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd(const float* logits, int T, int E, int k, float scale, const int32_t* idx,
                              const float* dg, __nv_bfloat16* dl, int ld, int sms, cudaStream_t s) {
  const int warps = T;
  int blocks = (warps + 7) / 8;
  if (blocks > sms * 16) blocks = sms * 16;
  if (blocks < 1) blocks = 1;
  // ld >= E, rounded up to 64; each lane covers experts lane, lane + 32, ... < 32 * EPL
  if (ld <= 128) k_router_bwd<4><<<blocks, 256, 0, s>>>(logits, T, E, k, scale, idx, dg, dl, ld);
  else if (ld <= 256) k_router_bwd<8><<<blocks, 256, 0, s>>>(logits, T, E, k, scale, idx, dg, dl, ld);
  else if (ld <= 512) k_router_bwd<16><<<blocks, 256, 0, s>>>(logits, T, E, k, scale, idx, dg, dl, ld);
  else if (ld <= 1024) k_router_bwd<32><<<blocks, 256, 0, s>>>(logits, T, E, k, scale, idx, dg, dl, ld);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_single_group(int32_t* row_off, int32_t* mb_off, int T, cudaStream_t s, int32_t* sp_off) {
  k_single_group<<<1, 32, 0, s>>>(row_off, mb_off, sp_off, T);
  return cudaGetLastError();
}

cudaError_t launch_update_bias(int64_t* counts, int64_t* tokens, int N, int Z, int k, float kp, float ki, float kd,
                               float decay, float target, const float* b0, float* eta, float* integ, float* eprev,
                               float* bias, cudaStream_t s) {
  k_update_bias<<<1, 1024, 0, s>>>(counts, tokens, N, Z, k, kp, ki, kd, decay, target, b0, eta, integ, eprev, bias);
  return cudaGetLastError();
}

}  // namespace zc
