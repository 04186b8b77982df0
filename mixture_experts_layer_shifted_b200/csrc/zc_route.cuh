// Routing of one token by one warp: softmax over the router logits, top-k on the
// bias-shifted scores, the gates.  Run by the routing kernel (k_softmax_topk); it is kept in
// a header of its own so that any kernel that routes (a router GEMM epilogue was one such
// variant, measured slower) follows the same rule.
//
// Sources (page title, section):
//  - LongCat-Flash technical summary (zhangjingwei.cn), 二 架構, part 1
//    "零計算專家": an expert-specific bias shifts the routing scores.
//  - LongCat-Flash tech-report thread (web3.cnouyi.fund): the bias selects only
//    (DeepSeek-V3-like auxiliary-loss-free balancing).
//  - LongCat-Flash-Lite N-gram article (onthewifi.com), part 02: the router is a
//    fused softmax + top-k + scaling step.
//
// Every floating-point operation that can change an integer decision (softmax,
// biased score, comparison) is written with an explicit rounding intrinsic so
// that the compiler cannot contract or reorder it; the rule it follows is:
//   m = max_e l_e (over the logits that are numbers);  u_e = zexp(l_e - m);
//   per lane p (e = p, p+32, ...): partial sums in ascending e; then a
//   butterfly over lane distance 16, 8, 4, 2, 1: partial += partner;
//   s_e = u_e / sum;  v_e = s_e + b_e;  top-k on v, ties to the lower id,
//   a NaN v ranking as -inf;  gate = scale * s.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace zc {

// exp for x <= 0 (the softmax only needs that range; larger x is still handled
// up to overflow).  Cody-Waite reduction: n = rint(x * fl32(1/ln2)),
// r = (x - n*C1) - n*C2 with C1 = ln2 truncated to 16 significant bits (n*C1 is
// exact for |n| < 256) and C2 = fl32(ln2 - C1); degree-7 Taylor polynomial of
// e^r with coefficients fl32(1/i!) in Horner form with fused multiply-adds;
// scaled by 2^n built in the exponent field; results under 2^-125 flush to 0.
__device__ __forceinline__ float zexp(float x) {
  if (!(x > -88.0f)) return 0.0f;
  const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));
  if (n < -125.0f) return 0.0f;
  if (n > 127.0f) return __int_as_float(0x7f800000);
  float r = __fmaf_rn(-n, 0x1.62e4p-1f, x);
  r = __fmaf_rn(-n, 0x1.7f7d1cp-20f, r);
  float p = 0x1.a01a02p-13f;
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);
  p = __fmaf_rn(p, r, 0x1.111112p-7f);
  p = __fmaf_rn(p, r, 0x1.555556p-5f);
  p = __fmaf_rn(p, r, 0x1.555556p-3f);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const float scale = __int_as_float(((int)n + 127) << 23);
  return __fmul_rn(p, scale);
}

// Selection key of a biased score: a NaN ranks as -inf (below every number), so a
// row whose scores are not all numbers still selects k distinct valid experts
// (the lowest untaken ids among the NaN ones) instead of an id out of range.
__device__ __forceinline__ float rank_key(float v) { return v == v ? v : -__int_as_float(0x7f800000); }

// Selection key of a biased score: unsigned, ordered like the scores (a NaN ranks
// as -inf, -0 as +0); 0 lies below every score's key and marks an expert already
// taken (or a padding slot past E).
__device__ __forceinline__ uint32_t sel_key(float v) {
  uint32_t b = __float_as_uint(rank_key(v));
  if (b == 0x80000000u) b = 0u;  // -0 compares equal to +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// (a, ea) ranks before (b, eb): the larger key, or the lower id on equal keys.
__device__ __forceinline__ bool ranks_before(uint32_t a, uint32_t ea, uint32_t b, uint32_t eb) {
  return a > b || (a == b && ea < eb);
}

// One token, one warp (all 32 lanes call it).  EPL = experts held per lane (E <= 32 EPL);
// lane p holds experts p, p + 32, ...  lt: the token's E logits; writes idx_row[0..k),
// gate_row[0..k) and, if scores_row is not null, its E scores.  slots: this warp's 96 words
// of shared memory.  Selection, exact, in two steps:
//  1. threshold: the k-th largest of the 32 lane maxima (ties counted), tau.  At least
//     k lanes hold a key >= tau, so every one of the k picks has a key >= tau;
//  2. the candidates (key >= tau) are compacted into one slot per lane -- each lane writes
//     its own at the prefix of the lanes' counts -- and sorted by (key descending, id
//     ascending) with a 32-lane bitonic network; lanes 0..k-1 then hold the picks in slot
//     order (the sort makes the order of the slots before it irrelevant).
// When more than 32 candidates reach tau (ties at the threshold, e.g. a row of NaN
// scores), the picks are taken one by one instead: a warp max of the lanes' best
// untaken keys, then a warp min of the ids holding it, the winning lane rescanning.
template <int EPL>
__device__ __forceinline__ void route_token(const float* __restrict__ lt, const float* __restrict__ bias, int E, int k,
                                            float scale, int32_t* __restrict__ idx_row, float* __restrict__ gate_row,
                                            float* __restrict__ scores_row, int lane, uint32_t* __restrict__ slots) {
  float u[EPL];
  float m = -__int_as_float(0x7f800000);
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    u[i] = e < E ? __ldcg(lt + e) : -__int_as_float(0x7f800000);  // through L2: other SMs wrote them
    m = fmaxf(m, u[i]);
  }
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, w));
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    u[i] = e < E ? zexp(__fsub_rn(u[i], m)) : 0.0f;
    if (e < E) acc = __fadd_rn(acc, u[i]);
  }
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, w));
  uint32_t key[EPL];
  uint32_t lmax = 0;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    u[i] = __fdiv_rn(u[i], acc);  // u now holds the score s
    key[i] = e < E ? sel_key(__fadd_rn(u[i], __ldg(bias + e))) : 0u;
    if (e < E && scores_row) scores_row[e] = u[i];
    lmax = max(lmax, key[i]);
  }
  // 1. tau = the k-th largest lane maximum
  uint32_t tau = 0, act = lmax;
  int need = k;
  for (int r = 0; r < k && need > 0; ++r) {
    const uint32_t g = __reduce_max_sync(0xffffffffu, act);
    need -= __popc(__ballot_sync(0xffffffffu, act == g));
    if (act == g) act = 0u;
    tau = g;
  }
  // 2. compaction of the candidates: lane c receives the c-th one (key, id, score)
  int mine = 0;
#pragma unroll
  for (int i = 0; i < EPL; ++i) mine += key[i] >= tau ? 1 : 0;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int count = __shfl_sync(0xffffffffu, incl, 31);
  uint32_t ck = 0u, ce = 0xffffffffu;
  float cs = 0.0f;
  if (count <= 32) {
    int at = incl - mine;  // this lane's first slot
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      if (key[i] >= tau) {
        slots[at] = key[i];
        slots[32 + at] = (uint32_t)(lane + 32 * i);
        slots[64 + at] = __float_as_uint(u[i]);
        ++at;
      }
    }
    __syncwarp();
    if (lane < count) {
      ck = slots[lane];
      ce = slots[32 + lane];
      cs = __uint_as_float(slots[64 + lane]);
    }
    __syncwarp();  // every lane has read its slot before the warp's next token writes them
  }
  int my_idx = 0;
  float my_gate = 0.0f;
  if (count <= 32) {
    // bitonic sort of the 32 slots, best first (empty slots: key 0, id ~0, last)
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const uint32_t ok = __shfl_xor_sync(0xffffffffu, ck, stride);
        const uint32_t oe = __shfl_xor_sync(0xffffffffu, ce, stride);
        const float os = __shfl_xor_sync(0xffffffffu, cs, stride);
        const bool lower = (lane & stride) == 0;
        const bool best_first = (lane & size) == 0;  // this block is sorted best first
        const bool other_before = ranks_before(ok, oe, ck, ce);
        // the lower lane of a best-first block keeps the better of the two
        if (other_before == (lower == best_first)) {
          ck = ok;
          ce = oe;
          cs = os;
        }
      }
    }
    my_idx = (int)ce;
    my_gate = __fmul_rn(scale, cs);
  } else {
    uint32_t bk = 0;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      if (key[i] > bk) {
        bk = key[i];
        bi = i;
      }
    }
    for (int j = 0; j < k; ++j) {
      const uint32_t gk = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t ge = __reduce_min_sync(0xffffffffu, bk == gk ? (uint32_t)(lane + 32 * bi) : 0xffffffffu);
      const int wl = (int)(ge & 31u);
      float ws = 0.0f;
      if (lane == wl) {
        bk = 0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          if (i == bi) {
            ws = u[i];
            key[i] = 0u;
          }
        }
        bi = 0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          if (key[i] > bk) {
            bk = key[i];
            bi = i;
          }
        }
      }
      ws = __shfl_sync(0xffffffffu, ws, wl);
      if (lane == j) {
        my_idx = (int)ge;
        my_gate = __fmul_rn(scale, ws);
      }
    }
  }
  if (lane < k) {
    idx_row[lane] = my_idx;
    gate_row[lane] = my_gate;
  }
}

}  // namespace zc
