/*
 * Oracle for the zero-computation-expert MoE layer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  It shares no code, header or
 * constant table with the CUDA library; the two are written separately from the
 * same definitions.
 *
 * Plain, slow, obviously correct C.  Floating point is fp64 unless a function
 * says it replicates the fp32 routing rule.  Built with -O2 -ffp-contract=off
 * (no fused multiply-add except where fma() is written out) and no fast-math.
 *
 * Sources (page title, section):
 *  - LongCat-Flash technical summary (zhangjingwei.cn), section 二 架構, part 1
 *    "零計算專家": Z zero-computation experts that only return their input; an
 *    expert-specific bias, driven by a PID controller, shifts the routing scores
 *    to keep the FFN/zero selection ratio near a target; corpus-level balance.
 *  - same page, 模型配置: 512 FFN experts + 256 zero experts, 12 activated per
 *    token, hidden 6144, expert intermediate 2048.
 *  - LongCat-Flash tech-report thread (web3.cnouyi.fund): the bias works like
 *    DeepSeek-V3's auxiliary-loss-free balancing (bias in selection only) with a
 *    decay schedule on its update.
 *  - LongCat-Flash-Lite N-gram article (onthewifi.com), part 02: the router is a
 *    fused "softmax + top-k + scaling" step.
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes): softmax over all N+Z experts; top-k on score+bias, ties to the
 * lower expert index, slots ordered by biased score then index; gate = scale *
 * unbiased score, no renormalisation; zero expert output = its input; FFN expert
 * = SwiGLU, W_d (silu(W_g x) * (W_u x)), no biases; FFN experts are ids 0..N-1,
 * zero experts N..N+Z-1; positional PID on the per-expert load error.
 *
 * Parity status of each function is stated beside it; pins live in tests/.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ZO_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------- */
/* Input element access: dtype 0 = float32, 1 = bf16 bit patterns (uint16).   */
/* bf16 -> float is exact (the 16 bits become the high half of the float).   */
/* ------------------------------------------------------------------------- */
static double elem(const void *p, int dtype, int64_t i) {
  if (dtype == 1) {
    uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
  }
  return (double)((const float *)p)[i];
}

/* ------------------------------------------------------------------------- */
/* Step 1: router logits  l[t,e] = sum_c x[t,c] W_r[e,c] + o[e]   (fp64)      */
/* Page: onthewifi.com part 02 (router logits feed softmax+top-k);            */
/* zhangjingwei.cn 二.1 (routing scores).  Pinned: tests/test_oracle_pins.py  */
/* ------------------------------------------------------------------------- */
ZO_EXPORT void zo_router_logits(const void *x, int x_dtype, const void *wr, int w_dtype,
                                const float *offset, int64_t T, int d, int E, double *logits) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += elem(x, x_dtype, t * d + c) * elem(wr, w_dtype, (int64_t)e * d + c);
      if (offset) acc += (double)offset[e];
      logits[t * E + e] = acc;
    }
  }
}

/* Step 2: s = softmax(l) over all E experts, fp64.  The shift m is the largest
 * logit that is a number (a NaN logit never compares greater). */
ZO_EXPORT void zo_softmax_f64(const double *l, int64_t T, int E, double *s) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const double *lt = l + t * E;
    double m = -INFINITY;
    for (int e = 0; e < E; ++e)
      if (lt[e] > m) m = lt[e];
    double sum = 0.0;
    for (int e = 0; e < E; ++e) sum += exp(lt[e] - m);
    for (int e = 0; e < E; ++e) s[t * E + e] = exp(lt[e] - m) / sum;
  }
}

/* Selection key: a biased score that is not a number ranks as -inf, below
 * every number, so k distinct valid experts are always chosen. */
static double key64(double v) { return v != v ? -INFINITY : v; }
static float key32(float v) { return v != v ? -INFINITY : v; }

/* Steps 3-5 (fp64): v = s + b; S = the k largest v, ties to the lower index,
 * slot order v descending then index ascending; gate = scale * s (bias never in
 * the gate, no renormalisation).  margin[t] = v_(k) - v_(k+1) (+inf if k == E),
 * used to exclude near-ties from index comparison.
 * Page: web3.cnouyi.fund (DSv3-like bias in selection); zhangjingwei.cn 二.1. */
ZO_EXPORT void zo_topk_f64(const double *s, const double *bias, int64_t T, int E, int k, double scale,
                           int32_t *idx, double *gate, double *margin) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const double *st = s + t * E;
    unsigned char *taken = (unsigned char *)calloc((size_t)E, 1);
    double last = 0.0;
    for (int j = 0; j < k; ++j) {
      int best = -1;
      double bv = 0.0;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        double v = key64(st[e] + (bias ? bias[e] : 0.0));
        if (best < 0 || v > bv) { best = e; bv = v; } /* strict '>' keeps the lower index on ties */
      }
      taken[best] = 1;
      idx[t * k + j] = best;
      gate[t * k + j] = scale * st[best];
      last = bv;
    }
    if (margin) {
      double next = -INFINITY;
      int found = 0;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        double v = key64(st[e] + (bias ? bias[e] : 0.0));
        if (!found || v > next) { next = v; found = 1; }
      }
      margin[t] = found ? last - next : INFINITY;
    }
    free(taken);
  }
}

/* ------------------------------------------------------------------------- */
/* fp32 routing replica.                                                     */
/*                                                                           */
/* Integer results (indices, counts, permutation) are decided by fp32        */
/* comparisons, so this replica takes the same decisions in the same         */
/* precision as the device kernel, from the same written rule:               */
/*   m = max_e l_e over the logits that are numbers (-inf if none);          */
/*   u_e = zexp(l_e - m)                                                     */
/*   sum: 32 partials, partial[p] = sum over e = p, p+32, ... (ascending);   */
/*        then for w = 16,8,4,2,1: partial[p] = partial[p] + partial[p^w]    */
/*   s_e = u_e / partial[0];  v_e = s_e + b_e;  top-k as in zo_topk_f64      */
/*   (a NaN v ranks as -inf);                                                */
/*   gate = scale * s.   Every operation rounds once to fp32.                */
/* zexp: Cody-Waite reduction with ln2 split into C1 (ln2 truncated to 16    */
/* significant bits, so n*C1 is exact for |n| < 256) and C2 = fl32(ln2-C1),  */
/* n = rint(x * fl32(1/ln2)); degree-7 Taylor polynomial (coefficients       */
/* fl32(1/i!)) in Horner form with explicit fma; scaled by 2^n through the   */
/* exponent bits; results below 2^-125 flush to zero.  Pinned against libm   */
/* exp to <= 2 ulp in tests.                                                 */
/* ------------------------------------------------------------------------- */
ZO_EXPORT float zo_zexp(float x) {
  const float L2E = 0x1.715476p+0f;
  const float C1 = 0x1.62e4p-1f;
  const float C2 = 0x1.7f7d1cp-20f;
  if (!(x > -88.0f)) return 0.0f;
  float n = rintf(x * L2E);
  if (n < -125.0f) return 0.0f;
  if (n > 127.0f) return INFINITY;
  float r = fmaf(-n, C1, x);
  r = fmaf(-n, C2, r);
  float p = 0x1.a01a02p-13f;    /* 1/7! */
  p = fmaf(p, r, 0x1.6c16c2p-10f); /* 1/6! */
  p = fmaf(p, r, 0x1.111112p-7f);  /* 1/5! */
  p = fmaf(p, r, 0x1.555556p-5f);  /* 1/4! */
  p = fmaf(p, r, 0x1.555556p-3f);  /* 1/3! */
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  int ni = (int)n;
  uint32_t bits = (uint32_t)(ni + 127) << 23;
  float scale;
  memcpy(&scale, &bits, 4);
  return p * scale;
}

ZO_EXPORT void zo_route_replica_f32(const float *logits, const float *bias, int64_t T, int E, int k,
                                    float scale, float *scores, int32_t *idx, float *gate) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const float *lt = logits + t * E;
    float *u = (float *)malloc(sizeof(float) * (size_t)E);
    unsigned char *taken = (unsigned char *)calloc((size_t)E, 1);
    float m = -INFINITY;
    for (int e = 0; e < E; ++e)
      if (lt[e] > m) m = lt[e];
    for (int e = 0; e < E; ++e) u[e] = zo_zexp(lt[e] - m);
    float part[32];
    for (int p = 0; p < 32; ++p) {
      float acc = 0.0f;
      for (int e = p; e < E; e += 32) acc = acc + u[e];
      part[p] = acc;
    }
    for (int w = 16; w >= 1; w >>= 1) {
      float nxt[32];
      for (int p = 0; p < 32; ++p) nxt[p] = part[p] + part[p ^ w];
      memcpy(part, nxt, sizeof(part));
    }
    const float sum = part[0];
    for (int e = 0; e < E; ++e) u[e] = u[e] / sum; /* u now holds s */
    if (scores)
      for (int e = 0; e < E; ++e) scores[t * E + e] = u[e];
    for (int j = 0; j < k; ++j) {
      int best = -1;
      float bv = 0.0f;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        float v = key32(u[e] + (bias ? bias[e] : 0.0f));
        if (best < 0 || v > bv) { best = e; bv = v; }
      }
      taken[best] = 1;
      idx[t * k + j] = best;
      gate[t * k + j] = scale * u[best];
    }
    free(taken);
    free(u);
  }
}

/* ------------------------------------------------------------------------- */
/* Integer stage (exact).  counts[e] over all E experts; offsets = exclusive */
/* scan over FFN experts 0..N-1 (offsets[N] = P, the FFN pairs); perm lists  */
/* the FFN pairs ordered by (expert asc, token asc), each entry t*k + j;     */
/* pos[t*k+j] = its place in perm, or -1 for a zero-expert slot.             */
/* Zero experts are routed to no expert computation at all (they cost        */
/* nothing, zhangjingwei.cn 二.1), so only FFN pairs enter the permutation.  */
/* ------------------------------------------------------------------------- */
ZO_EXPORT int64_t zo_integer_stage(const int32_t *idx, int64_t T, int k, int N, int E, int32_t *counts,
                                   int32_t *offsets, int32_t *perm, int32_t *pos) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t i = 0; i < T * k; ++i) counts[idx[i]]++;
  offsets[0] = 0;
  for (int e = 0; e < N; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t *fill = (int32_t *)calloc((size_t)N, sizeof(int32_t));
  for (int64_t t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      int e = idx[t * k + j];
      if (e < N) {
        int32_t p = offsets[e] + fill[e]++;
        perm[p] = (int32_t)(t * k + j);
        pos[t * k + j] = p;
      } else {
        pos[t * k + j] = -1;
      }
    }
  }
  free(fill);
  return offsets[N];
}

/* ------------------------------------------------------------------------- */
/* FFN expert (SwiGLU), fp64:  F(x) = W_d (silu(W_g x) * (W_u x)),           */
/* silu(z) = z / (1 + exp(-z)).  W_g, W_u are [inter, d]; W_d is [d, inter]. */
/* out[r, :] = F(xs[r, :]) for n rows.                                        */
/* ------------------------------------------------------------------------- */
ZO_EXPORT void zo_ffn_f64(const void *xs, int x_dtype, int64_t n, const void *wg, const void *wu,
                          const void *wd, int w_dtype, int d, int inter, double *out) {
  double *h = (double *)malloc(sizeof(double) * (size_t)inter);
  for (int64_t r = 0; r < n; ++r) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < inter; ++i) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < d; ++c) {
        const double xv = elem(xs, x_dtype, r * d + c);
        g += elem(wg, w_dtype, (int64_t)i * d + c) * xv;
        u += elem(wu, w_dtype, (int64_t)i * d + c) * xv;
      }
      h[i] = g / (1.0 + exp(-g)) * u;
    }
#pragma omp parallel for schedule(static)
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int i = 0; i < inter; ++i) acc += elem(wd, w_dtype, (int64_t)c * inter + i) * h[i];
      out[r * d + c] = acc;
    }
  }
  free(h);
}

/* ------------------------------------------------------------------------- */
/* Whole layer output for tokens with all weights in memory (small configs): */
/* y_t = sum_{j: e_j < N} g_j F_{e_j}(x_t) + (sum_{j: e_j >= N} g_j) x_t.     */
/* Zero experts return x unchanged (zhangjingwei.cn 二.1).                    */
/* wg/wu: [N, inter, d], wd: [N, d, inter].                                  */
/* ------------------------------------------------------------------------- */
ZO_EXPORT void zo_layer_f64(const void *x, int x_dtype, int64_t T, const int32_t *idx, const double *gate,
                            int k, int N, const void *wg, const void *wu, const void *wd, int w_dtype, int d,
                            int inter, double *y) {
  const int64_t wsz = (int64_t)inter * d;
  const size_t esz = (w_dtype == 1) ? 2 : 4;
  const size_t xsz = (x_dtype == 1) ? 2 : 4;
  for (int64_t t = 0; t < T; ++t) {
    double *yt = y + t * d;
    for (int c = 0; c < d; ++c) yt[c] = 0.0;
    double zsum = 0.0;
    double *f = (double *)malloc(sizeof(double) * (size_t)d);
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      const double g = gate[t * k + j];
      if (e >= N) {
        zsum += g;
        continue;
      }
      zo_ffn_f64((const char *)x + (size_t)(t * d) * xsz, x_dtype, 1, (const char *)wg + (size_t)(e * wsz) * esz,
                 (const char *)wu + (size_t)(e * wsz) * esz, (const char *)wd + (size_t)(e * wsz) * esz, w_dtype,
                 d, inter, f);
      for (int c = 0; c < d; ++c) yt[c] += g * f[c];
    }
    for (int c = 0; c < d; ++c) yt[c] += zsum * elem(x, x_dtype, t * d + c);
    free(f);
  }
}

/* ------------------------------------------------------------------------- */
/* Bias controller (fp32, every operation rounded once, no fma).             */
/* zhangjingwei.cn 二.1: a PID controller sets expert-specific bias terms so  */
/* the FFN/zero selection ratio stays near its target; corpus-level balance; */
/* web3.cnouyi.fund: a decay schedule on the bias update.  Reading:          */
/*   load  l_i = fl32(c_i) / fl32(T_acc)                                     */
/*   target tau_i = K/N (FFN) or (k-K)/Z (zero), K = target FFN picks/token   */
/*   error e_i = tau_i - l_i;  eta <- eta*decay                               */
/*   I_i <- I_i + eta*e_i                                                     */
/*   b_i <- ((kp*eta*e_i + ki*I_i) + kd*eta*(e_i - eprev_i)) + b0_i           */
/*   eprev_i <- e_i;  counts and T_acc reset to zero.                         */
/* state: eta[1], integ[E], eprev[E]; b0 = initial bias.  No-op if T_acc==0.  */
/* Convergence rate: parity unpinned (the pages give no gains).              */
/* ------------------------------------------------------------------------- */
ZO_EXPORT void zo_update_bias(int64_t *counts, int64_t *tokens, int N, int Z, int k, float kp, float ki, float kd,
                              float decay, float target_ffn, const float *b0, float *eta, float *integ,
                              float *eprev, float *bias) {
  const int E = N + Z;
  if (*tokens <= 0) return;
  const float tf = (float)*tokens;
  const float tau_f = target_ffn / (float)N;
  const float tau_z = Z > 0 ? ((float)k - target_ffn) / (float)Z : 0.0f;
  const float et = *eta * decay;
  *eta = et;
  const float kpe = kp * et;
  const float kde = kd * et;
  for (int i = 0; i < E; ++i) {
    const float load = (float)counts[i] / tf;
    const float tau = i < N ? tau_f : tau_z;
    const float err = tau - load;
    const float step = et * err;
    integ[i] = integ[i] + step;
    const float p = kpe * err;
    const float q = ki * integ[i];
    const float dd = kde * (err - eprev[i]);
    const float s1 = p + q;
    const float s2 = s1 + dd;
    bias[i] = s2 + b0[i];
    eprev[i] = err;
    counts[i] = 0;
  }
  *tokens = 0;
}

/* ------------------------------------------------------------------------- */
/* Block-scaled FP8 experts.                                                  */
/* LongCat-Flash technical summary (zhangjingwei.cn), 六 推理與部署, 定制內核    */
/* "量化": the same fine-grained block quantization as DeepSeek-V3, one scale   */
/* per [1,128] block of activations and per [128,128] block of weights.      */
/* Readings (the pages fix neither the code nor the scale format):            */
/*  - codes are FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa      */
/*    bits; no infinities; S.1111.111 is NaN; largest finite 448), rounded to  */
/*    nearest with ties to even, saturating at 448;                            */
/*  - a block's scale is a power of two stored as E8M0 (value 2^(c-127)): the  */
/*    smallest 2^E with amax <= 448 * 2^E (code clamped to [0, 254]); an all-  */
/*    zero block takes 2^0;  q = E4M3(v / 2^E), v ~ q * 2^E.                    */
/* Parity: pinned against torch's float8_e4m3fn conversion, boundary values   */
/* and closed forms in tests/test_oracle_pins.py.                             */
/* ------------------------------------------------------------------------- */

ZO_EXPORT double zo_e4m3_decode(uint8_t c) {
  const int s = c >> 7, E = (c >> 3) & 15, M = c & 7;
  if (E == 15 && M == 7) return NAN;
  const double v = (E == 0) ? ldexp((double)M, -9) : ldexp(8.0 + M, E - 10);
  return s ? -v : v;
}

ZO_EXPORT uint8_t zo_e4m3_encode(float v) {
  if (isnan(v)) return 0x7F;
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const double a = fabs((double)v);
  if (a >= 448.0) return sign | 0x7E;
  /* spacing of representable magnitudes around a: 2^-9 below the smallest
     normal 2^-6, else 2^(k-3) for a in [2^k, 2^(k+1)) */
  double q;
  if (a < ldexp(1.0, -6)) {
    q = ldexp(1.0, -9);
  } else {
    int e;
    frexp(a, &e); /* a in [2^(e-1), 2^e) */
    q = ldexp(1.0, e - 1 - 3);
  }
  const double n = a / q; /* exact: q is a power of two */
  double r = floor(n);
  const double frac = n - r;
  if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) == 1.0)) r += 1.0;
  const double val = r * q; /* <= 448 because a < 448 */
  if (val == 0.0) return sign;
  if (val < ldexp(1.0, -6)) return sign | (uint8_t)(val / ldexp(1.0, -9)); /* subnormal, M = 1..7 */
  int ee;
  const double m = frexp(val, &ee); /* val = m * 2^ee, m in [0.5, 1) */
  const int E = ee - 1 + 7;
  const int M = (int)((2.0 * m - 1.0) * 8.0);
  return sign | (uint8_t)(E << 3) | (uint8_t)M;
}

ZO_EXPORT uint8_t zo_e8m0_scale(float amax) {
  if (!(amax > 0.0f)) return 127;
  int e;
  frexp((double)amax, &e); /* amax in [2^k, 2^(k+1)), k = e - 1 */
  const int k = e - 1;
  const int E = ((double)amax <= 1.75 * ldexp(1.0, k)) ? k - 8 : k - 7; /* 448 = 1.75 * 2^8 */
  int code = E + 127;
  if (code < 0) code = 0;
  if (code > 254) code = 254;
  return (uint8_t)code;
}

/* src [rows, cols] (dtype 0 fp32, 1 bf16 bits), cols a multiple of 128;
   block_rows 1 ([1,128] blocks) or 128 ([128,128] blocks; a last partial row
   block is allowed).  codes [rows, cols]; scales [ceil(rows/block_rows), cols/128]. */
ZO_EXPORT void zo_quantize_blocks(const void *src, int dtype, int64_t rows, int64_t cols, int block_rows,
                                  uint8_t *codes, uint8_t *scales) {
  const int64_t nrb = (rows + block_rows - 1) / block_rows, ncb = cols / 128;
#pragma omp parallel for schedule(dynamic, 1) if (rows * cols > (1 << 20))
  for (int64_t rb = 0; rb < nrb; ++rb) {
    const int64_t r0 = rb * block_rows, r1 = (r0 + block_rows < rows) ? r0 + block_rows : rows;
    for (int64_t cb = 0; cb < ncb; ++cb) {
      double amax = 0.0;
      for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = cb * 128; c < cb * 128 + 128; ++c) {
          const double a = fabs(elem(src, dtype, r * cols + c));
          if (a > amax) amax = a;
        }
      const uint8_t sc = zo_e8m0_scale((float)amax); /* exact: amax is a source value */
      scales[rb * ncb + cb] = sc;
      const double inv = ldexp(1.0, 127 - (int)sc);
      for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = cb * 128; c < cb * 128 + 128; ++c)
          codes[r * cols + c] = zo_e4m3_encode((float)(elem(src, dtype, r * cols + c) * inv));
    }
  }
}

/* FFN expert on block-scaled FP8 operands, fp64 arithmetic on the dequantized
   values.  Each row of xs (dtype as zo_ffn_f64) is quantized per [1,128] here;
   the weights come as codes with [128,128] scales: wg, wu [inter, d] with
   scales [inter/128, d/128]; wd [d, inter] with scales [d/128, inter/128].
   h = silu(g) * u is rounded to fp32 and quantized per [1,128] before the down
   projection (reading: the kernel quantizes H from its fp32 values, so the
   quantization decision is taken in that precision).  out [n, d] fp64. */
ZO_EXPORT void zo_ffn_fp8_f64(const void *xs, int x_dtype, int64_t n, const uint8_t *wg, const uint8_t *sg,
                              const uint8_t *wu, const uint8_t *su, const uint8_t *wd, const uint8_t *sd, int d,
                              int inter, double *out) {
  const size_t xsz = (x_dtype == 1) ? 2 : 4;
  uint8_t *xq = (uint8_t *)malloc((size_t)d), *xs_sc = (uint8_t *)malloc((size_t)d / 128);
  uint8_t *hq = (uint8_t *)malloc((size_t)inter), *hs_sc = (uint8_t *)malloc((size_t)inter / 128);
  double *xv = (double *)malloc(sizeof(double) * (size_t)d);
  double *hv = (double *)malloc(sizeof(double) * (size_t)inter);
  float *h32 = (float *)malloc(sizeof(float) * (size_t)inter);
  const int dkb = d / 128, ikb = inter / 128;
  double tab[256]; /* code -> value; a scale 2^s multiplies exactly */
  for (int c = 0; c < 256; ++c) tab[c] = zo_e4m3_decode((uint8_t)c);
  for (int64_t r = 0; r < n; ++r) {
    zo_quantize_blocks((const char *)xs + (size_t)(r * d) * xsz, x_dtype, 1, d, 1, xq, xs_sc);
    for (int c = 0; c < d; ++c) xv[c] = ldexp(zo_e4m3_decode(xq[c]), (int)xs_sc[c / 128] - 127);
#pragma omp parallel for schedule(static)
    for (int i = 0; i < inter; ++i) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < d; ++c) {
        const double sgv = ldexp(1.0, (int)sg[(i / 128) * dkb + c / 128] - 127);
        const double suv = ldexp(1.0, (int)su[(i / 128) * dkb + c / 128] - 127);
        g += (tab[wg[(int64_t)i * d + c]] * sgv) * xv[c];
        u += (tab[wu[(int64_t)i * d + c]] * suv) * xv[c];
      }
      h32[i] = (float)(g / (1.0 + exp(-g)) * u);
    }
    zo_quantize_blocks(h32, 0, 1, inter, 1, hq, hs_sc);
    for (int i = 0; i < inter; ++i) hv[i] = ldexp(zo_e4m3_decode(hq[i]), (int)hs_sc[i / 128] - 127);
#pragma omp parallel for schedule(static)
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int i = 0; i < inter; ++i)
        acc += (tab[wd[(int64_t)c * inter + i]] * ldexp(1.0, (int)sd[(c / 128) * ikb + i / 128] - 127)) * hv[i];
      out[r * d + c] = acc;
    }
  }
  free(xq);
  free(xs_sc);
  free(hq);
  free(hs_sc);
  free(xv);
  free(hv);
  free(h32);
}

/* ------------------------------------------------------------------------- */
/* W4A4 experts.  A LongCat-Flash news page (gate.com post) says the model    */
/* serves with W4A4: expert weights and activations quantized to 4 bits.      */
/* The format is not given; reading: MXFP4 (OCP microscaling) -- E2M1 codes    */
/* (1 sign, 2 exponent bits with bias 1, 1 mantissa bit: 0, 0.5, 1, 1.5, 2, 3, */
/* 4, 6), round to nearest with ties to even, saturating at 6; one E8M0 scale  */
/* per 32 consecutive elements along the reduction dimension (every row of x, */
/* H and each weight matrix), the smallest 2^E with amax <= 6 * 2^E (code      */
/* clamped to [0, 254], 127 for an all-zero block).  Two codes per byte, the   */
/* even element in the low nibble.  Pinned in tests/test_oracle_pins.py.      */
/* ------------------------------------------------------------------------- */

ZO_EXPORT double zo_e2m1_decode(uint8_t c) {
  const int s = (c >> 3) & 1, E = (c >> 1) & 3, M = c & 1;
  const double v = (E == 0) ? 0.5 * M : ldexp(1.0 + 0.5 * M, E - 1);
  return s ? -v : v;
}

ZO_EXPORT uint8_t zo_e2m1_encode(float v) {
  const uint8_t sign = signbit(v) ? 0x8 : 0x0;
  const double a = fabs((double)v);
  if (!(a < 6.0)) return sign | 0x7; /* saturate (NaN included) */
  double q;                          /* spacing of representable magnitudes around a */
  if (a < 1.0) {
    q = 0.5;
  } else {
    int e;
    frexp(a, &e); /* a in [2^(e-1), 2^e) */
    q = ldexp(1.0, e - 1 - 1);
  }
  const double n = a / q;
  double r = floor(n);
  const double frac = n - r;
  if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) == 1.0)) r += 1.0;
  const double val = r * q;
  if (val < 1.0) return sign | (uint8_t)(val / 0.5); /* 0 or 0.5 */
  int ee;
  const double m = frexp(val, &ee); /* val = m * 2^ee, m in [0.5, 1) */
  const int E = ee - 1 + 1;
  const int M = (int)((2.0 * m - 1.0) * 2.0);
  return sign | (uint8_t)(E << 1) | (uint8_t)M;
}

ZO_EXPORT uint8_t zo_mx4_scale(float amax) {
  if (!(amax > 0.0f)) return 127;
  int e;
  frexp((double)amax, &e);
  const int k = e - 1; /* amax in [2^k, 2^(k+1)) */
  const int E = ((double)amax <= 1.5 * ldexp(1.0, k)) ? k - 2 : k - 1; /* 6 = 1.5 * 2^2 */
  int code = E + 127;
  if (code < 0) code = 0;
  if (code > 254) code = 254;
  return (uint8_t)code;
}

/* src [rows, cols] (dtype 0 fp32, 1 bf16 bits), cols a multiple of 32.
   codes [rows, cols/2] (two per byte, even element low); scales [rows, cols/32]. */
ZO_EXPORT void zo_quantize_mx4(const void *src, int dtype, int64_t rows, int64_t cols, uint8_t *codes,
                               uint8_t *scales) {
  const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static) if (rows * cols > (1 << 20))
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < nb; ++b) {
      double amax = 0.0;
      for (int64_t c = b * 32; c < b * 32 + 32; ++c) {
        const double a = fabs(elem(src, dtype, r * cols + c));
        if (a > amax) amax = a;
      }
      const uint8_t sc = zo_mx4_scale((float)amax);
      scales[r * nb + b] = sc;
      const double inv = ldexp(1.0, 127 - (int)sc);
      for (int64_t c = b * 32; c < b * 32 + 32; c += 2) {
        const uint8_t lo = zo_e2m1_encode((float)(elem(src, dtype, r * cols + c) * inv));
        const uint8_t hi = zo_e2m1_encode((float)(elem(src, dtype, r * cols + c + 1) * inv));
        codes[r * (cols / 2) + c / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
}

static double mx4_value(const uint8_t *codes, const uint8_t *scales, int64_t cols, int64_t r, int64_t c,
                        const double *tab) {
  const uint8_t byte = codes[r * (cols / 2) + c / 2];
  const uint8_t code = (c & 1) ? (byte >> 4) : (byte & 0xF);
  return tab[code] * ldexp(1.0, (int)scales[r * (cols / 32) + c / 32] - 127);
}

/* FFN expert on MXFP4 operands, fp64 arithmetic on the dequantized values.
   Each row of xs is quantized per [1,32] here; wg, wu [inter, d] and wd [d, inter]
   come as codes + scales ([1,32] along each row).  h = silu(g) * u is rounded to
   fp32 and quantized per [1,32] before the down projection (the kernel's
   precision, as for the FP8 expert).  out [n, d] fp64. */
ZO_EXPORT void zo_ffn_fp4_f64(const void *xs, int x_dtype, int64_t n, const uint8_t *wg, const uint8_t *sg,
                              const uint8_t *wu, const uint8_t *su, const uint8_t *wd, const uint8_t *sd, int d,
                              int inter, double *out) {
  const size_t xsz = (x_dtype == 1) ? 2 : 4;
  double tab[16];
  for (int c = 0; c < 16; ++c) tab[c] = zo_e2m1_decode((uint8_t)c);
  uint8_t *xq = (uint8_t *)malloc((size_t)d / 2), *xsc = (uint8_t *)malloc((size_t)d / 32);
  uint8_t *hq = (uint8_t *)malloc((size_t)inter / 2), *hsc = (uint8_t *)malloc((size_t)inter / 32);
  double *xv = (double *)malloc(sizeof(double) * (size_t)d), *hv = (double *)malloc(sizeof(double) * (size_t)inter);
  float *h32 = (float *)malloc(sizeof(float) * (size_t)inter);
  for (int64_t r = 0; r < n; ++r) {
    zo_quantize_mx4((const char *)xs + (size_t)(r * d) * xsz, x_dtype, 1, d, xq, xsc);
    for (int c = 0; c < d; ++c) xv[c] = mx4_value(xq, xsc, d, 0, c, tab);
#pragma omp parallel for schedule(static)
    for (int i = 0; i < inter; ++i) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < d; ++c) {
        const uint8_t bg = wg[(int64_t)i * (d / 2) + c / 2], bu = wu[(int64_t)i * (d / 2) + c / 2];
        const double sgv = ldexp(1.0, (int)sg[(int64_t)i * (d / 32) + c / 32] - 127);
        const double suv = ldexp(1.0, (int)su[(int64_t)i * (d / 32) + c / 32] - 127);
        g += (tab[(c & 1) ? bg >> 4 : bg & 0xF] * sgv) * xv[c];
        u += (tab[(c & 1) ? bu >> 4 : bu & 0xF] * suv) * xv[c];
      }
      h32[i] = (float)(g / (1.0 + exp(-g)) * u);
    }
    zo_quantize_mx4(h32, 0, 1, inter, hq, hsc);
    for (int i = 0; i < inter; ++i) hv[i] = mx4_value(hq, hsc, inter, 0, i, tab);
#pragma omp parallel for schedule(static)
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int i = 0; i < inter; ++i) acc += mx4_value(wd, sd, inter, c, i, tab) * hv[i];
      out[r * d + c] = acc;
    }
  }
  free(xq);
  free(xsc);
  free(hq);
  free(hsc);
  free(xv);
  free(hv);
  free(h32);
}

/* ------------------------------------------------------------------------- */
/* W4A4 as NVFP4 (the survey's name for the 4-bit format): E2M1 codes as in   */
/* MXFP4; one scale per 16 consecutive elements along the reduction dimension, */
/* an unsigned E4M3 value (UE4M3: the positive E4M3 values, 2^-9 .. 448); and  */
/* one fp32 scale g per tensor.  Reading (the pages name no format):           */
/*  - block scale: the smallest UE4M3 value s with amax <= 6 s g, decided in   */
/*    fp32: t = fl32(amax / fl32(6 g)), s = the smallest code value >= t (448  */
/*    at most); an all-zero block takes 1.0;                                   */
/*  - codes: e2m1(fl32(x * fl32(1 / fl32(s g)))), round to nearest even,       */
/*    saturating at 6;                                                         */
/*  - g: weights, one per expert matrix, fl32(amax(matrix) / 2688) (so the     */
/*    largest block scale is 448; 1 for an all-zero matrix); activations (x    */
/*    rows, silu(g)*u rows) g = 1: their magnitudes sit inside UE4M3's range.  */
/* Value = e2m1 * s * g.  Pinned in tests/test_oracle_pins.py.                 */
/* ------------------------------------------------------------------------- */

ZO_EXPORT float zo_nv4_global(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  const float r = amax / 2688.0f; /* 6 * 448, one fp32 division */
  return r;
}

ZO_EXPORT uint8_t zo_nv4_scale(float amax, float g) {
  if (!(amax > 0.0f)) return 0x38; /* 1.0 */
  const float six_g = 6.0f * g;
  const float t = amax / six_g;
  for (int c = 1; c <= 0x7E; ++c)
    if ((float)zo_e4m3_decode((uint8_t)c) >= t) return (uint8_t)c;
  return 0x7E; /* 448 */
}

/* src [rows, cols] (dtype 0 fp32, 1 bf16 bits), cols a multiple of 16; g the tensor's
   fp32 scale.  codes [rows, cols/2] (two per byte, even element low); scales
   [rows, cols/16] UE4M3 bytes. */
ZO_EXPORT void zo_quantize_nv4(const void *src, int dtype, int64_t rows, int64_t cols, float g, uint8_t *codes,
                               uint8_t *scales) {
  const int64_t nb = cols / 16;
#pragma omp parallel for schedule(static) if (rows * cols > (1 << 20))
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < nb; ++b) {
      double amax = 0.0;
      for (int64_t c = b * 16; c < b * 16 + 16; ++c) {
        const double a = fabs(elem(src, dtype, r * cols + c));
        if (a > amax) amax = a;
      }
      const uint8_t sc = zo_nv4_scale((float)amax, g);
      scales[r * nb + b] = sc;
      const float sg = (float)zo_e4m3_decode(sc) * g;
      const float inv = 1.0f / sg;
      for (int64_t c = b * 16; c < b * 16 + 16; c += 2) {
        const uint8_t lo = zo_e2m1_encode((float)elem(src, dtype, r * cols + c) * inv);
        const uint8_t hi = zo_e2m1_encode((float)elem(src, dtype, r * cols + c + 1) * inv);
        codes[r * (cols / 2) + c / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
}

static double nv4_value(const uint8_t *codes, const uint8_t *scales, int64_t cols, int64_t r, int64_t c,
                        const double *tab) {
  const uint8_t byte = codes[r * (cols / 2) + c / 2];
  const uint8_t code = (c & 1) ? (byte >> 4) : (byte & 0xF);
  return tab[code] * zo_e4m3_decode(scales[r * (cols / 16) + c / 16]);
}

/* FFN expert on NVFP4 operands, fp64 arithmetic on the dequantized values.  Each
   row of xs is quantized per [1,16] here with g = 1; wg, wu [inter, d] and wd
   [d, inter] come as codes + UE4M3 scales ([1,16] along each row) and their
   matrices' fp32 scales gg, gu, gd.  h = silu(g) * u is rounded to fp32 and
   quantized per [1,16] (g = 1) before the down projection.  out [n, d] fp64. */
ZO_EXPORT void zo_ffn_nv4_f64(const void *xs, int x_dtype, int64_t n, const uint8_t *wg, const uint8_t *sg, float gg,
                              const uint8_t *wu, const uint8_t *su, float gu, const uint8_t *wd, const uint8_t *sd,
                              float gd, int d, int inter, double *out) {
  const size_t xsz = (x_dtype == 1) ? 2 : 4;
  double tab[16];
  for (int c = 0; c < 16; ++c) tab[c] = zo_e2m1_decode((uint8_t)c);
  uint8_t *xq = (uint8_t *)malloc((size_t)d / 2), *xsc = (uint8_t *)malloc((size_t)d / 16);
  uint8_t *hq = (uint8_t *)malloc((size_t)inter / 2), *hsc = (uint8_t *)malloc((size_t)inter / 16);
  double *xv = (double *)malloc(sizeof(double) * (size_t)d), *hv = (double *)malloc(sizeof(double) * (size_t)inter);
  float *h32 = (float *)malloc(sizeof(float) * (size_t)inter);
  for (int64_t r = 0; r < n; ++r) {
    zo_quantize_nv4((const char *)xs + (size_t)(r * d) * xsz, x_dtype, 1, d, 1.0f, xq, xsc);
    for (int c = 0; c < d; ++c) xv[c] = nv4_value(xq, xsc, d, 0, c, tab);
#pragma omp parallel for schedule(static)
    for (int i = 0; i < inter; ++i) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < d; ++c) {
        g += nv4_value(wg, sg, d, i, c, tab) * xv[c];
        u += nv4_value(wu, su, d, i, c, tab) * xv[c];
      }
      g *= (double)gg;
      u *= (double)gu;
      h32[i] = (float)(g / (1.0 + exp(-g)) * u);
    }
    zo_quantize_nv4(h32, 0, 1, inter, 1.0f, hq, hsc);
    for (int i = 0; i < inter; ++i) hv[i] = nv4_value(hq, hsc, inter, 0, i, tab);
#pragma omp parallel for schedule(static)
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int i = 0; i < inter; ++i) acc += nv4_value(wd, sd, inter, c, i, tab) * hv[i];
      out[r * d + c] = acc * (double)gd;
    }
  }
  free(xq);
  free(xsc);
  free(hq);
  free(hsc);
  free(xv);
  free(hv);
  free(h32);
}

/* ------------------------------------------------------------------------- */
/* Backward pass (training), fp64.                                            */
/* LongCat-Flash technical summary (zhangjingwei.cn), 五 訓練基礎設施: the MoE   */
/* layer trains with a deterministic ScatterAdd and a fused GemmAdd (the fp32  */
/* gradient addition inside the GEMM epilogue).  The mathematics is the chain  */
/* rule through the forward above, with the routing decisions (which experts   */
/* a token picked) held fixed: they are a selection, not a differentiable      */
/* function.  Reading: the bias enters only the selection, so it receives no   */
/* gradient and contributes none; the logit offset is a constant.             */
/*   y_t = sum_j g_tj F_ej(x_t) + (sum over zero slots g_tj) x_t                */
/*   g_tj = scale * s_ej,  s = softmax(W_r x_t + o)                             */
/*   F(x) = W_d h,  h = silu(a) * b,  a = W_g x,  b = W_u x                      */
/* Given dy: dF = g dy;  dg_tj = <dy, F(x)> (FFN) or <dy, x> (zero);            */
/*   dh = W_d^T dF;  da = dh * b * silu'(a);  db = dh * silu(a);               */
/*   silu'(a) = sig(a) (1 + a (1 - sig(a)));                                    */
/*   dW_d += dF h^T;  dW_g += da x^T;  dW_u += db x^T;                           */
/*   dx += W_g^T da + W_u^T db (FFN slots) + g dy (zero slots);                  */
/*   ds_e = scale * dg (the slot that picked e);  dl = s * (ds - <s, ds>);      */
/*   dW_r += dl x^T;  dx += W_r^T dl.                                          */
/* Pinned by central finite differences in tests/test_oracle_pins.py.         */
/* Gradients are ADDED into dwr [E,d], dwg [N,inter,d], dwu, dwd [N,d,inter] */
/* (each may be NULL: skipped); dx [T,d] is written.  s [T,E] are the softmax */
/* scores of the forward.                                                     */
/* ------------------------------------------------------------------------- */
ZO_EXPORT void zo_layer_bwd_f64(const void *x, int x_dtype, int64_t T, int d, int E, int N, int k, int inter,
                                const void *wr, const void *wg, const void *wu, const void *wd, int w_dtype,
                                const int32_t *idx, const double *s, double scale, const double *dy, double *dx,
                                double *dwr, double *dwg, double *dwu, double *dwd) {
  double *xv = (double *)malloc(sizeof(double) * (size_t)d);
  double *a = (double *)malloc(sizeof(double) * (size_t)inter), *b = (double *)malloc(sizeof(double) * (size_t)inter);
  double *hh = (double *)malloc(sizeof(double) * (size_t)inter), *dh = (double *)malloc(sizeof(double) * (size_t)inter);
  double *F = (double *)malloc(sizeof(double) * (size_t)d), *dF = (double *)malloc(sizeof(double) * (size_t)d);
  double *ds = (double *)malloc(sizeof(double) * (size_t)E), *dl = (double *)malloc(sizeof(double) * (size_t)E);
  const int64_t wsz = (int64_t)inter * d;
  for (int64_t t = 0; t < T; ++t) {
    const double *dyt = dy + t * d;
    double *dxt = dx + t * d;
    for (int c = 0; c < d; ++c) {
      xv[c] = elem(x, x_dtype, t * d + c);
      dxt[c] = 0.0;
    }
    for (int e = 0; e < E; ++e) ds[e] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      const double g = scale * s[t * E + e];
      if (e >= N) { /* zero expert: F(x) = x */
        double dg = 0.0;
        for (int c = 0; c < d; ++c) {
          dg += dyt[c] * xv[c];
          dxt[c] += g * dyt[c];
        }
        ds[e] += scale * dg;
        continue;
      }
      const int64_t eo = (int64_t)e * wsz;
      for (int i = 0; i < inter; ++i) {
        double av = 0.0, bv = 0.0;
        for (int c = 0; c < d; ++c) {
          av += elem(wg, w_dtype, eo + (int64_t)i * d + c) * xv[c];
          bv += elem(wu, w_dtype, eo + (int64_t)i * d + c) * xv[c];
        }
        a[i] = av;
        b[i] = bv;
        hh[i] = av / (1.0 + exp(-av)) * bv;
      }
      double dg = 0.0;
      for (int c = 0; c < d; ++c) {
        double f = 0.0;
        for (int i = 0; i < inter; ++i) f += elem(wd, w_dtype, eo + (int64_t)c * inter + i) * hh[i];
        F[c] = f;
        dg += dyt[c] * f;
        dF[c] = g * dyt[c];
      }
      ds[e] += scale * dg;
      for (int i = 0; i < inter; ++i) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += elem(wd, w_dtype, eo + (int64_t)c * inter + i) * dF[c];
        dh[i] = acc;
      }
      if (dwd)
        for (int c = 0; c < d; ++c)
          for (int i = 0; i < inter; ++i) dwd[eo + (int64_t)c * inter + i] += dF[c] * hh[i];
      for (int i = 0; i < inter; ++i) {
        const double sg = 1.0 / (1.0 + exp(-a[i]));
        const double da = dh[i] * b[i] * sg * (1.0 + a[i] * (1.0 - sg));
        const double db = dh[i] * a[i] * sg;
        for (int c = 0; c < d; ++c) {
          if (dwg) dwg[eo + (int64_t)i * d + c] += da * xv[c];
          if (dwu) dwu[eo + (int64_t)i * d + c] += db * xv[c];
          dxt[c] += elem(wg, w_dtype, eo + (int64_t)i * d + c) * da + elem(wu, w_dtype, eo + (int64_t)i * d + c) * db;
        }
      }
    }
    /* router: softmax Jacobian */
    double sds = 0.0;
    for (int e = 0; e < E; ++e) sds += s[t * E + e] * ds[e];
    for (int e = 0; e < E; ++e) dl[e] = s[t * E + e] * (ds[e] - sds);
    for (int e = 0; e < E; ++e)
      for (int c = 0; c < d; ++c) {
        if (dwr) dwr[(int64_t)e * d + c] += dl[e] * xv[c];
        dxt[c] += elem(wr, w_dtype, (int64_t)e * d + c) * dl[e];
      }
  }
  free(xv);
  free(a);
  free(b);
  free(hh);
  free(dh);
  free(F);
  free(dF);
  free(ds);
  free(dl);
}
