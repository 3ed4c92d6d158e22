/*
 * moe_oracle.c -- plain, slow CPU reference for the batch-1 MXFP4 MoE decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares no
 * code, header, table or helper with the CUDA library under
 * moe_decode_weight_router_b200/csrc, and neither side includes the other.
 *
 * Every value is computed in fp64 from the same quantised bytes the GPU reads,
 * except where a step is *defined* in fp32 (the LM-head e4m3 quantiser and the
 * MXFP8 activation quantiser, whose bytes must match the GPU's bit for bit).
 * No blocking, fusion or reordering beyond the plain definition.
 *
 * Sources (the pages give names and shapes, never bit layouts or formulas):
 *  - "知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的三种方法" (the DGX Spark
 *    MoE knowledge card), section 方法/产品要点 ("methods"), item 1: routed experts
 *    run an MXFP4 MoE kernel with moe_intermediate_size = 768; item 2: the LM
 *    head (vocabulary GEMM 157,184 x 2,560, BF16 in the checkpoint) gets an
 *    online dynamic FP8 quantisation; item 3: a 4-token verify window can fire
 *    up to 32 experts; section 事件概述 ("overview"): each MoE layer routes a
 *    token to 8 of 512 routed experts plus 1 shared expert.
 *  - "英伟达称不换芯片也能提速：DGX Spark靠软件优化多吐42.5%的token", section
 *    不换卡，快在哪: FP8 halves the LM-head read bytes.
 *  - OCP Microscaling Formats (MX) Specification v1.0: FP4 E2M1 element,
 *    E8M0 shared scale (2^(e-127), 0xFF = NaN), FP8 E4M3 element (bias 7,
 *    max normal 448, no infinities, S.1111.111 = NaN), block size 32, and the
 *    shared-exponent rule floor(log2(amax)) - emax_elem used for MXFP8.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - routing = softmax over all experts, top-k on the logits (ties to the lower
 *    index), weights renormalised over the k selected (equals the softmax of
 *    the k selected logits);
 *  - MXFP4 codes packed two per byte along the input dimension, element 2j in
 *    the low nibble of byte j; scale b covers input elements [32b, 32b+32);
 *  - W13 rows [0, I) are the gate projection, rows [I, 2I) the up projection;
 *    SwiGLU a = silu(gate) * up;
 *  - decode activations stay BF16 (weights-only quantisation);
 *  - LM head: one fp32 scale per output row, s = amax/448 (1.0 when amax = 0),
 *    codes = e4m3 round-to-nearest-even, saturating, of w/s computed in fp32;
 *  - chained layers: h <- h + y, next input bf16(RMSNorm(h)), unit weight,
 *    eps 1e-6; the LM head reads bf16(RMSNorm(h_L));
 *  - prefill chunk: activations and the SwiGLU output quantised to MXFP8
 *    (e4m3 codes, E8M0 scale per 32) before the routed products; the shared
 *    expert stays BF16 with its SwiGLU output rounded to BF16.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

#ifdef _OPENMP
#include <omp.h>
#endif

/* Host threads the parallel loops below use (n >= 1); timing only, no arithmetic. */
EXPORT void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------------- */
/* Formats                                                                    */
/* ------------------------------------------------------------------------- */

/* FP4 E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 * e = 0 is subnormal: m * 0.5.  Otherwise 2^(e-1) * (1 + m/2). */
EXPORT double orc_e2m1(unsigned code) {
  unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
  double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
  return s ? -mag : mag;
}

/* E8M0 shared scale: 2^(e-127); 0xFF encodes NaN. */
EXPORT double orc_e8m0(unsigned e) {
  if (e == 255u) return NAN;
  return ldexp(1.0, (int)e - 127);
}

/* FP8 E4M3 ("FN" variant): bit 7 sign, bits 6..3 exponent (bias 7),
 * bits 2..0 mantissa.  e = 0 is subnormal m/8 * 2^-6.  No infinities;
 * exponent 15 with mantissa 7 is NaN. */
EXPORT double orc_e4m3(unsigned code) {
  unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
  if (e == 15u && m == 7u) return NAN;
  double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, (int)e - 7);
  return s ? -mag : mag;
}

/* BF16 bits -> value (the upper half of an IEEE binary32). */
EXPORT double orc_bf16(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Nearest BF16 to v, ties to the even significand (IEEE round-to-nearest-even),
 * computed directly on the fp64 value: one rounding, no detour through fp32. */
EXPORT uint16_t orc_bf16_rne(double v) {
  if (isnan(v)) return 0x7FC0u;
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (isinf(a)) return sign | 0x7F80u;
  if (a == 0.0) return sign;
  int ex;
  (void)frexp(a, &ex);           /* a = f * 2^ex, f in [0.5, 1) */
  int qe = ex - 8;               /* 8 significant bits: quantum 2^(ex-8) */
  if (qe < -133) qe = -133;      /* subnormal quantum 2^-133 */
  double n = ldexp(a, -qe);      /* exact */
  double fl = floor(n), r = n - fl;
  if (r > 0.5 || (r == 0.5 && fmod(fl, 2.0) == 1.0)) fl += 1.0;
  double res = ldexp(fl, qe);
  /* largest finite bf16 = (2 - 2^-7) * 2^127; anything that rounds above it is inf */
  if (res > ldexp(255.0, 120)) return sign | 0x7F80u;
  float f = (float)res; /* exact: res has <= 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return sign | (uint16_t)(u >> 16);
}

/* e4m3 encode of an fp32 value: the nearest finite e4m3 value by exhaustive
 * search over the 127 non-negative finite codes, ties to the even code (the
 * even mantissa); magnitudes at or above 448 saturate to 448; sign kept
 * (a value that rounds to zero keeps its sign: -0 = 0x80); NaN -> 0x7F. */
EXPORT uint8_t orc_e4m3_encode(float v) {
  if (isnan(v)) return 0x7Fu;
  unsigned sign = signbit(v) ? 0x80u : 0u;
  double a = fabs((double)v);
  if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);
  unsigned best = 0;
  double bd = INFINITY;
  for (unsigned c = 0; c <= 0x7Eu; ++c) {
    double d = fabs(orc_e4m3(c) - a);
    if (d < bd || (d == bd && (c & 1u) == 0u)) {
      bd = d;
      best = c;
    }
  }
  return (uint8_t)(sign | best);
}

/* MXFP4 element (row r, column h) of a row-major [rows][cols] tensor whose codes
 * are [rows][cols/2] bytes and scales [rows][cols/32] bytes. */
static double mxfp4_at(const uint8_t* codes, const uint8_t* scales, int cols, long r, int h) {
  uint8_t byte = codes[r * (long)(cols / 2) + h / 2];
  unsigned nib = (h & 1) ? (byte >> 4) : (byte & 15u);
  return orc_e2m1(nib) * orc_e8m0(scales[r * (long)(cols / 32) + h / 32]);
}

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* ------------------------------------------------------------------------- */
/* Router                                                                     */
/* ------------------------------------------------------------------------- */

/* Per token t: l[e] = sum_h x[t,h] * Wr[e,h] (bf16 inputs, fp64 sums); the k
 * largest logits by (value descending, index ascending); weights = softmax of
 * the selected logits (= full softmax renormalised over the selected).
 * margin[t] = l_(k) - l_(k+1), the gap that decides the last selection
 * (+inf when k == E).  logits_out may be NULL. */
EXPORT void orc_route(const uint16_t* x, int M, int H, const uint16_t* wr, int E, int k,
                      int32_t* ids, double* w, double* logits_out, double* margin) {
  double* l = (double*)malloc(sizeof(double) * (size_t)E);
  char* taken = (char*)malloc((size_t)E);
  for (int t = 0; t < M; ++t) {
#pragma omp parallel for schedule(static)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += orc_bf16(x[(long)t * H + h]) * orc_bf16(wr[(long)e * H + h]);
      l[e] = acc;
    }
    if (logits_out)
      for (int e = 0; e < E; ++e) logits_out[(long)t * E + e] = l[e];
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e; /* strict '>' keeps the lower index */
      taken[best] = 1;
      ids[t * k + j] = best;
    }
    double next = -INFINITY;
    int have_next = 0;
    for (int e = 0; e < E; ++e)
      if (!taken[e] && (!have_next || l[e] > next)) {
        next = l[e];
        have_next = 1;
      }
    margin[t] = have_next ? l[ids[t * k + k - 1]] - next : INFINITY;
    double lmax = l[ids[t * k]], den = 0.0;
    for (int j = 0; j < k; ++j) den += exp(l[ids[t * k + j]] - lmax);
    for (int j = 0; j < k; ++j) w[t * k + j] = exp(l[ids[t * k + j]] - lmax) / den;
  }
  free(l);
  free(taken);
}

/* ------------------------------------------------------------------------- */
/* MoE layer, decode (weights MXFP4, activations BF16)                        */
/* ------------------------------------------------------------------------- */

/* y[t,:] = sum_j w[t,j] * W2_{e} (silu(Wg_{e} x_t) * Wu_{e} x_t),  e = ids[t,j]
 *        + Ws2 (silu(Wsg x_t) * Wsu x_t)                          (if shared)
 * Routed tensors are indexed by expert id in [0, nE):
 *   w13c [nE][2I][H/2], w13s [nE][2I][H/32], w2c [nE][H][I/2], w2s [nE][H][I/32].
 * Shared: sw13 bf16 [2Is][H], sw2 bf16 [H][Is]; pass NULL (or Is = 0) for none.
 * A weight w[t,j] of exactly 0 still evaluates the expert (no skipping). */
EXPORT void orc_moe_layer(const uint16_t* x, int M, int H, int I, int nE, int k,
                          const int32_t* ids, const double* w,
                          const uint8_t* w13c, const uint8_t* w13s,
                          const uint8_t* w2c, const uint8_t* w2s,
                          const uint16_t* sw13, const uint16_t* sw2, int Is,
                          double* y) {
  int Imax = I > Is ? I : Is;
  double* xd = (double*)malloc(sizeof(double) * (size_t)H);
  double* a = (double*)malloc(sizeof(double) * (size_t)Imax);
  for (int t = 0; t < M; ++t) {
    for (int h = 0; h < H; ++h) xd[h] = orc_bf16(x[(long)t * H + h]);
    for (int h = 0; h < H; ++h) y[(long)t * H + h] = 0.0;
    for (int j = 0; j < k; ++j) {
      int e = ids[t * k + j];
      double wt = w[t * k + j];
      if (e < 0 || e >= nE) { /* an id outside the expert range poisons the row */
        for (int h = 0; h < H; ++h) y[(long)t * H + h] = NAN;
        continue;
      }
      const long base13 = (long)e * 2 * I;
#pragma omp parallel for schedule(static)
      for (int r = 0; r < I; ++r) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
          g += mxfp4_at(w13c, w13s, H, base13 + r, h) * xd[h];
          u += mxfp4_at(w13c, w13s, H, base13 + I + r, h) * xd[h];
        }
        a[r] = silu(g) * u;
      }
      const long base2 = (long)e * H;
#pragma omp parallel for schedule(static)
      for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int r = 0; r < I; ++r) acc += mxfp4_at(w2c, w2s, I, base2 + h, r) * a[r];
        y[(long)t * H + h] += wt * acc;
      }
    }
    if (sw13 && sw2 && Is > 0) {
#pragma omp parallel for schedule(static)
      for (int r = 0; r < Is; ++r) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
          g += orc_bf16(sw13[(long)r * H + h]) * xd[h];
          u += orc_bf16(sw13[(long)(Is + r) * H + h]) * xd[h];
        }
        a[r] = silu(g) * u;
      }
#pragma omp parallel for schedule(static)
      for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int r = 0; r < Is; ++r) acc += orc_bf16(sw2[(long)h * Is + r]) * a[r];
        y[(long)t * H + h] += acc;
      }
    }
  }
  free(xd);
  free(a);
}

/* ------------------------------------------------------------------------- */
/* Layer chaining stand-in and the LM head                                    */
/* ------------------------------------------------------------------------- */

/* x_out[t,:] = bf16( h[t,:] / sqrt(mean_h h[t,h]^2 + eps) )  (unit weight). */
EXPORT void orc_rmsnorm_bf16(const double* h, int M, int H, double eps, uint16_t* x_out) {
  for (int t = 0; t < M; ++t) {
    double ss = 0.0;
    for (int i = 0; i < H; ++i) ss += h[(long)t * H + i] * h[(long)t * H + i];
    double r = 1.0 / sqrt(ss / (double)H + eps);
    for (int i = 0; i < H; ++i) x_out[(long)t * H + i] = orc_bf16_rne(h[(long)t * H + i] * r);
  }
}

/* Online FP8 quantisation of a BF16 [V][H] LM head, defined in fp32:
 *   amax_v = max_h |W[v,h]|;  s_v = amax_v / 448 (fp32 division; 1.0 if amax_v = 0)
 *   q[v,h] = e4m3_rne_sat( W[v,h] / s_v )   (fp32 division)                 */
EXPORT void orc_lmhead_quantize(const uint16_t* wt, int V, int H, uint8_t* q, float* s) {
#pragma omp parallel for schedule(static)
  for (int v = 0; v < V; ++v) {
    float amax = 0.0f;
    for (int h = 0; h < H; ++h) {
      float a = fabsf((float)orc_bf16(wt[(long)v * H + h]));
      if (a > amax) amax = a;
    }
    volatile float sv = (amax == 0.0f) ? 1.0f : amax / 448.0f;
    s[v] = sv;
    for (int h = 0; h < H; ++h) {
      volatile float qv = (float)orc_bf16(wt[(long)v * H + h]) / sv;
      q[(long)v * H + h] = orc_e4m3_encode(qv);
    }
  }
}

/* logits[t,v] = s_v * sum_h e4m3(q[v,h]) * x[t,h]   (fp64)
 * argmax[t] = the largest logit, lowest index on ties; gap[t] = top1 - top2. */
EXPORT void orc_lmhead_logits(const uint16_t* x, int M, int V, int H, const uint8_t* q, const float* s,
                              double* logits, int32_t* argmax, double* gap) {
  double* xd = (double*)malloc(sizeof(double) * (size_t)H);
  for (int t = 0; t < M; ++t) {
    for (int h = 0; h < H; ++h) xd[h] = orc_bf16(x[(long)t * H + h]);
#pragma omp parallel for schedule(static)
    for (int v = 0; v < V; ++v) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h) acc += orc_e4m3(q[(long)v * H + h]) * xd[h];
      logits[(long)t * V + v] = (double)s[v] * acc;
    }
    int best = 0;
    for (int v = 1; v < V; ++v)
      if (logits[(long)t * V + v] > logits[(long)t * V + best]) best = v;
    double second = -INFINITY;
    for (int v = 0; v < V; ++v)
      if (v != best && logits[(long)t * V + v] > second) second = logits[(long)t * V + v];
    argmax[t] = best;
    gap[t] = logits[(long)t * V + best] - second;
  }
  free(xd);
}

/* ------------------------------------------------------------------------- */
/* Prefill chunk: MXFP8 activations (OCP MX conversion rule)                  */
/* ------------------------------------------------------------------------- */

/* Quantise rows of fp32 values to MXFP8 (E4M3 elements, one E8M0 scale per 32):
 *   amax = max |v| over the block; s = floor(log2 amax) - 8 (8 = the E4M3
 *   emax), clamped to [-127, 127]; s = -127 and all codes 0 when amax = 0;
 *   q = e4m3_rne_sat(v * 2^-s) (an exact fp32 scaling); stored scale = s + 127.
 * v [M][K] fp32, q [M][K] bytes, se [M][K/32] bytes. */
EXPORT void orc_mxfp8_quantize(const float* v, int M, int K, uint8_t* q, uint8_t* se) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < M; ++t) {
    for (int b = 0; b < K / 32; ++b) {
      const float* blk = v + (long)t * K + 32L * b;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i)
        if (fabs((double)blk[i]) > amax) amax = fabs((double)blk[i]);
      int s;
      if (amax == 0.0) {
        s = -127;
      } else {
        int ex;
        (void)frexp(amax, &ex); /* amax = f 2^ex, f in [0.5,1): floor(log2 amax) = ex - 1 */
        s = (ex - 1) - 8;
        if (s < -127) s = -127;
        if (s > 127) s = 127;
      }
      se[(long)t * (K / 32) + b] = (uint8_t)(s + 127);
      for (int i = 0; i < 32; ++i) {
        volatile float sc = (float)ldexp((double)blk[i], -s); /* exact power-of-two scaling */
        q[(long)t * K + 32L * b + i] = (amax == 0.0) ? 0u : orc_e4m3_encode(sc);
      }
    }
  }
}

/* Dequantised MXFP8 value of element i of row t. */
static double mxfp8_at(const uint8_t* q, const uint8_t* se, int K, long t, int i) {
  return orc_e4m3(q[t * K + i]) * orc_e8m0(se[t * (long)(K / 32) + i / 32]);
}

/* Prefill layer over a subset of tokens.  x is bf16 [M][H]; only the tokens
 * listed in tok[0..nt) are evaluated, writing y[j][:] for tok[j].
 * Routed path: x -> MXFP8 (per token, per 32 along H), W13 MXFP4 product in
 * fp64, a = silu(g) u in fp64, a rounded to fp32 then MXFP8 (per 32 along I),
 * W2 product in fp64, weighted sum.  Shared path: BF16 weights and x, fp64
 * sums, a_s rounded to BF16 before Ws2. */
EXPORT void orc_moe_layer_prefill(const uint16_t* x, int M, int H, int I, int nE, int k,
                                  const int32_t* ids, const double* w,
                                  const uint8_t* w13c, const uint8_t* w13s,
                                  const uint8_t* w2c, const uint8_t* w2s,
                                  const uint16_t* sw13, const uint16_t* sw2, int Is,
                                  const int32_t* tok, int nt, double* y) {
  (void)M;
  int Imax = I > Is ? I : Is;
  float* xf = (float*)malloc(sizeof(float) * (size_t)H);
  uint8_t* xq = (uint8_t*)malloc((size_t)H);
  uint8_t* xs = (uint8_t*)malloc((size_t)(H / 32));
  double* xd = (double*)malloc(sizeof(double) * (size_t)H);
  double* xb = (double*)malloc(sizeof(double) * (size_t)H);
  double* a = (double*)malloc(sizeof(double) * (size_t)Imax);
  float* af = (float*)malloc(sizeof(float) * (size_t)Imax);
  uint8_t* aq = (uint8_t*)malloc((size_t)Imax);
  uint8_t* as = (uint8_t*)malloc((size_t)(Imax / 32 + 1));
  for (int jt = 0; jt < nt; ++jt) {
    long t = tok[jt];
    for (int h = 0; h < H; ++h) {
      xb[h] = orc_bf16(x[t * H + h]);
      xf[h] = (float)xb[h];
    }
    orc_mxfp8_quantize(xf, 1, H, xq, xs);
    for (int h = 0; h < H; ++h) xd[h] = mxfp8_at(xq, xs, H, 0, h);
    double* yt = y + (long)jt * H;
    for (int h = 0; h < H; ++h) yt[h] = 0.0;
    for (int j = 0; j < k; ++j) {
      int e = ids[t * k + j];
      double wt = w[t * k + j];
      if (e < 0 || e >= nE) { /* an id outside the expert range poisons the row */
        for (int h = 0; h < H; ++h) yt[h] = NAN;
        continue;
      }
      const long base13 = (long)e * 2 * I;
#pragma omp parallel for schedule(static)
      for (int r = 0; r < I; ++r) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
          g += mxfp4_at(w13c, w13s, H, base13 + r, h) * xd[h];
          u += mxfp4_at(w13c, w13s, H, base13 + I + r, h) * xd[h];
        }
        a[r] = silu(g) * u;
        af[r] = (float)a[r];
      }
      orc_mxfp8_quantize(af, 1, I, aq, as);
      const long base2 = (long)e * H;
#pragma omp parallel for schedule(static)
      for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int r = 0; r < I; ++r) acc += mxfp4_at(w2c, w2s, I, base2 + h, r) * mxfp8_at(aq, as, I, 0, r);
        yt[h] += wt * acc;
      }
    }
    if (sw13 && sw2 && Is > 0) {
#pragma omp parallel for schedule(static)
      for (int r = 0; r < Is; ++r) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
          g += orc_bf16(sw13[(long)r * H + h]) * xb[h];
          u += orc_bf16(sw13[(long)(Is + r) * H + h]) * xb[h];
        }
        a[r] = orc_bf16(orc_bf16_rne(silu(g) * u));
      }
#pragma omp parallel for schedule(static)
      for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int r = 0; r < Is; ++r) acc += orc_bf16(sw2[(long)h * Is + r]) * a[r];
        yt[h] += acc;
      }
    }
  }
  free(xf); free(xq); free(xs); free(xd); free(xb); free(a); free(af); free(aq); free(as);
}
