/*
 * CPU oracle of the fused grouped W4A16 routed-expert MoE layer, in plain C.
 *
 * TEST INFRASTRUCTURE ONLY, like the numpy oracle beside it: only tests/,
 * __graft_entry__.smoke() and bench.py's CPU-baseline/reference legs may load
 * it. It shares no code, header, table or constant generator with the CUDA
 * library, and none with the numpy oracle either: the two oracles are written
 * independently from the same definitions and checked against each other.
 *
 * Source: "Every Expert Counts: ExactMoE for Memory-Efficient W4A16
 * Inference" (A. Saab, arXiv 2608.15383):
 *   - Abstract: only the routed experts are quantised, four-bit, symmetric,
 *     in groups of 128; router and activations stay BF16; exactness means
 *     that every chosen expert is run and top-k routing is left as it was.
 *   - Figure 1 caption: the order of the steps. The BF16 router picks the
 *     experts, the tokens are gathered per chosen expert, fused grouped
 *     kernels run the active experts, and they read the packed codes and
 *     scales directly, with no FP16 copy of any expert.
 * The pages give no formula, so each function below states the plainest
 * reading of those passages it implements (the same readings as the numpy
 * oracle): quantiser s = bf16_rn(absmax/7) (fp32 divide), q = clamp(rint(w/s),
 * -8, 7) (fp32 divide, ties to even), s = 0 and q = 0 for an all-zero group;
 * offset-binary nibbles u = q + 8, k = 8j + 2i + h of a row at bits 4(i+4h)
 * of little-endian word j; router logits bf16_rn of an fp64 sum; top-k on
 * fp32 keys (logit + bias, NaN as -inf), ties to the lower index, ordered by
 * descending key then ascending index, weights the full-softmax
 * probabilities (optionally renormalised); grouping stable by expert;
 * SwiGLU with exact dequantised weights q*s, fp64 sums, h rounded to BF16;
 * combine in fp64 in j order with one BF16 rounding.
 *
 * Arithmetic is fp64 except where floating point decides an integer (the
 * quantiser, the top-k comparison), which runs in fp32. Loops are the plain
 * definitions; OpenMP only runs independent experts or tokens side by side
 * (each result is computed by one thread in a fixed order, so the results do
 * not depend on the thread count).
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (see c_oracle.py).
 */
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EO_GROUP 128

/* ------------------------------------------------------------ BF16 helpers */

static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Nearest BF16 value of a double, ties to even, one rounding from the exact
 * value: for |x| = m * 2^e (0.5 <= m < 1) the spacing is 2^(e-8), never finer
 * than 2^-133; at or above 2^128 the result is infinite. */
static double round_bf16(double x) {
  if (!isfinite(x) || x == 0.0) return x;
  int e;
  frexp(x, &e);
  int ue = e - 8;
  if (ue < -133) ue = -133;
  double r = ldexp(nearbyint(ldexp(x, -ue)), ue);
  if (fabs(r) >= ldexp(1.0, 128)) r = copysign(INFINITY, x);
  return r;
}

/* Bits of a value that is already BF16-representable. */
static uint16_t bf16_bits(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------- A1: quantise and pack */

/* w [N][K] BF16 bits -> packed [N][K/2] bytes and scales [N][K/128] BF16 bits.
 * Returns 0, or -1 when K is not a multiple of 128. */
int eo_quantize_pack(const uint16_t *w, int N, int K, uint8_t *packed, uint16_t *scales) {
  if (K % EO_GROUP) return -1;
  const int G = K / EO_GROUP;
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const uint16_t *wg = w + (size_t)n * K + (size_t)g * EO_GROUP;
      float absmax = 0.0f;
      for (int i = 0; i < EO_GROUP; ++i) {
        float a = fabsf(bf16_to_f32(wg[i]));
        if (a > absmax) absmax = a;
      }
      const float s32 = absmax / 7.0f;
      const uint16_t sb = bf16_bits(round_bf16((double)s32));
      scales[(size_t)n * G + g] = sb;
      const float s = bf16_to_f32(sb);
      uint8_t *row = packed + (size_t)n * (K / 2) + (size_t)g * (EO_GROUP / 2);
      for (int j = 0; j < EO_GROUP / 8; ++j) {
        uint32_t word = 0;
        for (int i = 0; i < 4; ++i)
          for (int h = 0; h < 2; ++h) {
            const int kk = 8 * j + 2 * i + h;
            int q = 0;
            if (s != 0.0f) {
              const float r = rintf(bf16_to_f32(wg[kk]) / s);
              q = r > 7.0f ? 7 : (r < -8.0f ? -8 : (int)r);
            }
            word |= (uint32_t)(q + 8) << (4 * (i + 4 * h));
          }
        row[4 * j + 0] = (uint8_t)(word & 0xFF);
        row[4 * j + 1] = (uint8_t)((word >> 8) & 0xFF);
        row[4 * j + 2] = (uint8_t)((word >> 16) & 0xFF);
        row[4 * j + 3] = (uint8_t)(word >> 24);
      }
    }
  }
  return 0;
}

/* One row of a packed matrix back to its exact values q * s (fp64). */
static void dequant_row(const uint8_t *prow, const uint16_t *srow, int K, double *out) {
  for (int k = 0; k < K; ++k) {
    const int j = k / 8, i = (k % 8) / 2, h = k % 2;
    const uint32_t word = (uint32_t)prow[4 * j] | ((uint32_t)prow[4 * j + 1] << 8) |
                          ((uint32_t)prow[4 * j + 2] << 16) | ((uint32_t)prow[4 * j + 3] << 24);
    const int q = (int)((word >> (4 * (i + 4 * h))) & 0xF) - 8;
    out[k] = (double)q * (double)bf16_to_f32(srow[k / EO_GROUP]);
  }
}

/* packed [N][K/2] + scales -> w [N][K] (fp64), the exact dequantised matrix. */
void eo_dequantize(const uint8_t *packed, const uint16_t *scales, int N, int K, double *w) {
  for (int n = 0; n < N; ++n)
    dequant_row(packed + (size_t)n * (K / 2), scales + (size_t)n * (K / EO_GROUP), K, w + (size_t)n * K);
}

/* ------------------------------------------------------ A2: router logits */

/* logits[t][e] = bf16_rn(sum_h x[t][h] * wr[e][h]), fp64 sum in h order. */
void eo_router_logits(const uint16_t *x, const uint16_t *wr, int T, int H, int E, uint16_t *logits) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += (double)bf16_to_f32(x[(size_t)t * H + h]) * (double)bf16_to_f32(wr[(size_t)e * H + h]);
      logits[(size_t)t * E + e] = bf16_bits(round_bf16(acc));
    }
}

/* ------------------------------------------------ A3: softmax + top-k */

/* ids [T][k], w [T][k]. bias may be NULL. Returns 0, or -1 for a bad k. */
int eo_route_topk(const uint16_t *logits, const float *bias, int T, int E, int k, int renorm, int32_t *ids,
                  double *w) {
  if (k < 1 || k > E) return -1;
  float *key = (float *)malloc(sizeof(float) * (size_t)E);
  char *taken = (char *)malloc((size_t)E);
  if (!key || !taken) { free(key); free(taken); return -2; }
  for (int t = 0; t < T; ++t) {
    float m = -INFINITY;
    for (int e = 0; e < E; ++e) {
      float v = bf16_to_f32(logits[(size_t)t * E + e]);
      if (bias) v = v + bias[e];
      if (isnan(v)) v = -INFINITY;
      key[e] = v;
      taken[e] = 0;
      if (v > m) m = v;
    }
    /* k rounds: the largest untaken key, the lowest index among equals */
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || key[e] > key[best])) best = e;
      taken[best] = 1;
      ids[(size_t)t * k + j] = best;
    }
    /* full softmax over all experts, fp64 */
    double sum = 0.0;
    for (int e = 0; e < E; ++e) sum += exp((double)key[e] - (double)m);
    double wsum = 0.0;
    for (int j = 0; j < k; ++j) {
      const double p = exp((double)key[ids[(size_t)t * k + j]] - (double)m) / sum;
      w[(size_t)t * k + j] = p;
      wsum += p;
    }
    if (renorm)
      for (int j = 0; j < k; ++j) w[(size_t)t * k + j] /= wsum;
  }
  free(key);
  free(taken);
  return 0;
}

/* ------------------------------------------------------------ A4: grouping */

/* counts [E], offsets [E+1], sorted_pair [T*k], pair_pos [T*k]. Pairs p =
 * t*k + j are listed by expert, and by p within an expert. Returns 0, or -1
 * for an expert id outside [0, E). */
int eo_group_tokens(const int32_t *ids, int T, int k, int E, int32_t *counts, int32_t *offsets, int32_t *sorted_pair,
                    int32_t *pair_pos) {
  const long P = (long)T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (long p = 0; p < P; ++p) {
    if (ids[p] < 0 || ids[p] >= E) return -1;
    counts[ids[p]] += 1;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
  if (!next) return -2;
  for (int e = 0; e < E; ++e) next[e] = offsets[e];
  for (long p = 0; p < P; ++p) {
    const int32_t r = next[ids[p]]++;
    sorted_pair[r] = (int32_t)p;
    pair_pos[p] = r;
  }
  free(next);
  return 0;
}

/* ---------------------------------------------- A5 + A6: expert SwiGLU FFN */

/* The packed experts of one layer: per matrix [E][N][K/2] codes and
 * [E][N][K/128] scale bits (gate, up: N = I, K = H; down: N = H, K = I). */
typedef struct {
  const uint8_t *gq, *uq, *dq;
  const uint16_t *gs, *us, *ds;
  int E, H, I;
} eo_experts;

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* Rows of one expert: xr [R][H] (fp64, BF16 values) -> h [R][I] (BF16 values)
 * and y [R][H] (fp64). Rows of W are dequantised one at a time. */
static int expert_rows(const eo_experts *X, int e, const double *xr, int R, double *h, double *y) {
  const int H = X->H, I = X->I;
  double *wg = (double *)malloc(sizeof(double) * (size_t)H);
  double *wu = (double *)malloc(sizeof(double) * (size_t)H);
  double *wd = (double *)malloc(sizeof(double) * (size_t)I);
  if (!wg || !wu || !wd) { free(wg); free(wu); free(wd); return -2; }
  const size_t gq_e = (size_t)e * I * (H / 2), gs_e = (size_t)e * I * (H / EO_GROUP);
  for (int i = 0; i < I; ++i) {
    dequant_row(X->gq + gq_e + (size_t)i * (H / 2), X->gs + gs_e + (size_t)i * (H / EO_GROUP), H, wg);
    dequant_row(X->uq + gq_e + (size_t)i * (H / 2), X->us + gs_e + (size_t)i * (H / EO_GROUP), H, wu);
    for (int r = 0; r < R; ++r) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < H; ++c) {
        g += xr[(size_t)r * H + c] * wg[c];
        u += xr[(size_t)r * H + c] * wu[c];
      }
      h[(size_t)r * I + i] = round_bf16(silu(g) * u);
    }
  }
  const size_t dq_e = (size_t)e * H * (I / 2), ds_e = (size_t)e * H * (I / EO_GROUP);
  for (int n = 0; n < H; ++n) {
    dequant_row(X->dq + dq_e + (size_t)n * (I / 2), X->ds + ds_e + (size_t)n * (I / EO_GROUP), I, wd);
    for (int r = 0; r < R; ++r) {
      double acc = 0.0;
      for (int c = 0; c < I; ++c) acc += h[(size_t)r * I + c] * wd[c];
      y[(size_t)r * H + n] = acc;
    }
  }
  free(wg);
  free(wu);
  free(wd);
  return 0;
}

/* Grouped form: for each expert, its rows in sorted order (token =
 * sorted_pair[r] / k). x [T][H] BF16 bits; h [P][I], y [P][H] fp64. */
int eo_grouped_ffn(const uint16_t *x, int T, const int32_t *sorted_pair, const int32_t *offsets, int k,
                   const uint8_t *gq, const uint16_t *gs, const uint8_t *uq, const uint16_t *us, const uint8_t *dq,
                   const uint16_t *ds, int E, int H, int I, double *h, double *y) {
  if (H % EO_GROUP || I % EO_GROUP) return -1;
  const eo_experts X = {gq, uq, dq, gs, us, ds, E, H, I};
  int status = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int e = 0; e < E; ++e) {
    const int lo = offsets[e], R = offsets[e + 1] - offsets[e];
    if (R <= 0) continue;
    double *xr = (double *)malloc(sizeof(double) * (size_t)R * H);
    if (!xr) {
#pragma omp atomic write
      status = -2;
      continue;
    }
    for (int r = 0; r < R; ++r) {
      const int t = sorted_pair[lo + r] / k;
      for (int c = 0; c < H; ++c) xr[(size_t)r * H + c] = (double)bf16_to_f32(x[(size_t)t * H + c]);
    }
    if (expert_rows(&X, e, xr, R, h + (size_t)lo * I, y + (size_t)lo * H) != 0) {
#pragma omp atomic write
      status = -2;
    }
    free(xr);
  }
  (void)T;
  return status;
}

/* ------------------------------------------------------------- A7: combine */

/* out[t][n] = bf16_rn(res[t][n] + sum_j w[t][j] * y[pair_pos[t*k+j]][n]),
 * j in order; a pair with pair_pos < 0 contributes nothing. residual may be
 * NULL (BF16 bits otherwise). */
void eo_combine(const double *y, const double *w, const int32_t *pair_pos, const uint16_t *residual, int T, int k,
                int H, uint16_t *out) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t)
    for (int n = 0; n < H; ++n) {
      double acc = residual ? (double)bf16_to_f32(residual[(size_t)t * H + n]) : 0.0;
      for (int j = 0; j < k; ++j) {
        const int32_t r = pair_pos[(size_t)t * k + j];
        if (r < 0) continue;
        acc = acc + w[(size_t)t * k + j] * y[(size_t)r * H + n];
      }
      out[(size_t)t * H + n] = bf16_bits(round_bf16(acc));
    }
}

/* ------------------------------------------------------- the whole layer */

/* Per-token form: for each token, each chosen expert in j order, a
 * matrix-vector SwiGLU from freshly dequantised rows. ids [T][k], w [T][k]. */
int eo_layer_per_token(const uint16_t *x, const int32_t *ids, const double *w, int T, int k, const uint8_t *gq,
                       const uint16_t *gs, const uint8_t *uq, const uint16_t *us, const uint8_t *dq,
                       const uint16_t *ds, int E, int H, int I, const uint16_t *residual, uint16_t *out) {
  if (H % EO_GROUP || I % EO_GROUP) return -1;
  const eo_experts X = {gq, uq, dq, gs, us, ds, E, H, I};
  int status = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    double *xr = (double *)malloc(sizeof(double) * (size_t)H);
    double *hh = (double *)malloc(sizeof(double) * (size_t)I);
    double *yy = (double *)malloc(sizeof(double) * (size_t)H);
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);
    if (!xr || !hh || !yy || !acc) {
#pragma omp atomic write
      status = -2;
      free(xr); free(hh); free(yy); free(acc);
      continue;
    }
    for (int c = 0; c < H; ++c) {
      xr[c] = (double)bf16_to_f32(x[(size_t)t * H + c]);
      acc[c] = residual ? (double)bf16_to_f32(residual[(size_t)t * H + c]) : 0.0;
    }
    for (int j = 0; j < k; ++j) {
      const int e = ids[(size_t)t * k + j];
      if (e < 0 || e >= E || expert_rows(&X, e, xr, 1, hh, yy) != 0) {
#pragma omp atomic write
        status = -1;
        continue;
      }
      for (int c = 0; c < H; ++c) acc[c] = acc[c] + w[(size_t)t * k + j] * yy[c];
    }
    for (int c = 0; c < H; ++c) out[(size_t)t * H + c] = bf16_bits(round_bf16(acc[c]));
    free(xr);
    free(hh);
    free(yy);
    free(acc);
  }
  return status;
}

/* Router -> top-k -> grouping -> grouped FFN -> combine, all in this oracle.
 * logits [T][E] (BF16 bits), ids, w [T][k] are outputs too. residual: 1 adds
 * x to the output (the stack's x + MoE(x)). */
int eo_moe_layer(const uint16_t *x, const uint16_t *wr, int T, int H, int I, int E, int k, const float *bias,
                 int renorm, int residual, const uint8_t *gq, const uint16_t *gs, const uint8_t *uq,
                 const uint16_t *us, const uint8_t *dq, const uint16_t *ds, uint16_t *logits, int32_t *ids,
                 double *w, uint16_t *out) {
  const long P = (long)T * k;
  eo_router_logits(x, wr, T, H, E, logits);
  int st = eo_route_topk(logits, bias, T, E, k, renorm, ids, w);
  if (st) return st;
  int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
  int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
  int32_t *sp = (int32_t *)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1));
  int32_t *pp = (int32_t *)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1));
  double *h = (double *)malloc(sizeof(double) * (size_t)(P > 0 ? P : 1) * I);
  double *y = (double *)malloc(sizeof(double) * (size_t)(P > 0 ? P : 1) * H);
  if (!counts || !offsets || !sp || !pp || !h || !y) st = -2;
  if (!st) st = eo_group_tokens(ids, T, k, E, counts, offsets, sp, pp);
  if (!st) st = eo_grouped_ffn(x, T, sp, offsets, k, gq, gs, uq, us, dq, ds, E, H, I, h, y);
  if (!st) eo_combine(y, w, pp, residual ? x : NULL, T, k, H, out);
  free(counts);
  free(offsets);
  free(sp);
  free(pp);
  free(h);
  free(y);
  return st;
}

/* Threads for later OpenMP regions (0 or less: leave as is). */
void eo_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Threads an OpenMP region would use (for reporting). */
int eo_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
