/*
 * moe_oracle.c -- plain CPU oracle for one mixed-precision routed-expert layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's compute path may call,
 * link or load this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA implementation: the storage format is decoded here
 * from its written definition (include/moe.h documents the same format for the
 * library's users), and every floating-point step is done in IEEE binary64.
 *
 * What it computes, with the passage each step follows (page "Every Expert
 * Counts: ExactMoE for Memory-Efficient W4A16 Inference", arXiv 2608.15383):
 *
 *   router   z_t = W_r h_t, bf16 operands, binary64 sum          -- Section 3.1, routing equation
 *   route    S_t = TopK(z_t, k) over the router logits        -- Section 3.1, routing equation
 *            ties between equal logits go to the lower expert id (the top-k
 *            rule is "unchanged" and must be deterministic); the gating weights
 *            are a softmax over the k selected logits (Section 3.4 speaks of
 *            "router weights" and of Equation 2, which the page does not
 *            print; this is the renormalised top-k reading).
 *   permute  tokens grouped by selected expert (Figure 1 caption), experts in
 *            id order, tokens in ascending order inside each group, no token
 *            dropped (Abstract: "no expert is pruned").
 *   dequant  W = q * s with symmetric group-128 scales along K  -- Section 3.2
 *            ("dequantized values define the corresponding mathematical
 *            operations", Section 3.1).
 *   FFN      h = silu(x Wg^T) * (x Wu^T),  y = h Wd^T            -- Section 3.1
 *            names Wg, Wu, Wd; the SwiGLU form is the reading taken.
 *   combine  out_t = sum_j w_{t,j} y_{t,j}, weights not renormalised per wave
 *            -- Section 3.4.
 *   quantise s = max|W| / Q rounded to fp16, q = clip(round(W / s)) with Q = 7,
 *            range [-8, 7] for INT4 -- Section 3.2 equation; INT8 by analogy
 *            with Q = 127, range [-128, 127].
 *
 * Parity pins: every function here is pinned by tests under tests/ against
 * brute force, closed forms, invariants or library routines (numpy / torch).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_BF16 = 0, OR_INT8 = 1, OR_INT4 = 2 };
enum { OR_OK = 0, OR_ERR_ARG = -1, OR_ERR_NAN = -2, OR_ERR_NOMEM = -3 };

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bfloat16 is the upper half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_fp16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 31;
  int frac = h & 1023;
  double v;
  if (expo == 0)
    v = ldexp((double)frac, -24); /* subnormal: frac * 2^-24 */
  else if (expo == 31)
    v = frac ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + frac), expo - 25); /* (1 + frac/1024) 2^(e-15) */
  return sign ? -v : v;
}

/* Round a non-negative double that is an exact multiple of 2^-1 or finer to
 * the nearest integer, ties to even (IEEE roundTiesToEven). */
static double round_half_even(double v) {
  double fl = floor(v);
  double diff = v - fl;
  if (diff > 0.5) return fl + 1.0;
  if (diff < 0.5) return fl;
  return fmod(fl, 2.0) == 0.0 ? fl : fl + 1.0;
}

/* binary32 -> binary16, round to nearest, ties to even; overflow to inf. */
uint16_t oracle_fp16_from_float(float f) {
  double a = fabs((double)f);
  uint16_t sign = signbit(f) ? 0x8000 : 0;
  if (isnan(f)) return 0x7E00;
  if (a == 0.0) return sign;
  int ex;
  frexp(a, &ex); /* a = m * 2^ex, m in [0.5, 1) => unbiased exponent ex-1 */
  int e = ex - 1;
  if (e < -14) {
    /* subnormal grid: spacing 2^-24; m in [0, 1024] (1024 = smallest normal) */
    double m = round_half_even(ldexp(a, 24));
    return sign | (uint16_t)m; /* m == 1024 encodes exponent 1, fraction 0 */
  }
  double m = round_half_even(ldexp(a, 10 - e)); /* in [1024, 2048] */
  if (m == 2048.0) {
    m = 1024.0;
    e += 1;
  }
  if (e > 15) return sign | 0x7C00;
  return sign | (uint16_t)(((e + 15) << 10) | ((int)m - 1024));
}

/* ------------------------------------------------------------------------ */
/* Storage format (one weight matrix of `rows` x `K`, K contiguous)           */
/*   BF16: uint16 bf16 bits [rows][K]                                         */
/*   INT8: int8 two's complement [rows][K]                                    */
/*   INT4: uint8 [rows][K/2]; element k in byte k/2, even k in the low        */
/*         nibble, stored offset-binary u = q + 8                             */
/*   scales (INT8/INT4): fp16 [K/128][rows], group-major                      */
/* ------------------------------------------------------------------------ */

/* Integer code of element (row, k). */
static int code_at(int prec, const void* w, int K, int row, int k) {
  if (prec == OR_INT8) {
    return (int)((const int8_t*)w)[(size_t)row * K + k];
  }
  const uint8_t* p = (const uint8_t*)w;
  uint8_t byte = p[(size_t)row * (K / 2) + k / 2];
  int u = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
  return u - 8;
}

/* Dequantised row: out[k] = q * s (exact in binary64), or the bf16 value. */
static void load_row(int prec, const void* w, const uint16_t* s, int rows, int K,
                     int row, double* out) {
  if (prec == OR_BF16) {
    const uint16_t* b = (const uint16_t*)w + (size_t)row * K;
    for (int k = 0; k < K; ++k) out[k] = oracle_bf16_to_double(b[k]);
    return;
  }
  for (int k = 0; k < K; ++k) {
    double scale = oracle_fp16_to_double(s[(size_t)(k / 128) * rows + row]);
    out[k] = (double)code_at(prec, w, K, row, k) * scale;
  }
}

/* Public: dequantise a whole matrix into binary64 (tests use it on tiny sizes). */
int oracle_dequantize(int prec, const void* w, const uint16_t* s, int rows, int K,
                      double* out) {
  if (rows < 0 || K <= 0 || (prec != OR_BF16 && K % 128 != 0)) return OR_ERR_ARG;
  for (int r = 0; r < rows; ++r) load_row(prec, w, s, rows, K, r, out + (size_t)r * K);
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Quantiser (ExactMoE Section 3.2; INT8 by analogy)                         */
/* ------------------------------------------------------------------------ */

/* w: bf16 bits [rows][K]; writes the codes in the storage format above and
 * the fp16 scales [K/128][rows].  The scale is max|W| / Q computed in binary32
 * and rounded to fp16; the code uses the rounded scale:
 * q = clip(rint_even(W / s)), the quotient taken in binary32. */
int oracle_quantize(const uint16_t* w, int rows, int K, int prec, void* q_out,
                    uint16_t* s_out) {
  if (rows < 0 || K <= 0 || K % 128 != 0) return OR_ERR_ARG;
  if (prec != OR_INT8 && prec != OR_INT4) return OR_ERR_ARG;
  const int Q = (prec == OR_INT4) ? 7 : 127;
  const int qmin = -(Q + 1), qmax = Q;
  if (prec == OR_INT4) memset(q_out, 0, (size_t)rows * (K / 2));
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    for (int g = 0; g < K / 128; ++g) {
      float amax = 0.0f;
      for (int j = 0; j < 128; ++j) {
        float v = (float)oracle_bf16_to_double(w[(size_t)r * K + g * 128 + j]);
        if (fabsf(v) > amax) amax = fabsf(v);
      }
      float ratio = amax / (float)Q;
      uint16_t s16 = oracle_fp16_from_float(ratio);
      s_out[(size_t)g * rows + r] = s16;
      float s = (float)oracle_fp16_to_double(s16);
      for (int j = 0; j < 128; ++j) {
        int k = g * 128 + j;
        float v = (float)oracle_bf16_to_double(w[(size_t)r * K + k]);
        int q = 0;
        if (s != 0.0f) {
          float quot = v / s;
          double rq = (quot < 0) ? -round_half_even(-(double)quot)
                                 : round_half_even((double)quot);
          if (rq < qmin) rq = qmin;
          if (rq > qmax) rq = qmax;
          q = (int)rq;
        }
        if (prec == OR_INT8) {
          ((int8_t*)q_out)[(size_t)r * K + k] = (int8_t)q;
        } else {
          uint8_t* p = (uint8_t*)q_out + (size_t)r * (K / 2) + k / 2;
          uint8_t u = (uint8_t)(q + 8);
          *p |= (k % 2 == 0) ? u : (uint8_t)(u << 4);
        }
      }
    }
  }
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Routing (Section 3.1 routing equation)                                    */
/* ------------------------------------------------------------------------ */

/* Router projection z_t = W_r h_t (Section 3.1 routing equation; the router
 * stays in BF16, Abstract): h bf16 [T][H] (one hidden state per token), wr
 * bf16 [E][H] (row e = expert e's router row) -> z [T][E] in binary64.  Every
 * bf16 value and every product of two is exact in binary64; the products are
 * summed in ascending hidden index. */
int oracle_router_logits(const uint16_t* h, const uint16_t* wr, int T, int H, int E,
                         double* z) {
  if (T < 0 || H <= 0 || E <= 0) return OR_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c)
        acc += oracle_bf16_to_double(h[(size_t)t * H + c]) *
               oracle_bf16_to_double(wr[(size_t)e * H + c]);
      z[(size_t)t * E + e] = acc;
    }
  }
  return OR_OK;
}

/* logits fp32 [T][E]. Writes idx [T][k] (descending logit, ties -> lower id)
 * and weights [T][k] in binary64.  renormalize != 0: softmax over the k
 * selected logits; renormalize == 0: the full softmax over all E logits,
 * evaluated at the selected experts.  Logits must be finite. */
int oracle_route_topk(const float* logits, int T, int E, int k, int renormalize,
                      int32_t* idx, double* w) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return OR_ERR_ARG;
  char* chosen = (char*)malloc((size_t)E);
  if (!chosen) return OR_ERR_NOMEM;
  int rc = OR_OK;
  for (int t = 0; t < T && rc == OR_OK; ++t) {
    const float* z = logits + (size_t)t * E;
    for (int e = 0; e < E; ++e) {
      if (!isfinite(z[e])) rc = OR_ERR_NAN;
      chosen[e] = 0;
    }
    if (rc != OR_OK) break;
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (chosen[e]) continue;
        if (best < 0 || z[e] > z[best]) best = e; /* equal: keep lower id */
      }
      chosen[best] = 1;
      idx[(size_t)t * k + j] = best;
    }
    double m, den = 0.0;
    if (renormalize) {
      m = (double)z[idx[(size_t)t * k]];
      for (int j = 0; j < k; ++j) den += exp((double)z[idx[(size_t)t * k + j]] - m);
    } else {
      m = (double)z[0];
      for (int e = 1; e < E; ++e)
        if ((double)z[e] > m) m = (double)z[e];
      for (int e = 0; e < E; ++e) den += exp((double)z[e] - m);
    }
    for (int j = 0; j < k; ++j)
      w[(size_t)t * k + j] = exp((double)z[idx[(size_t)t * k + j]] - m) / den;
  }
  free(chosen);
  return rc;
}

/* ------------------------------------------------------------------------ */
/* Permutation (Figure 1: tokens grouped by selected expert)                 */
/* ------------------------------------------------------------------------ */

/* A pair is invalid when its id lies outside [0, E) or repeats an id of an
 * earlier slot of the same token (a top-k set has distinct members). */
static int pair_invalid(const int32_t* idx, int E, int k, int t, int j) {
  int e = idx[(size_t)t * k + j];
  if (e < 0 || e >= E) return 1;
  for (int jj = 0; jj < j; ++jj)
    if (idx[(size_t)t * k + jj] == e) return 1;
  return 0;
}

/* Counting sort of the (token, slot) pairs by expert, stable by token.
 * offsets [E+1], perm_token [rows] (row -> token), dest_row [T*k]
 * (pair -> row, -1 for an invalid pair).
 * Returns the number of invalid pairs (0 for valid input). */
int oracle_permute(const int32_t* idx, int T, int E, int k, int32_t* offsets,
                   int32_t* perm_token, int32_t* dest_row) {
  if (T < 0 || E <= 0 || k <= 0) return OR_ERR_ARG;
  int32_t* cursor = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  if (!cursor) return OR_ERR_NOMEM;
  int invalid = 0;
  for (int e = 0; e <= E; ++e) offsets[e] = 0;
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j)
      if (!pair_invalid(idx, E, k, t, j)) offsets[idx[(size_t)t * k + j] + 1] += 1;
  for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
  for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      size_t p = (size_t)t * k + j;
      int e = idx[p];
      if (pair_invalid(idx, E, k, t, j)) {
        dest_row[p] = -1;
        invalid += 1;
        continue;
      }
      int row = cursor[e]++;
      dest_row[p] = row;
      perm_token[row] = t;
    }
  }
  free(cursor);
  return invalid;
}

/* ------------------------------------------------------------------------ */
/* Expert FFN (Section 3.1 names Wg, Wu, Wd; SwiGLU reading)                 */
/* ------------------------------------------------------------------------ */

typedef struct {
  int prec;
  const void* w13;     /* [2I][H]: rows 0..I-1 gate, I..2I-1 up */
  const uint16_t* s13; /* [H/128][2I] */
  const void* w2;      /* [H][I] */
  const uint16_t* s2;  /* [I/128][H] */
} oracle_expert;

/* y[H] = Wd (silu(Wg x) * (Wu x)); scratch must hold max(H, I) + I doubles. */
static void expert_ffn(const oracle_expert* ex, const double* x, int H, int I,
                       double* scratch, double* y) {
  double* row = scratch;          /* max(H, I) */
  double* h = scratch + (H > I ? H : I);
  for (int n = 0; n < I; ++n) {
    double g = 0.0, u = 0.0;
    load_row(ex->prec, ex->w13, ex->s13, 2 * I, H, n, row);
    for (int c = 0; c < H; ++c) g += x[c] * row[c];
    load_row(ex->prec, ex->w13, ex->s13, 2 * I, H, I + n, row);
    for (int c = 0; c < H; ++c) u += x[c] * row[c];
    h[n] = g / (1.0 + exp(-g)) * u;
  }
  for (int m = 0; m < H; ++m) {
    double acc = 0.0;
    load_row(ex->prec, ex->w2, ex->s2, H, I, m, row);
    for (int n = 0; n < I; ++n) acc += h[n] * row[n];
    y[m] = acc;
  }
}

static int check_shapes(int H, int I, int E) {
  return (H > 0 && I > 0 && E > 0 && H % 128 == 0 && I % 128 == 0);
}

/* Grouped FFN over permuted rows: for every row r of expert e
 * (offsets[e] <= r < offsets[e+1]), y_perm[r] = FFN_e(x_perm[r]).
 * x_perm bf16 bits [rows][H]; y_perm binary64 [rows][H].  `rows_sel`
 * (length n_sel) restricts the computation to those rows (NULL: all rows). */
int oracle_grouped_ffn(const uint16_t* x_perm, const int32_t* offsets, int H, int I,
                       int E, const int* prec, const void* const* w13,
                       const uint16_t* const* s13, const void* const* w2,
                       const uint16_t* const* s2, const int32_t* rows_sel,
                       int n_sel, double* y_perm) {
  if (!check_shapes(H, I, E)) return OR_ERR_ARG;
  int nrows = offsets[E];
  int n = rows_sel ? n_sel : nrows;
  int rc = OR_OK;
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)H);
    double* scratch = (double*)malloc(sizeof(double) * (size_t)((H > I ? H : I) + I));
    if (!x || !scratch) {
#pragma omp atomic write
      rc = OR_ERR_NOMEM;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int i = 0; i < n; ++i) {
        int r = rows_sel ? rows_sel[i] : i;
        int e = 0;
        while (e < E && !(offsets[e] <= r && r < offsets[e + 1])) ++e;
        if (e == E) continue;
        oracle_expert ex = {prec[e], w13[e], s13[e], w2[e], s2[e]};
        for (int c = 0; c < H; ++c)
          x[c] = oracle_bf16_to_double(x_perm[(size_t)r * H + c]);
        expert_ffn(&ex, x, H, I, scratch, y_perm + (size_t)i * H);
      }
    }
    free(x);
    free(scratch);
  }
  return rc;
}

/* ------------------------------------------------------------------------ */
/* Combine (Section 3.4: router weights kept, wave outputs summed)           */
/* ------------------------------------------------------------------------ */

/* out[t] = sum_j w[t][j] * y_perm[dest_row[t][j]], pairs with dest_row < 0
 * skipped.  y_perm binary64 [rows][H]; out binary64 [T][H]. */
int oracle_combine(const double* y_perm, const int32_t* dest_row, const double* w,
                   int T, int k, int H, double* out) {
  if (T < 0 || k <= 0 || H <= 0) return OR_ERR_ARG;
  for (int t = 0; t < T; ++t) {
    double* o = out + (size_t)t * H;
    for (int c = 0; c < H; ++c) o[c] = 0.0;
    for (int j = 0; j < k; ++j) {
      int r = dest_row[(size_t)t * k + j];
      if (r < 0) continue;
      double wj = w[(size_t)t * k + j];
      for (int c = 0; c < H; ++c) o[c] += wj * y_perm[(size_t)r * H + c];
    }
  }
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Whole layer for a chosen set of tokens                                    */
/* ------------------------------------------------------------------------ */

/* Routes every token, then evaluates out[t] = sum_j w_{t,j} FFN_{S_j}(x_t) for
 * the n_tok tokens listed in `tokens` (NULL: all T).  out binary64
 * [n_tok][H].  idx/w receive the routing of all T tokens. */
int oracle_moe_layer(const float* logits, const uint16_t* x, int T, int H, int I,
                     int E, int k, int renormalize, const int* prec,
                     const void* const* w13, const uint16_t* const* s13,
                     const void* const* w2, const uint16_t* const* s2,
                     const int32_t* tokens, int n_tok, int32_t* idx, double* w,
                     double* out) {
  if (!check_shapes(H, I, E)) return OR_ERR_ARG;
  int rc = oracle_route_topk(logits, T, E, k, renormalize, idx, w);
  if (rc != OR_OK) return rc;
  int n = tokens ? n_tok : T;
#pragma omp parallel
  {
    double* xt = (double*)malloc(sizeof(double) * (size_t)H);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    double* scratch = (double*)malloc(sizeof(double) * (size_t)((H > I ? H : I) + I));
    if (!xt || !y || !scratch) {
#pragma omp atomic write
      rc = OR_ERR_NOMEM;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int i = 0; i < n; ++i) {
        int t = tokens ? tokens[i] : i;
        double* o = out + (size_t)i * H;
        for (int c = 0; c < H; ++c) {
          xt[c] = oracle_bf16_to_double(x[(size_t)t * H + c]);
          o[c] = 0.0;
        }
        for (int j = 0; j < k; ++j) {
          int e = idx[(size_t)t * k + j];
          oracle_expert ex = {prec[e], w13[e], s13[e], w2[e], s2[e]};
          expert_ffn(&ex, xt, H, I, scratch, y);
          double wj = w[(size_t)t * k + j];
          for (int c = 0; c < H; ++c) o[c] += wj * y[c];
        }
      }
    }
    free(xt);
    free(y);
    free(scratch);
  }
  return rc;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads of the later parallel regions (n >= 1).  The work is split over
 * (expert, row) and (token) only, so no result depends on it. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
