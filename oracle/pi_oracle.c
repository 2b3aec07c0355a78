/*
 * pi_oracle.c -- plain CPU oracle for the predictor-gated, neuron-level sparse
 * FFN block of activation-sparse LLM decoding (PowerInfer).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library in
 * activation_sparse_decode_gemv_b200/ never calls it, and this file shares no
 * code, header, table or helper with that library.
 *
 * What it computes, and where the pages say so ("PowerInfer: Fast Large
 * Language Model Serving with a Consumer-grade GPU", Elamur Research summary,
 * and the reboot-conseil overview):
 *   - per-layer predictor: a small model scores every FFN neuron and guesses
 *     which ones fire (Summary, second paragraph; Key points, Accuracy).  Here
 *     the predictor is the rank-r factorised scorer s = P2 (P1 u) + bias, and
 *     neuron i fires iff s_i > 0.
 *   - neuron-aware sparse operator: only the rows of the active neurons are
 *     read and combined, and the inactive ones are never touched (Summary,
 *     second paragraph; Interesting ideas I4: kernels index the weight rows
 *     and columns of the neurons themselves, with no sparse format).
 *     The result is exactly the dense FFN sum restricted to the chosen set:
 *         y_b = sum_{i in S_b} phi_i(u_b) * W2T_i
 *     with phi = ReLU(W1_i . u + b1_i) (OPT, Key points: ReLU) or
 *     phi = SiLU(Wg_i . u) * (Wu_i . u) (LLaMA2 / SwiGLU, Key points).
 *   - quantized models (Summary: 4-bit models; Key points: Speed): int4
 *     weights in 32-element groups with an fp16 scale, value = scale*(q-8).
 *
 * Arithmetic: every sum is accumulated in IEEE double, in the plain index
 * order of its definition, with no blocking or reordering.  fp16 inputs are
 * decoded exactly to double by this file's own binary16 decoder.  The only
 * steps done in binary32 are the two where floating point decides a stored
 * code of the CUDA path: the fp16 code of the RMS-normalised FFN input of a
 * stacked layer, and the fp32 residual stream, whose storage type is fixed by
 * the interface (the residual x is a float buffer).
 *
 * Parity pins: see tests/test_oracle_pins.py.  SiLU (exp from libm) is
 * pinned by its symmetry identities and limits, and its value against an
 * arbitrary-precision evaluation of z / (1 + e^-z) to 4 units in the last
 * place.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_EINVAL 1

enum { OR_F32 = 0, OR_F16 = 1, OR_INT4G32 = 2 };
enum { OR_RELU = 0, OR_SWIGLU = 1 };

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16 <-> double, written from the format's definition.      */
/* ------------------------------------------------------------------------ */

double or_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* round-half-to-even of a non-negative double to an integer-valued double */
static double rne(double q) {
  double r = floor(q);
  double frac = q - r;
  if (frac > 0.5) return r + 1.0;
  if (frac < 0.5) return r;
  return (fmod(r, 2.0) == 0.0) ? r : r + 1.0;
}

/* nearest binary16 to the binary32 value x, ties to even (IEEE default) */
uint16_t or_float_to_half(float xf) {
  double x = (double)xf;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  if (isnan(x)) return 0x7e00;
  double ax = fabs(x);
  if (ax == 0.0) return sign;
  if (isinf(ax)) return (uint16_t)(sign | 0x7c00);
  if (ax < ldexp(1.0, -14)) {
    /* subnormal range: multiples of 2^-24; 1024 * 2^-24 is the smallest normal */
    double m = rne(ax * ldexp(1.0, 24));
    return (uint16_t)(sign | (uint16_t)m);
  }
  int ex;
  frexp(ax, &ex); /* ax = fr * 2^ex, fr in [0.5, 1) */
  int E = ex - 1; /* ax in [2^E, 2^(E+1)) */
  double m = rne(ax * ldexp(1.0, 10 - E)); /* in [1024, 2048] */
  if (m == 2048.0) {
    m = 1024.0;
    E += 1;
  }
  if (E + 15 >= 31) return (uint16_t)(sign | 0x7c00); /* overflow to inf */
  return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(m - 1024.0));
}

/* ------------------------------------------------------------------------ */
/* element access                                                           */
/* ------------------------------------------------------------------------ */

/* one element of an [rows x d] weight matrix of the given storage type.
 * int4g32: row-major packed nibbles, d/2 bytes per row, element 2k in the low
 * nibble of byte k and 2k+1 in the high nibble; scales fp16 [rows x d/32];
 * value = scale * (q - 8). */
static double w_elem(const void *w, const uint16_t *sc, int wtype, int d, long row, int col) {
  switch (wtype) {
  case OR_F32:
    return (double)((const float *)w)[row * (long)d + col];
  case OR_F16:
    return or_half_to_double(((const uint16_t *)w)[row * (long)d + col]);
  case OR_INT4G32: {
    uint8_t byte = ((const uint8_t *)w)[row * (long)(d / 2) + col / 2];
    int q = (col & 1) ? (byte >> 4) : (byte & 15);
    double s = or_half_to_double(sc[row * (long)(d / 32) + col / 32]);
    return s * (double)(q - 8);
  }
  }
  return NAN;
}

/* one element of the FFN input u [B x d]: fp32 or fp16 */
static double u_elem(const void *u, int utype, int d, int b, int k) {
  if (utype == OR_F32) return (double)((const float *)u)[(long)b * d + k];
  return or_half_to_double(((const uint16_t *)u)[(long)b * d + k]);
}

/* decode a whole weight row into double (used by the int4 dequant pin) */
int or_dequant_row(int wtype, int d, const void *w, const uint16_t *sc, long row, double *out) {
  if (d <= 0 || (wtype == OR_INT4G32 && d % 32)) return OR_EINVAL;
  for (int k = 0; k < d; ++k) out[k] = w_elem(w, sc, wtype, d, row, k);
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* predictor: h = P1 u, s = P2 h + bias, fires iff s > 0                    */
/* ------------------------------------------------------------------------ */

/* Inputs: P1 [r x d], P2 [f x r] of type ptype (fp32/fp16), bias [f] fp32,
 * u [B x d] of type utype.  Outputs (any may be NULL except idx/count):
 * h [B x r], s [B x f], band [B x f] (the rounding band inside which an fp32
 * evaluation may land on either side of 0; see below), idx [B x f] ascending
 * active neuron ids of token b in row b, count [B].
 *
 * Band: an fp32 evaluation of s differs from this double one by rounding.
 * The band is 16 * 2^-24 * (sqrt(r) sum_j |P2_ij h_j|
 *                           + sqrt(d) sqrt(sum_j (P2_ij a_j)^2)
 *                           + |bias_i|),   a_j = sum_k |P1_jk u_k|,
 * a probabilistic rounding-error bound in the style of Higham & Mary
 * (SIAM J. Sci. Comput. 41(5), 2019) with a safety factor of 16: the error
 * of a length-n fp32 sum is at most ~sqrt(n) 2^-24 times the sum of the
 * absolute terms, and the independent errors of the r stage-1 sums h_j reach
 * s_i through the weights P2_ij, so they combine in quadrature.  Neurons
 * with |s_i| <= band_i may be classified either way by an fp32 evaluation. */
int or_predict(int d, int f, int r, int ptype, const void *p1, const void *p2, const float *bias,
               int utype, const void *u, int B, double *h_out, double *s_out, double *band_out,
               int32_t *idx, int32_t *count) {
  if (d <= 0 || f <= 0 || r <= 0 || B <= 0 || !p1 || !p2 || !bias || !u || !idx || !count)
    return OR_EINVAL;
  if (ptype != OR_F32 && ptype != OR_F16) return OR_EINVAL;
  double *h = (double *)malloc(sizeof(double) * r);
  double *habs = (double *)malloc(sizeof(double) * r);
  if (!h || !habs) {
    free(h);
    free(habs);
    return OR_EINVAL;
  }
  for (int b = 0; b < B; ++b) {
    for (int j = 0; j < r; ++j) {
      double acc = 0.0, aabs = 0.0;
      for (int k = 0; k < d; ++k) {
        double t = w_elem(p1, NULL, ptype, d, j, k) * u_elem(u, utype, d, b, k);
        acc += t;
        aabs += fabs(t);
      }
      h[j] = acc;
      habs[j] = aabs;
      if (h_out) h_out[(long)b * r + j] = acc;
    }
    int n = 0;
    for (int i = 0; i < f; ++i) {
      double acc = 0.0, t1 = 0.0, t2 = 0.0;
      for (int j = 0; j < r; ++j) {
        double p = w_elem(p2, NULL, ptype, r, i, j);
        acc += p * h[j];
        t1 += fabs(p * h[j]);
        t2 += (p * habs[j]) * (p * habs[j]);
      }
      double s = acc + (double)bias[i];
      if (s_out) s_out[(long)b * f + i] = s;
      if (band_out)
        band_out[(long)b * f + i] =
            16.0 * ldexp(1.0, -24) * (sqrt((double)r) * t1 + sqrt((double)d) * sqrt(t2) + fabs((double)bias[i]));
      if (s > 0.0) idx[(long)b * f + n++] = i;
    }
    count[b] = n;
  }
  free(h);
  free(habs);
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* neuron activation phi_i(u_b) and the FFN sums                            */
/* ------------------------------------------------------------------------ */

typedef struct {
  int d, f, act, wtype, utype;
  const void *w_up, *w_gate, *w_down_t;
  const uint16_t *s_up, *s_gate, *s_down_t;
  const float *b_up; /* ReLU bias b1 [f]; ignored for SwiGLU */
} or_ffn;

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* phi_i(u_b): ReLU(W1_i . u + b1_i) or SiLU(Wg_i . u) * (Wu_i . u) */
static double neuron_phi(const or_ffn *L, const void *u, int b, long i) {
  int d = L->d;
  if (L->act == OR_RELU) {
    double pre = 0.0;
    for (int k = 0; k < d; ++k) pre += w_elem(L->w_up, L->s_up, L->wtype, d, i, k) * u_elem(u, L->utype, d, b, k);
    pre += (double)L->b_up[i];
    return pre > 0.0 ? pre : 0.0;
  }
  double g = 0.0, v = 0.0;
  for (int k = 0; k < d; ++k) {
    double uk = u_elem(u, L->utype, d, b, k);
    g += w_elem(L->w_gate, L->s_gate, L->wtype, d, i, k) * uk;
    v += w_elem(L->w_up, L->s_up, L->wtype, d, i, k) * uk;
  }
  return silu(g) * v;
}

static int ffn_check(const or_ffn *L) {
  if (L->d <= 0 || L->f <= 0 || !L->w_up || !L->w_down_t) return 0;
  if (L->act != OR_RELU && L->act != OR_SWIGLU) return 0;
  if (L->act == OR_RELU && !L->b_up) return 0;
  if (L->act == OR_SWIGLU && !L->w_gate) return 0;
  if (L->wtype == OR_INT4G32) {
    if (L->d % 32) return 0;
    if (!L->s_up || !L->s_down_t || (L->act == OR_SWIGLU && !L->s_gate)) return 0;
  } else if (L->wtype != OR_F32 && L->wtype != OR_F16) {
    return 0;
  }
  return 1;
}

/* all phi [B x f] (dense, for diagnostics and the exact-ReLU-mask pin) */
int or_neuron_phi(const or_ffn *L, const void *u, int B, double *phi) {
  if (!ffn_check(L) || !u || B <= 0 || !phi) return OR_EINVAL;
  for (int b = 0; b < B; ++b)
    for (long i = 0; i < L->f; ++i) phi[(long)b * L->f + i] = neuron_phi(L, u, b, i);
  return OR_OK;
}

/* ReLU pre-activation W1_i . u + b1_i [B x f] (defines the exact mask) */
int or_relu_preact(const or_ffn *L, const void *u, int B, double *pre) {
  if (!ffn_check(L) || L->act != OR_RELU || !u || B <= 0 || !pre) return OR_EINVAL;
  int d = L->d;
  for (int b = 0; b < B; ++b)
    for (long i = 0; i < L->f; ++i) {
      double acc = 0.0;
      for (int k = 0; k < d; ++k) acc += w_elem(L->w_up, L->s_up, L->wtype, d, i, k) * u_elem(u, L->utype, d, b, k);
      pre[(long)b * L->f + i] = acc + (double)L->b_up[i];
    }
  return OR_OK;
}

/* Masked sparse FFN: y_b = sum over n < count[b] of phi_{idx[b][n]}(u_b) W2T_{idx[b][n]},
 * idx row b at idx + b*idx_stride, strictly ascending ids in [0, f).
 * Returns OR_EINVAL for an out-of-range, repeated or unsorted id. */
int or_ffn_masked(const or_ffn *L, const void *u, int B, const int32_t *idx, const int32_t *count,
                  long idx_stride, double *y) {
  if (!ffn_check(L) || !u || B <= 0 || !idx || !count || !y) return OR_EINVAL;
  int d = L->d;
  for (int b = 0; b < B; ++b) {
    double *yb = y + (long)b * d;
    for (int k = 0; k < d; ++k) yb[k] = 0.0;
    if (count[b] < 0 || count[b] > L->f) return OR_EINVAL;
    int32_t prev = -1;
    for (int n = 0; n < count[b]; ++n) {
      int32_t i = idx[(long)b * idx_stride + n];
      if (i <= prev || i >= L->f) return OR_EINVAL;
      prev = i;
      double phi = neuron_phi(L, u, b, i);
      for (int k = 0; k < d; ++k) yb[k] += phi * w_elem(L->w_down_t, L->s_down_t, L->wtype, d, i, k);
    }
  }
  return OR_OK;
}

/* Dense FFN: the same sum over every neuron i = 0 .. f-1. */
int or_ffn_dense(const or_ffn *L, const void *u, int B, double *y) {
  if (!ffn_check(L) || !u || B <= 0 || !y) return OR_EINVAL;
  int d = L->d;
  for (int b = 0; b < B; ++b) {
    double *yb = y + (long)b * d;
    for (int k = 0; k < d; ++k) yb[k] = 0.0;
    for (long i = 0; i < L->f; ++i) {
      double phi = neuron_phi(L, u, b, i);
      for (int k = 0; k < d; ++k) yb[k] += phi * w_elem(L->w_down_t, L->s_down_t, L->wtype, d, i, k);
    }
  }
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* stacked layers                                                           */
/* ------------------------------------------------------------------------ */

/* Pre-FFN normalisation of a stacked layer's input (the pages name none; the
 * parameter-free RMS norm is this build's reading, without which the
 * residual stream of a deep stack diverges):
 *     u_k = fp16( x_k / sqrt(mean_k(x_k^2) + 1e-6) ).
 * The fp16 code is a stored decision of the CUDA path, so it is taken in the
 * same binary32 steps: the mean of squares is summed in double and rounded
 * once to float, then sqrt, divide and the fp16 rounding are single IEEE
 * binary32 operations.  Also returns, per token, the smallest relative
 * distance of a quotient to an fp16 rounding midpoint (decision margin). */
int or_rmsnorm_f16(int d, int B, const float *x, uint16_t *u, double *margin) {
  if (d <= 0 || B <= 0 || !x || !u) return OR_EINVAL;
  for (int b = 0; b < B; ++b) {
    const float *xb = x + (long)b * d;
    double ss = 0.0;
    for (int k = 0; k < d; ++k) ss += (double)xb[k] * (double)xb[k];
    float mean = (float)(ss / (double)d);
    volatile float t = mean + 1e-6f; /* volatile: one binary32 rounding per step */
    volatile float den = sqrtf(t);
    double mmin = INFINITY;
    for (int k = 0; k < d; ++k) {
      volatile float q = xb[k] / den;
      u[(long)b * d + k] = or_float_to_half(q);
      /* distance from q to the nearest fp16 midpoint, relative to |q| */
      double aq = fabs((double)q);
      if (aq > 0.0 && aq < 65504.0) {
        int ex;
        frexp(aq, &ex);
        int E = ex - 1;
        if (E < -14) E = -14;
        double ulp = ldexp(1.0, E - 10);
        double pos = aq / ulp; /* midpoints sit at integer + 0.5 */
        double dist = fabs(pos - floor(pos) - 0.5) * ulp / aq;
        if (dist < mmin) mmin = dist;
      }
    }
    if (margin) margin[b] = mmin;
  }
  return OR_OK;
}

/* One stacked layer: FFN block plus its predictor. */
typedef struct {
  or_ffn ffn;
  int rank, ptype;
  const void *p1, *p2;
  const float *p_bias;
} or_layer;

/* Stack of L layers: for each layer l, u = rmsnorm(x) (fp16), S = predicted
 * set of u, y = masked FFN over S (double), x = float(x + y).  x [B x d] is
 * float in/out.  Optional outputs: idx_trace [L x B x f], count_trace [L x B],
 * y_trace [L x B x d], s_margin [L x B] = min_i (|s_i| - band_i), u_margin
 * [L x B] = smallest relative distance of an fp16 decision to a midpoint. */
int or_stack(const or_layer *layers, int L, float *x, int B, int32_t *idx_trace, int32_t *count_trace,
             double *y_trace, double *s_margin, double *u_margin) {
  if (!layers || L <= 0 || !x || B <= 0) return OR_EINVAL;
  int d = layers[0].ffn.d;
  for (int l = 0; l < L; ++l) {
    const or_layer *ly = &layers[l];
    if (ly->ffn.d != d || ly->ffn.utype != OR_F16) return OR_EINVAL;
    int f = ly->ffn.f;
    uint16_t *u = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)B * d);
    double *s = (double *)malloc(sizeof(double) * (size_t)B * f);
    double *band = (double *)malloc(sizeof(double) * (size_t)B * f);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)B * f);
    int32_t *cnt = (int32_t *)malloc(sizeof(int32_t) * (size_t)B);
    double *y = (double *)malloc(sizeof(double) * (size_t)B * d);
    double *um = (double *)malloc(sizeof(double) * (size_t)B);
    int rc = (u && s && band && idx && cnt && y && um) ? OR_OK : OR_EINVAL;
    if (rc == OR_OK) rc = or_rmsnorm_f16(d, B, x, u, um);
    if (rc == OR_OK)
      rc = or_predict(d, f, ly->rank, ly->ptype, ly->p1, ly->p2, ly->p_bias, OR_F16, u, B, NULL, s, band, idx, cnt);
    if (rc == OR_OK) rc = or_ffn_masked(&ly->ffn, u, B, idx, cnt, f, y);
    if (rc == OR_OK) {
      for (int b = 0; b < B; ++b) {
        for (int k = 0; k < d; ++k) x[(long)b * d + k] = (float)((double)x[(long)b * d + k] + y[(long)b * d + k]);
        if (count_trace) count_trace[(long)l * B + b] = cnt[b];
        if (idx_trace) memcpy(idx_trace + ((long)l * B + b) * f, idx + (long)b * f, sizeof(int32_t) * f);
        if (y_trace) memcpy(y_trace + ((long)l * B + b) * d, y + (long)b * d, sizeof(double) * d);
        if (s_margin) {
          double m = INFINITY;
          for (int i = 0; i < f; ++i) {
            double g = fabs(s[(long)b * f + i]) - band[(long)b * f + i];
            if (g < m) m = g;
          }
          s_margin[(long)l * B + b] = m;
        }
        if (u_margin) u_margin[(long)l * B + b] = um[b];
      }
    }
    free(u);
    free(s);
    free(band);
    free(idx);
    free(cnt);
    free(y);
    free(um);
    if (rc != OR_OK) return rc;
  }
  return OR_OK;
}
