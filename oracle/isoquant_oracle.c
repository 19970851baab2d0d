/*
 * isoquant_oracle.c -- plain, slow, fp64 CPU oracle for IsoQuant
 * compressed-space attention.  TEST INFRASTRUCTURE ONLY (see the header):
 * nothing on the product path includes, links or calls this file.
 *
 * Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via
 * Fused Compressed-Space Attention", Abstract (Walsh-Hadamard transform,
 * then block-diagonal SO(4) rotations, then 3-bit scalar quantization;
 * attention directly on the packed 3-bit tensors).  Every reading the pages
 * leave open is listed in isoquant_oracle.h.
 *
 * Every step is written the plain way: the Hadamard transform is the
 * explicit O(d^2) sum with the Sylvester matrix entries, the SO(4) blocks
 * are explicit quaternion products, softmax is max-subtracted fp64.
 */
#include "isoquant_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- codebook */

static double std_pdf(double z) { return exp(-0.5 * z * z) / sqrt(2.0 * M_PI); }
static double std_cdf(double z) { return 0.5 * erfc(-z / sqrt(2.0)); }

/* Lloyd's two optimality conditions for a minimum-MSE scalar quantizer of
 * N(0,1): each threshold is the midpoint of its two neighbouring levels, and
 * each level is the conditional mean of its cell,
 *   c_i = (pdf(t_{i-1}) - pdf(t_i)) / (cdf(t_i) - cdf(t_{i-1})).
 * Iterated from uniformly spaced levels until the levels stop moving. */
int orc_lloyd_max_gauss(int nlev, double *levels, double *thresholds,
                        double *distortion) {
  if (nlev < 2 || nlev > 64) return -1;
  for (int i = 0; i < nlev; ++i)
    levels[i] = -2.0 + 4.0 * (i + 0.5) / nlev;
  int it;
  for (it = 1; it <= 200000; ++it) {
    for (int k = 0; k < nlev - 1; ++k)
      thresholds[k] = 0.5 * (levels[k] + levels[k + 1]);
    double change = 0.0;
    for (int i = 0; i < nlev; ++i) {
      double lo_pdf = (i == 0) ? 0.0 : std_pdf(thresholds[i - 1]);
      double hi_pdf = (i == nlev - 1) ? 0.0 : std_pdf(thresholds[i]);
      double lo_cdf = (i == 0) ? 0.0 : std_cdf(thresholds[i - 1]);
      double hi_cdf = (i == nlev - 1) ? 1.0 : std_cdf(thresholds[i]);
      double c = (lo_pdf - hi_pdf) / (hi_cdf - lo_cdf);
      double dc = fabs(c - levels[i]);
      if (dc > change) change = dc;
      levels[i] = c;
    }
    if (change < 1e-15) break;
  }
  for (int k = 0; k < nlev - 1; ++k)
    thresholds[k] = 0.5 * (levels[k] + levels[k + 1]);
  if (distortion) *distortion = orc_gauss_distortion(nlev, levels, thresholds);
  return it > 200000 ? -1 : it;
}

/* E[(Z - Q(Z))^2] for Z ~ N(0,1), cell by cell, using
 *   int_a^b z^2 pdf = cdf(b)-cdf(a) + a pdf(a) - b pdf(b),
 *   int_a^b z pdf   = pdf(a) - pdf(b). */
double orc_gauss_distortion(int nlev, const double *levels,
                            const double *thresholds) {
  double total = 0.0;
  for (int i = 0; i < nlev; ++i) {
    double a_pdf, b_pdf, a_cdf, b_cdf, a_z_pdf, b_z_pdf;
    if (i == 0) { a_pdf = 0; a_cdf = 0; a_z_pdf = 0; }
    else {
      double a = thresholds[i - 1];
      a_pdf = std_pdf(a); a_cdf = std_cdf(a); a_z_pdf = a * a_pdf;
    }
    if (i == nlev - 1) { b_pdf = 0; b_cdf = 1; b_z_pdf = 0; }
    else {
      double b = thresholds[i];
      b_pdf = std_pdf(b); b_cdf = std_cdf(b); b_z_pdf = b * b_pdf;
    }
    double m0 = b_cdf - a_cdf;
    double m1 = a_pdf - b_pdf;
    double m2 = m0 + a_z_pdf - b_z_pdf;
    double c = levels[i];
    total += m2 - 2.0 * c * m1 + c * c * m0;
  }
  return total;
}

/* Round to the nearest fp16 value, ties to even, by scaling to the fp16
 * quantum of the target binade (exact in fp64) and rounding to an integer. */
uint16_t orc_f64_to_f16(double x, int *saturated) {
  if (isnan(x)) return 0x7E00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a >= 65520.0) {            /* would round to infinity: saturate */
    if (saturated) *saturated = 1;
    return sign | 0x7BFF;
  }
  double quantum;
  if (a < ldexp(1.0, -14)) {
    quantum = ldexp(1.0, -24);   /* subnormal spacing */
  } else {
    int e;
    frexp(a, &e);                /* a = m 2^e, m in [0.5, 1) */
    quantum = ldexp(1.0, (e - 1) - 10);
  }
  double k = nearbyint(a / quantum);  /* default rounding mode: to even */
  double v = k * quantum;
  if (v < ldexp(1.0, -14)) return sign | (uint16_t)k;  /* subnormal / zero */
  int e;
  double m = frexp(v, &e);       /* v = m 2^e, m in [0.5,1) */
  int exp_field = (e - 1) + 15;
  uint16_t mant = (uint16_t)((m * 2.0 - 1.0) * 1024.0);
  return sign | (uint16_t)(exp_field << 10) | mant;
}

double orc_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp(1.0 + m / 1024.0, e - 15);
  return sign ? -v : v;
}

int orc_format(int bits, int *levels, int *per_word, int *words) {
  if (bits < 2 || bits > 4) return -1;
  const int cpw = 32 / bits;
  if (levels) *levels = 1 << bits;
  if (per_word) *per_word = cpw;
  if (words) *words = (ORC_D + cpw - 1) / cpw;
  return 0;
}

void orc_codebook_b(int bits, double *levels16, double *thresholds) {
  int nlev = 0;
  orc_format(bits, &nlev, NULL, NULL);
  double lv[ORC_MAX_LEVELS], th[ORC_MAX_LEVELS - 1], dist;
  orc_lloyd_max_gauss(nlev, lv, th, &dist);
  for (int i = 0; i < nlev; ++i)
    levels16[i] = orc_f16_to_f64(orc_f64_to_f16(lv[i], NULL));
  for (int k = 0; k < nlev - 1; ++k)
    thresholds[k] = 0.5 * (levels16[k] + levels16[k + 1]);
}

void orc_codebook(double levels16[ORC_LEVELS], double thresholds[ORC_LEVELS - 1]) {
  orc_codebook_b(3, levels16, thresholds);
}

/* ---------------------------------------------------------------- rotation */

void orc_qmul(const double a[4], const double b[4], double out[4]) {
  double w = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
  double x = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
  double y = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
  double z = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
  out[0] = w; out[1] = x; out[2] = y; out[3] = z;
}

static void qconj(const double a[4], double out[4]) {
  out[0] = a[0]; out[1] = -a[1]; out[2] = -a[2]; out[3] = -a[3];
}

void orc_normalise_quats(const float *raw, double *unit) {
  for (int k = 0; k < ORC_BLOCKS * 2; ++k) {
    double s = 0.0;
    for (int c = 0; c < 4; ++c) s += (double)raw[4 * k + c] * (double)raw[4 * k + c];
    double inv = 1.0 / sqrt(s);
    for (int c = 0; c < 4; ++c) unit[4 * k + c] = (double)raw[4 * k + c] * inv;
  }
}

/* H[i][j] = (-1)^popcount(i & j): the Sylvester construction
 * H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]] in natural order. */
int orc_hadamard_entry(int i, int j) {
  return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

static void hadamard_normalised(const double *in, double *out) {
  const double s = 1.0 / sqrt((double)ORC_D);
  for (int i = 0; i < ORC_D; ++i) {
    double acc = 0.0;
    for (int j = 0; j < ORC_D; ++j) acc += orc_hadamard_entry(i, j) * in[j];
    out[i] = acc * s;
  }
}

void orc_rotate(const int8_t *signs, const double *uq, const double *x,
                double *y) {
  double t[ORC_D], u[ORC_D];
  for (int j = 0; j < ORC_D; ++j) t[j] = signs[j] * x[j];      /* D */
  hadamard_normalised(t, u);                                   /* Hn */
  for (int b = 0; b < ORC_BLOCKS; ++b) {                       /* B */
    const double *ql = uq + 8 * b, *qr = uq + 8 * b + 4;
    double cr[4], tmp[4];
    qconj(qr, cr);
    orc_qmul(ql, u + 4 * b, tmp);
    orc_qmul(tmp, cr, y + 4 * b);
  }
}

void orc_unrotate(const int8_t *signs, const double *uq, const double *y,
                  double *x) {
  double t[ORC_D], u[ORC_D];
  for (int b = 0; b < ORC_BLOCKS; ++b) {                       /* B^T */
    const double *ql = uq + 8 * b, *qr = uq + 8 * b + 4;
    double cl[4], tmp[4];
    qconj(ql, cl);
    orc_qmul(cl, y + 4 * b, tmp);
    orc_qmul(tmp, qr, t + 4 * b);
  }
  hadamard_normalised(t, u);                                   /* Hn^-1 = Hn */
  for (int j = 0; j < ORC_D; ++j) x[j] = signs[j] * u[j];      /* D^-1 = D */
}

/* ------------------------------------------------------ quantize and pack */

int orc_compress_b(int bits, int n, const double *x, const int8_t *signs,
                   const double *uq, uint32_t *codes, uint16_t *norms,
                   double *z_out) {
  int nlev, cpw, nw;
  orc_format(bits, &nlev, &cpw, &nw);
  double lv[ORC_MAX_LEVELS], th[ORC_MAX_LEVELS - 1];
  orc_codebook_b(bits, lv, th);
  int saturated = 0;
  for (int v = 0; v < n; ++v) {
    const double *xv = x + (size_t)v * ORC_D;
    double ss = 0.0;
    for (int j = 0; j < ORC_D; ++j) ss += xv[j] * xv[j];
    double nrm = sqrt(ss);
    int sat = 0;
    norms[v] = orc_f64_to_f16(nrm, &sat);
    saturated += sat;
    double y[ORC_D];
    orc_rotate(signs, uq, xv, y);
    uint32_t *w = codes + (size_t)v * nw;
    memset(w, 0, sizeof(uint32_t) * nw);
    for (int j = 0; j < ORC_D; ++j) {
      double z = (nrm > 0.0) ? sqrt((double)ORC_D) * y[j] / nrm : 0.0;
      if (z_out) z_out[(size_t)v * ORC_D + j] = z;
      uint32_t c = 0;
      for (int k = 0; k < nlev - 1; ++k) c += (z > th[k]) ? 1u : 0u;
      w[j / cpw] |= c << (bits * (j % cpw));
    }
  }
  return saturated;
}

int orc_compress(int n, const double *x, const int8_t *signs,
                 const double *uq, uint32_t *codes, uint16_t *norms,
                 double *z_out) {
  return orc_compress_b(3, n, x, signs, uq, codes, norms, z_out);
}

void orc_unpack_b(int bits, const uint32_t *words, uint8_t *codes) {
  int cpw;
  orc_format(bits, NULL, &cpw, NULL);
  const uint32_t mask = (1u << bits) - 1u;
  for (int j = 0; j < ORC_D; ++j)
    codes[j] = (uint8_t)((words[j / cpw] >> (bits * (j % cpw))) & mask);
}

void orc_unpack(const uint32_t *words, uint8_t *codes) { orc_unpack_b(3, words, codes); }

/* Centroid vector in rotated space, scaled by the stored norm:
 * (n16 / sqrt(128)) * C[code_j]. */
static void centroid_scaled(int bits, const uint32_t *words, uint16_t norm16,
                            const double *lv, double *out) {
  uint8_t c[ORC_D];
  orc_unpack_b(bits, words, c);
  double s = orc_f16_to_f64(norm16) / sqrt((double)ORC_D);
  for (int j = 0; j < ORC_D; ++j) out[j] = s * lv[c[j]];
}

void orc_dequantize_b(int bits, const uint32_t *words, uint16_t norm16,
                      const int8_t *signs, const double *uq, double *x_hat) {
  double lv[ORC_MAX_LEVELS], th[ORC_MAX_LEVELS - 1], yhat[ORC_D];
  orc_codebook_b(bits, lv, th);
  centroid_scaled(bits, words, norm16, lv, yhat);
  orc_unrotate(signs, uq, yhat, x_hat);
}

void orc_dequantize(const uint32_t *words, uint16_t norm16,
                    const int8_t *signs, const double *uq, double *x_hat) {
  orc_dequantize_b(3, words, norm16, signs, uq, x_hat);
}

/* ---------------------------------------------------------------- attention */

static void softmax_weighted_sum(int L, int limit, const double *scores,
                                 const double *vals /* [L][128] */,
                                 double *out) {
  memset(out, 0, sizeof(double) * ORC_D);
  if (limit <= 0) return;
  double m = -INFINITY;
  for (int t = 0; t < limit; ++t) if (scores[t] > m) m = scores[t];
  double l = 0.0;
  for (int t = 0; t < limit; ++t) {
    double p = exp(scores[t] - m);
    l += p;
    for (int j = 0; j < ORC_D; ++j) out[j] += p * vals[(size_t)t * ORC_D + j];
  }
  for (int j = 0; j < ORC_D; ++j) out[j] /= l;
  (void)L;
}

void orc_attend_b(int bits, int R, int L, const double *q, const uint32_t *kcodes,
                  const uint16_t *knorms, const uint32_t *vcodes,
                  const uint16_t *vnorms, const int *limit, double scale,
                  const int8_t *signs, const double *uq, double *out) {
  int nw;
  orc_format(bits, NULL, NULL, &nw);
  double lv[ORC_MAX_LEVELS], th[ORC_MAX_LEVELS - 1];
  orc_codebook_b(bits, lv, th);
  double *kc = (double *)malloc(sizeof(double) * (size_t)L * ORC_D + 8);
  double *vc = (double *)malloc(sizeof(double) * (size_t)L * ORC_D + 8);
  double *sc = (double *)malloc(sizeof(double) * (size_t)L + 8);
  /* rotated-space centroids of every token, norm applied */
  for (int t = 0; t < L; ++t) {
    centroid_scaled(bits, kcodes + (size_t)t * nw, knorms[t], lv, kc + (size_t)t * ORC_D);
    centroid_scaled(bits, vcodes + (size_t)t * nw, vnorms[t], lv, vc + (size_t)t * ORC_D);
  }
  for (int r = 0; r < R; ++r) {
    double qr[ORC_D], o[ORC_D];
    orc_rotate(signs, uq, q + (size_t)r * ORC_D, qr);          /* q~ = R q */
    int lim = limit[r] < L ? limit[r] : L;
    for (int t = 0; t < lim; ++t) {
      double acc = 0.0;
      for (int j = 0; j < ORC_D; ++j) acc += qr[j] * kc[(size_t)t * ORC_D + j];
      sc[t] = scale * acc;
    }
    softmax_weighted_sum(L, lim, sc, vc, o);                   /* o~ */
    if (lim > 0) orc_unrotate(signs, uq, o, out + (size_t)r * ORC_D);  /* R^-1 o~ */
    else memset(out + (size_t)r * ORC_D, 0, sizeof(double) * ORC_D);
  }
  free(kc); free(vc); free(sc);
}

void orc_attend(int R, int L, const double *q, const uint32_t *kcodes,
                const uint16_t *knorms, const uint32_t *vcodes,
                const uint16_t *vnorms, const int *limit, double scale,
                const int8_t *signs, const double *uq, double *out) {
  orc_attend_b(3, R, L, q, kcodes, knorms, vcodes, vnorms, limit, scale, signs, uq, out);
}

void orc_attend_bruteforce_b(int bits, int R, int L, const double *q,
                             const uint32_t *kcodes, const uint16_t *knorms,
                             const uint32_t *vcodes, const uint16_t *vnorms,
                             const int *limit, double scale,
                             const int8_t *signs, const double *uq,
                             double *out) {
  int nw;
  orc_format(bits, NULL, NULL, &nw);
  double *kx = (double *)malloc(sizeof(double) * (size_t)L * ORC_D + 8);
  double *vx = (double *)malloc(sizeof(double) * (size_t)L * ORC_D + 8);
  double *sc = (double *)malloc(sizeof(double) * (size_t)L + 8);
  for (int t = 0; t < L; ++t) {
    orc_dequantize_b(bits, kcodes + (size_t)t * nw, knorms[t], signs, uq, kx + (size_t)t * ORC_D);
    orc_dequantize_b(bits, vcodes + (size_t)t * nw, vnorms[t], signs, uq, vx + (size_t)t * ORC_D);
  }
  for (int r = 0; r < R; ++r) {
    int lim = limit[r] < L ? limit[r] : L;
    for (int t = 0; t < lim; ++t) {
      double acc = 0.0;
      for (int j = 0; j < ORC_D; ++j) acc += q[(size_t)r * ORC_D + j] * kx[(size_t)t * ORC_D + j];
      sc[t] = scale * acc;
    }
    softmax_weighted_sum(L, lim, sc, vx, out + (size_t)r * ORC_D);
  }
  free(kx); free(vx); free(sc);
}

void orc_attend_bruteforce(int R, int L, const double *q,
                           const uint32_t *kcodes, const uint16_t *knorms,
                           const uint32_t *vcodes, const uint16_t *vnorms,
                           const int *limit, double scale,
                           const int8_t *signs, const double *uq,
                           double *out) {
  orc_attend_bruteforce_b(3, R, L, q, kcodes, knorms, vcodes, vnorms, limit, scale, signs, uq, out);
}
