/*
 * isoquant_oracle.h -- plain fp64 CPU oracle for IsoQuant compressed-space
 * attention.  TEST INFRASTRUCTURE ONLY: the product path never includes,
 * links or calls anything declared here.  Only the test suite, the smoke
 * check and the CPU-baseline leg of the benchmark use it.
 *
 * Source of the method: "RotaryQuant: Fitting 120B MoE Models on Consumer
 * Hardware via Fused Compressed-Space Attention" (arXiv 2608.08081),
 * Abstract: a Walsh-Hadamard transform followed by block-diagonal SO(4)
 * rotations isotropizes each KV head vector (d = 128, 256 stored parameters
 * per head) before 3-bit scalar quantization; attention then runs directly on
 * the packed 3-bit tensors without materialising full-precision KV.
 *
 * The pages leave the quantizer, packing and conventions open.  The readings
 * this oracle follows (and which the CUDA library follows independently):
 *   - y = B * Hn * D * x: sign flips D first, then the normalised Sylvester
 *     Hadamard transform Hn = H/sqrt(128) (natural order), then 32 SO(4)
 *     blocks, block b acting on coordinates 4b..4b+3 seen as the quaternion
 *     (w,x,y,z) by v -> qL (x) v (x) conj(qR) (Hamilton product).
 *   - norm n = ||x||_2 in fp64, stored as fp16 (round to nearest even,
 *     saturating at 65504).
 *   - z_j = sqrt(128) * y_j / n with the unrounded n; code_j = number of
 *     thresholds t_k with z_j > t_k (ties go to the lower code).  Levels are
 *     the 8-level Lloyd-Max levels for N(0,1) rounded to fp16, ascending,
 *     code 0 = most negative; thresholds are midpoints of adjacent levels.
 *   - ten codes per little-endian 32-bit word, code j at bits 3*(j%10) of
 *     word j/10; 13 words per vector, unused bits zero.
 *   - scores s_t = scale * (n16_t / sqrt(128)) * <R q, C[code_t]>,
 *     softmax over the visible tokens, o = R^-1 sum_t p_t (n16v_t/sqrt(128))
 *     C[codev_t].
 */
#ifndef ISOQUANT_ORACLE_H
#define ISOQUANT_ORACLE_H
#include <stdint.h>

#define ORC_D 128
#define ORC_BLOCKS 32
#define ORC_WORDS 13
#define ORC_LEVELS 8
#define ORC_MAX_LEVELS 16

#ifdef __cplusplus
extern "C" {
#endif

/* Lloyd iteration for the nlev-level minimum-MSE quantizer of N(0,1).
 * levels[nlev], thresholds[nlev-1], *distortion = E[(Z-Q(Z))^2].
 * Returns the iteration count, or -1 if it did not converge. */
int orc_lloyd_max_gauss(int nlev, double *levels, double *thresholds,
                        double *distortion);

/* MSE of the quantizer (levels, midpoint thresholds) under N(0,1). */
double orc_gauss_distortion(int nlev, const double *levels,
                            const double *thresholds);

/* fp64 -> fp16 bits, round to nearest even; |x| >= 65520 saturates to
 * +-65504 and sets *saturated (if non-null). */
uint16_t orc_f64_to_f16(double x, int *saturated);
double orc_f16_to_f64(uint16_t h);

/* The canonical codebook: fp16-rounded Lloyd-Max levels (as doubles) and
 * the midpoints between adjacent levels. */
void orc_codebook(double levels16[ORC_LEVELS], double thresholds[ORC_LEVELS - 1]);

/* Other bit widths (the pages' system quantizes weights at 2, 4 and 8 bits;
 * its KV path is 3-bit): bits in {2, 3, 4} gives 2^bits fp16-rounded
 * Lloyd-Max levels and midpoint thresholds, floor(32 / bits) codes per word
 * (16, 10, 8; code j at bits bits*(j % per_word) of word j / per_word) and
 * ceil(128 / per_word) words per vector (8, 13, 16).  orc_format returns -1
 * for other widths.  The *_b functions below take the width; the functions
 * without the suffix are bits = 3. */
int orc_format(int bits, int *levels, int *per_word, int *words);
void orc_codebook_b(int bits, double *levels16, double *thresholds);
int orc_compress_b(int bits, int n, const double *x, const int8_t *signs,
                   const double *unit_quats, uint32_t *codes, uint16_t *norms,
                   double *z);
void orc_unpack_b(int bits, const uint32_t *words, uint8_t *codes);
void orc_dequantize_b(int bits, const uint32_t *words, uint16_t norm16,
                      const int8_t *signs, const double *unit_quats,
                      double *x_hat);
void orc_attend_b(int bits, int R, int L, const double *q, const uint32_t *kcodes,
                  const uint16_t *knorms, const uint32_t *vcodes,
                  const uint16_t *vnorms, const int *limit, double scale,
                  const int8_t *signs, const double *unit_quats, double *out);
void orc_attend_bruteforce_b(int bits, int R, int L, const double *q,
                             const uint32_t *kcodes, const uint16_t *knorms,
                             const uint32_t *vcodes, const uint16_t *vnorms,
                             const int *limit, double scale,
                             const int8_t *signs, const double *unit_quats,
                             double *out);

/* Hamilton product out = a (x) b, quaternions as (w, x, y, z). */
void orc_qmul(const double a[4], const double b[4], double out[4]);

/* Normalise raw per-head parameters [32][2][4] (left, right) to unit
 * quaternions in fp64. */
void orc_normalise_quats(const float *raw, double *unit);

/* Sylvester Hadamard entry (+1/-1), natural order. */
int orc_hadamard_entry(int i, int j);

/* y = B Hn D x and its inverse x = D Hn B^T y for one head. */
void orc_rotate(const int8_t *signs, const double *unit_quats,
                const double *x, double *y);
void orc_unrotate(const int8_t *signs, const double *unit_quats,
                  const double *y, double *x);

/* Compress n vectors x[n][128] of one head.  codes[n][13], norms[n] (fp16
 * bits); z[n][128] optional (may be NULL).  Returns the number of
 * saturated norms. */
int orc_compress(int n, const double *x, const int8_t *signs,
                 const double *unit_quats, uint32_t *codes, uint16_t *norms,
                 double *z);

/* Unpack one canonical 13-word vector into 128 codes. */
void orc_unpack(const uint32_t *words, uint8_t *codes);

/* Compressed-space attention for one KV head.
 * q[R][128] un-rotated queries; K/V: codes[L][13], norms[L] (fp16 bits);
 * limit[r] = number of leading tokens row r sees (0 <= limit <= L);
 * out[R][128].  A row with limit 0 outputs zeros. */
void orc_attend(int R, int L, const double *q, const uint32_t *kcodes,
                const uint16_t *knorms, const uint32_t *vcodes,
                const uint16_t *vnorms, const int *limit, double scale,
                const int8_t *signs, const double *unit_quats, double *out);

/* Same result by brute force: every K/V vector is dequantized and
 * un-rotated, then ordinary softmax attention runs with the un-rotated q. */
void orc_attend_bruteforce(int R, int L, const double *q,
                           const uint32_t *kcodes, const uint16_t *knorms,
                           const uint32_t *vcodes, const uint16_t *vnorms,
                           const int *limit, double scale,
                           const int8_t *signs, const double *unit_quats,
                           double *out);

/* Dequantize one vector back to the input space:
 * x_hat = R^-1 (n16/sqrt(128) * C[code]). */
void orc_dequantize(const uint32_t *words, uint16_t norm16,
                    const int8_t *signs, const double *unit_quats,
                    double *x_hat);

#ifdef __cplusplus
}
#endif
#endif
