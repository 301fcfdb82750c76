/*
 * Seeded synthetic input generator shared by the host (oracle side) and the
 * device (bulk inputs for the CUDA path).  It holds none of the codec's
 * arithmetic: it only draws numbers.
 *
 * Counter-based: every element is a pure function of (seed, stream, element
 * index), so any row of any tensor can be generated on its own, on either
 * side, in any order.
 *
 * Bits: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
 * as easy as 1, 2, 3", SC'11), written from the paper's definition:
 * 10 rounds of two 32x32->64 multiplies, key bumped by the Weyl constants
 * between rounds.
 * Normals: Box-Muller in binary64 from two 53-bit uniforms.
 * Student-t(df), integer df: Z / sqrt(chi2 / df), chi2 = sum of df squared
 * normals.  Row factor: exp(sigma * Z_row).  Values are rounded
 * binary64 -> binary32 (RN) -> bfloat16 (RNE) when bf16 is requested.
 *
 * Compiled by gcc (host) and by nvcc (device, with -fmad=false so that no
 * multiply-add is contracted); the only library calls are log, sqrt, cos,
 * sin and exp, so host and device agree except for last-ulp differences of
 * those functions, which a test checks on samples.
 */
#ifndef VQ3R_SYNTH_GEN_H
#define VQ3R_SYNTH_GEN_H

#include <stdint.h>
#include <math.h>

#ifdef __CUDACC__
#define SYNTH_FN __host__ __device__ static inline
#else
#define SYNTH_FN static inline
#endif

/* stream purposes (high byte of the 32-bit stream id) */
#define SYNTH_P_VALUE   1u  /* element values */
#define SYNTH_P_ROWF    2u  /* per-row log-normal factor */
#define SYNTH_P_OUTLIER 3u  /* outlier positions and signs */
#define SYNTH_P_SAMPLE  4u  /* training-vector / expert selection keys */

enum { SYNTH_DIST_NORMAL = 0, SYNTH_DIST_STUDENT_T = 1 };
enum { SYNTH_OUT_F32 = 0, SYNTH_OUT_BF16 = 1 };

typedef struct {
  int32_t kind;        /* SYNTH_DIST_NORMAL or SYNTH_DIST_STUDENT_T */
  int32_t df;          /* degrees of freedom for Student-t (integer >= 1) */
  double row_sigma;    /* >0: multiply each row by exp(row_sigma * Z_row) */
  double outlier_p;    /* probability that an element is replaced by an outlier */
  double outlier_mag;  /* outlier magnitude (before the row factor) */
} synth_dist;

SYNTH_FN void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; r++) {
    if (r) { k0 += W0; k1 += W1; }
    uint64_t p0 = (uint64_t)M0 * (uint64_t)x0;
    uint64_t p1 = (uint64_t)M1 * (uint64_t)x2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    x0 = hi1 ^ x1 ^ k0;
    x1 = lo1;
    x2 = hi0 ^ x3 ^ k1;
    x3 = lo0;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

SYNTH_FN uint32_t synth_stream(uint32_t purpose, uint32_t tag) {
  return (purpose << 24) ^ (tag & 0x00FFFFFFu);
}

/* Four raw words for (seed, stream, element e, draw d). */
SYNTH_FN void synth_words(uint64_t seed, uint32_t stream, uint64_t e, uint32_t d, uint32_t w[4]) {
  uint32_t ctr[4] = {(uint32_t)e, (uint32_t)(e >> 32), d, (uint32_t)(seed >> 32)};
  uint32_t key[2] = {(uint32_t)seed, stream};
  synth_philox4x32_10(ctr, key, w);
}

/* 53-bit uniform in [0,1) from two words. */
SYNTH_FN double synth_u53(uint32_t a, uint32_t b) {
  uint64_t m = ((uint64_t)(a >> 5) << 26) | (uint64_t)(b >> 6);
  return (double)m * (1.0 / 9007199254740992.0);
}

/* Normals 2*pair and 2*pair+1 of element e (Box-Muller). */
SYNTH_FN void synth_normal_pair(uint64_t seed, uint32_t stream, uint64_t e, uint32_t pair, double* z0, double* z1) {
  uint32_t w[4];
  synth_words(seed, stream, e, pair, w);
  double u1 = synth_u53(w[0], w[1]) + (1.0 / 9007199254740992.0); /* (0,1] */
  double u2 = synth_u53(w[2], w[3]);                                /* [0,1) */
  double rho = sqrt(-2.0 * log(u1));
  double th = 6.283185307179586 * u2;
  *z0 = rho * cos(th);
  *z1 = rho * sin(th);
}

SYNTH_FN double synth_normal(uint64_t seed, uint32_t stream, uint64_t e, uint32_t j) {
  double a, b;
  synth_normal_pair(seed, stream, e, j >> 1, &a, &b);
  return (j & 1u) ? b : a;
}

/* Student-t with integer df: normals 0..df of element e. */
SYNTH_FN double synth_student_t(uint64_t seed, uint32_t stream, uint64_t e, int df) {
  double z = 0.0, chi2 = 0.0;
  for (int j = 0; j <= df; j += 2) {
    double a, b;
    synth_normal_pair(seed, stream, e, (uint32_t)(j >> 1), &a, &b);
    if (j == 0) z = a; else chi2 = chi2 + a * a;
    if (j + 1 <= df) chi2 = chi2 + b * b;
  }
  return z / sqrt(chi2 / (double)df);
}

SYNTH_FN double synth_row_factor(uint64_t seed, uint32_t tag, uint64_t row, double sigma) {
  if (!(sigma > 0.0)) return 1.0;
  return exp(sigma * synth_normal(seed, synth_stream(SYNTH_P_ROWF, tag), row, 0));
}

/* Value of element (row, col) of a rows x cols tensor, before output rounding,
 * given its row factor. */
SYNTH_FN double synth_value(uint64_t seed, uint32_t tag, int64_t cols, int64_t row, int64_t col,
                            const synth_dist* d, double rowf) {
  uint64_t e = (uint64_t)row * (uint64_t)cols + (uint64_t)col;
  uint32_t sv = synth_stream(SYNTH_P_VALUE, tag);
  double v;
  if (d->kind == SYNTH_DIST_STUDENT_T) v = synth_student_t(seed, sv, e, d->df);
  else v = synth_normal(seed, sv, e, 0);
  if (d->outlier_p > 0.0) {
    uint32_t w[4];
    synth_words(seed, synth_stream(SYNTH_P_OUTLIER, tag), e, 0, w);
    if (synth_u53(w[0], w[1]) < d->outlier_p) v = (w[2] & 1u) ? -d->outlier_mag : d->outlier_mag;
  }
  return v * rowf;
}

SYNTH_FN float synth_round_f32(double v) { return (float)v; }

/* binary32 -> bfloat16 bits, round to nearest even; NaN kept quiet. */
SYNTH_FN uint16_t synth_f32_to_bf16(float f) {
  union { float f; uint32_t u; } c; c.f = f;
  uint32_t u = c.u;
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u = u + 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* Sampling key of item i: a 64-bit draw; the k smallest keys are a uniform
 * sample without replacement, in key order. */
SYNTH_FN uint64_t synth_sample_key(uint64_t seed, uint32_t tag, uint64_t i) {
  uint32_t w[4];
  synth_words(seed, synth_stream(SYNTH_P_SAMPLE, tag), i, 0, w);
  return ((uint64_t)w[0] << 32) | (uint64_t)w[1];
}

#endif
