/*
 * VQ3R oracle: a plain, slow CPU statement of what the VQ3R codec computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library; the product path
 * (the CUDA library and its Python binding) never does, and shares no code
 * with it.
 *
 * Source: "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验"
 * (xdnf.cn/news/289497).
 *   §2 (what VQ3R is): 3 stages, each a 256-entry codebook of 8-dim vectors
 *       with a 1-byte index, one FP16 per-row scale, 3.00 bits/weight;
 *       reconstruction W ~ scale x (C1[i1] + C2[i2] + C3[i3]); stage 1 fits
 *       the vector, stage 2 the stage-1 residual, stage 3 the stage-2
 *       residual; codebooks per layer by Lloyd k-means.
 *   §3.1 (Gate 3 table): relative Frobenius error as the metric; the
 *       rtn4-row int4 per-row baseline; vq2 = the first two stages.
 *   §4 (engineering loop): a single pass over the three stages that keeps
 *       only the winning indices.
 *
 * The pages leave open: the scale's value and rounding, the summation
 * orders, the distance formula and tie rule, Lloyd's initialisation and
 * empty clusters, and the rtn4-row details.  The readings taken here:
 *   - scale = binary16(RMS of the row), RMS from a binary64 sum of squares in
 *     a fixed order (per-vector sums, 128 strided partials, halving tree),
 *     one rounding to binary16 (RNE), overflow saturating to 65504;
 *   - r = (float)w / (float)scale, r = 0 when the scale is 0;
 *   - d_j = sum_k (r_k - c_jk)^2 in binary32, k ascending, each operation
 *     rounded (no fused multiply-add); the lowest index wins ties;
 *   - decode: (float)scale * ((C1 + C2) + C3) in binary32;
 *   - Lloyd: init = first 256 training vectors, assignment by the encoder's
 *     distance and tie rule, centroid = binary64 mean rounded to binary32,
 *     an empty cluster keeps its centroid, a fixed number of iterations;
 *   - rtn4-row: symmetric, scale = binary16(max|w| / 7), q = clamp(rint(w /
 *     scale), -8, 7).
 *
 * Build: C11, -O2 -ffp-contract=off, no fast-math (binary32 and binary64
 * arithmetic exactly as written; x86-64 SSE evaluates float in float).
 * OpenMP runs independent rows in parallel; no result depends on the
 * thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F16 = 2 };
#define ORC_K 256 /* codewords per stage (§2) */
#define ORC_D 8   /* dimensions per vector (§2) */

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---------------- IEEE 754 binary16 / bfloat16 conversions ---------------- */

/* binary64 -> binary16 bits, round to nearest even.  saturate != 0 maps an
 * overflow to +-65504 (the scale reading); otherwise to +-inf. */
static uint16_t fp16_from_double(double x, int saturate) {
  if (isnan(x)) return 0x7E00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (a >= 65520.0) return sign | (saturate ? 0x7BFF : 0x7C00);
  int e;
  frexp(a, &e);     /* a = m * 2^e, m in [0.5, 1) */
  e -= 1;           /* a in [2^e, 2^(e+1)) */
  if (e < -14) {    /* subnormal range: quantum 2^-24 */
    double q = rint(ldexp(a, 24));
    return sign | (uint16_t)q; /* q == 1024 encodes 2^-14 */
  }
  double q = rint(ldexp(a, 10 - e)); /* in [1024, 2048] */
  if (q == 2048.0) { q = 1024.0; e += 1; }
  if (e > 15) return sign | (saturate ? 0x7BFF : 0x7C00);
  return sign | (uint16_t)(((e + 15) << 10) | ((int)q - 1024));
}

uint16_t orc_fp16_from_double_sat(double x) { return fp16_from_double(x, 1); }
uint16_t orc_fp16_from_float(float x) { return fp16_from_double((double)x, 0); }

double orc_fp16_to_double(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(m + 1024), e - 25);
  return s ? -v : v;
}

float orc_bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* binary32 -> bfloat16 bits by round to nearest, ties to even on the 16
 * dropped bits (a NaN stays a quiet NaN). */
uint16_t orc_bf16_from_float(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x0040u);
  const uint32_t rest = u & 0xFFFFu, keep = u >> 16;
  if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) return (uint16_t)(keep + 1u);
  return (uint16_t)keep;
}

static float load_w(const void* W, int dtype, int64_t i) {
  if (dtype == ORC_BF16) return orc_bf16_to_float(((const uint16_t*)W)[i]);
  if (dtype == ORC_F16) return (float)orc_fp16_to_double(((const uint16_t*)W)[i]);
  return ((const float*)W)[i];
}

/* ---------------- per-row FP16 scale (§2), RMS reading ---------------- */

/* Sum of squares of one row in the fixed binary64 order: per-vector sums
 * q_v = ((w0^2 + w1^2) + ...) + w7^2; 128 partials t_p over v = p mod 128,
 * v ascending; then t_p += t_{p+h} for h = 64, 32, ..., 1. */
double orc_row_sumsq(const void* W, int dtype, int64_t row, int64_t cols) {
  int64_t V = cols / ORC_D;
  double t[128];
  for (int p = 0; p < 128; p++) {
    t[p] = 0.0;
    for (int64_t v = p; v < V; v += 128) {
      double q = 0.0;
      for (int k = 0; k < ORC_D; k++) {
        double w = (double)load_w(W, dtype, row * cols + v * ORC_D + k);
        q = (k == 0) ? w * w : q + w * w;
      }
      t[p] = t[p] + q;
    }
  }
  for (int h = 64; h >= 1; h >>= 1)
    for (int p = 0; p < h; p++) t[p] = t[p] + t[p + h];
  return t[0];
}

uint16_t orc_row_scale(const void* W, int dtype, int64_t row, int64_t cols) {
  double ss = orc_row_sumsq(W, dtype, row, cols);
  return orc_fp16_from_double_sat(sqrt(ss / (double)cols));
}

void orc_row_scales(const void* W, int dtype, int64_t rows, int64_t cols, uint16_t* scales) {
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; i++) scales[i] = orc_row_scale(W, dtype, i, cols);
}

/* ---------------- greedy residual assignment (§2, §4) ---------------- */

/* Nearest codeword of one stage: d_j = sum_k (r_k - c_jk)^2, binary32, k
 * ascending, no fused operations; strict '<' keeps the lowest index. */
static int nearest(const float* r, const float* C) {
  float best = INFINITY;
  int bi = 0;
  for (int j = 0; j < ORC_K; j++) {
    const float* c = C + ORC_D * j;
    float e = r[0] - c[0];
    float d = e * e;
    for (int k = 1; k < ORC_D; k++) {
      float ek = r[k] - c[k];
      float sq = ek * ek;
      d = d + sq;
    }
    if (d < best) { best = d; bi = j; }
  }
  return bi;
}

/* Greedy encode of n normalised vectors r (n x 8): for each stage, the
 * nearest codeword of the running residual, then residual -= codeword.
 * idx is n x nstages (vector-major); resid_out (optional) gets the final
 * residual. */
void orc_encode_vectors(const float* r_in, int64_t n, const float* codebooks, int nstages,
                        uint8_t* idx, float* resid_out) {
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; i++) {
    float r[ORC_D];
    for (int k = 0; k < ORC_D; k++) r[k] = r_in[i * ORC_D + k];
    for (int s = 0; s < nstages; s++) {
      const float* C = codebooks + (int64_t)s * ORC_K * ORC_D;
      int j = nearest(r, C);
      idx[i * nstages + s] = (uint8_t)j;
      for (int k = 0; k < ORC_D; k++) r[k] = r[k] - C[ORC_D * j + k];
    }
    if (resid_out)
      for (int k = 0; k < ORC_D; k++) resid_out[i * ORC_D + k] = r[k];
  }
}

/* Normalise vector v of row i by its scale: r = (float)w / (float)s. */
static void normalise(const void* W, int dtype, int64_t cols, int64_t i, int64_t v, uint16_t s, float* r) {
  float sf = (float)orc_fp16_to_double(s);
  for (int k = 0; k < ORC_D; k++) {
    float w = load_w(W, dtype, i * cols + v * ORC_D + k);
    r[k] = (sf == 0.0f) ? 0.0f : w / sf;
  }
}

/* Normalised vectors of n rows (n x cols) given their scales: out is
 * (n * cols/8) x 8, r = (float)w / (float)scale, 0 when the scale is 0. */
void orc_normalize_rows(const void* W, int dtype, int64_t n, int64_t cols, const uint16_t* scales, float* out) {
  int64_t V = cols / ORC_D;
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; i++)
    for (int64_t v = 0; v < V; v++) normalise(W, dtype, cols, i, v, scales[i], out + (i * V + v) * ORC_D);
}

/* Encode a rows x cols matrix: scales[rows] (binary16 bits) and index planes
 * idx[nstages][rows][cols/8], plane-major, each plane row-major. */
int orc_encode(const void* W, int dtype, int64_t rows, int64_t cols, const float* codebooks, int nstages,
               uint8_t* idx, uint16_t* scales) {
  if (rows < 0 || cols < ORC_D || cols % ORC_D || nstages < 1 || nstages > 3) return 2;
  int64_t V = cols / ORC_D;
  #pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < rows; i++) {
    uint16_t s = orc_row_scale(W, dtype, i, cols);
    scales[i] = s;
    for (int64_t v = 0; v < V; v++) {
      float r[ORC_D];
      normalise(W, dtype, cols, i, v, s, r);
      for (int st = 0; st < nstages; st++) {
        const float* C = codebooks + (int64_t)st * ORC_K * ORC_D;
        int j = nearest(r, C);
        idx[((int64_t)st * rows + i) * V + v] = (uint8_t)j;
        for (int k = 0; k < ORC_D; k++) r[k] = r[k] - C[ORC_D * j + k];
      }
    }
  }
  return 0;
}

/* Encode only the listed rows of W (W holds just those rows, n x cols);
 * outputs are n x ... in the same plane-major layout. */
int orc_encode_rows(const void* Wrows, int dtype, int64_t n, int64_t cols, const float* codebooks,
                    uint8_t* idx, uint16_t* scales) {
  return orc_encode(Wrows, dtype, n, cols, codebooks, 3, idx, scales);
}

/* ---------------- decode (§2 reconstruction rule) ---------------- */

/* w_hat = (float)scale * ((C1[i1] + C2[i2]) + C3[i3]) in binary32 (fewer
 * terms for nstages < 3).  out_dtype ORC_F32, ORC_F16 (RNE of the binary32
 * value, overflow to inf) or ORC_BF16 (RNE of the binary32 value; the
 * weights a bf16 tensor-core product consumes). */
int orc_decode(const uint8_t* idx, const uint16_t* scales, const float* codebooks, int64_t rows, int64_t cols,
               int nstages, void* out, int out_dtype) {
  if (rows < 0 || cols < ORC_D || cols % ORC_D || nstages < 1 || nstages > 3) return 2;
  int64_t V = cols / ORC_D;
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; i++) {
    float sf = (float)orc_fp16_to_double(scales[i]);
    for (int64_t v = 0; v < V; v++) {
      for (int k = 0; k < ORC_D; k++) {
        float acc = codebooks[(int64_t)idx[i * V + v] * ORC_D + k];
        for (int st = 1; st < nstages; st++) {
          int j = idx[((int64_t)st * rows + i) * V + v];
          acc = acc + codebooks[((int64_t)st * ORC_K + j) * ORC_D + k];
        }
        float w = sf * acc;
        int64_t o = i * cols + v * ORC_D + k;
        if (out_dtype == ORC_F16) ((uint16_t*)out)[o] = orc_fp16_from_float(w);
        else if (out_dtype == ORC_BF16) ((uint16_t*)out)[o] = orc_bf16_from_float(w);
        else ((float*)out)[o] = w;
      }
    }
  }
  return 0;
}

/* ---------------- relative Frobenius error (§3.1 metric) ---------------- */

/* sqrt(sum (w - w_hat)^2 / sum w^2), binary64 sums in element order. */
double orc_rel_frobenius(const void* W, int dtype, const float* What, int64_t n) {
  double num = 0.0, den = 0.0;
  for (int64_t i = 0; i < n; i++) {
    double w = (double)load_w(W, dtype, i);
    double e = w - (double)What[i];
    num = num + e * e;
    den = den + w * w;
  }
  return sqrt(num / den);
}

/* ---------------- GEMV with the decoded matrix ---------------- */

/* y[b][i] = sum_c w_hat[i][c] * x[b][c] in binary64 (c ascending). */
int orc_gemv(const float* What, int64_t rows, int64_t cols, const void* x, int x_dtype, int B, double* y) {
  if (rows < 0 || cols < 1 || B < 1) return 2;
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; i++) {
    for (int b = 0; b < B; b++) {
      double acc = 0.0;
      for (int64_t c = 0; c < cols; c++)
        acc = acc + (double)What[i * cols + c] * (double)load_w(x, x_dtype, (int64_t)b * cols + c);
      y[(int64_t)b * rows + i] = acc;
    }
  }
  return 0;
}

/* ---------------- Lloyd k-means codebook training (§2, §4) ---------------- */

/* Train nstages codebooks on n normalised vectors (n >= 256): stage s is
 * trained on the residuals left by stages 1..s-1.  Each stage starts from its
 * first 256 training vectors and runs `iters` iterations of (assign with the
 * encoder's distance and tie rule; centroid = binary64 mean of its members in
 * vector order, rounded to binary32; empty clusters keep their centroid).
 * The next stage's set is r - C[nearest] under the final centroids.
 * trace (optional, nstages x (iters + 1)) gets the binary64 total squared
 * distance of each assignment step, the last one under the final centroids. */
int orc_lloyd_train(const float* vecs, int64_t n, int iters, int nstages, float* codebooks, double* trace) {
  if (n < ORC_K || iters < 0 || nstages < 1 || nstages > 3) return 2;
  float* R = (float*)malloc(sizeof(float) * (size_t)n * ORC_D);
  int* a = (int*)malloc(sizeof(int) * (size_t)n);
  double* sum = (double*)malloc(sizeof(double) * ORC_K * ORC_D);
  int64_t* cnt = (int64_t*)malloc(sizeof(int64_t) * ORC_K);
  if (!R || !a || !sum || !cnt) { free(R); free(a); free(sum); free(cnt); return 3; }
  memcpy(R, vecs, sizeof(float) * (size_t)n * ORC_D);
  for (int s = 0; s < nstages; s++) {
    float* C = codebooks + (int64_t)s * ORC_K * ORC_D;
    memcpy(C, R, sizeof(float) * ORC_K * ORC_D);
    for (int it = 0; it <= iters; it++) {
      double dist = 0.0;
      #pragma omp parallel for schedule(static)
      for (int64_t i = 0; i < n; i++) a[i] = nearest(R + i * ORC_D, C);
      for (int64_t i = 0; i < n; i++)
        for (int k = 0; k < ORC_D; k++) {
          double e = (double)R[i * ORC_D + k] - (double)C[a[i] * ORC_D + k];
          dist = dist + e * e;
        }
      if (trace) trace[(int64_t)s * (iters + 1) + it] = dist;
      if (it == iters) break;
      memset(sum, 0, sizeof(double) * ORC_K * ORC_D);
      memset(cnt, 0, sizeof(int64_t) * ORC_K);
      for (int64_t i = 0; i < n; i++) {
        cnt[a[i]]++;
        for (int k = 0; k < ORC_D; k++) sum[a[i] * ORC_D + k] = sum[a[i] * ORC_D + k] + (double)R[i * ORC_D + k];
      }
      for (int j = 0; j < ORC_K; j++)
        if (cnt[j] > 0)
          for (int k = 0; k < ORC_D; k++) C[j * ORC_D + k] = (float)(sum[j * ORC_D + k] / (double)cnt[j]);
    }
    for (int64_t i = 0; i < n; i++)
      for (int k = 0; k < ORC_D; k++) R[i * ORC_D + k] = R[i * ORC_D + k] - C[a[i] * ORC_D + k];
  }
  free(R); free(a); free(sum); free(cnt);
  return 0;
}

/* ---------------- rtn4-row baseline (§3.1) ---------------- */

/* Symmetric int4 round-to-nearest with one binary16 scale per row:
 * scale = binary16(max|w| / 7), q = clamp(rint(w / scale), -8, 7),
 * w_hat = q * scale (exact in binary32). */
int orc_rtn4_row(const void* W, int dtype, int64_t rows, int64_t cols, float* What, uint16_t* scales) {
  if (rows < 0 || cols < 1) return 2;
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; i++) {
    double amax = 0.0;
    for (int64_t c = 0; c < cols; c++) {
      double a = fabs((double)load_w(W, dtype, i * cols + c));
      if (a > amax) amax = a;
    }
    uint16_t sh = orc_fp16_from_double_sat(amax / 7.0);
    if (scales) scales[i] = sh;
    double s = orc_fp16_to_double(sh);
    for (int64_t c = 0; c < cols; c++) {
      double q = 0.0;
      if (s > 0.0) {
        q = rint((double)load_w(W, dtype, i * cols + c) / s);
        if (q < -8.0) q = -8.0;
        if (q > 7.0) q = 7.0;
      }
      What[i * cols + c] = (float)(q * s);
    }
  }
  return 0;
}

/* ---------------- exhaustive joint search (lower bound for greedy) ---------------- */

/* For each of n normalised vectors, the (i1, i2, i3) minimising
 * sum_k (r_k - (C1[i1]_k + C2[i2]_k + C3[i3]_k))^2 over all 256^3 triples,
 * evaluated in binary64. */
void orc_bruteforce_joint(const float* r, int64_t n, const float* codebooks, int32_t* best_idx, double* best_err) {
  const float* C1 = codebooks;
  const float* C2 = codebooks + ORC_K * ORC_D;
  const float* C3 = codebooks + 2 * ORC_K * ORC_D;
  for (int64_t i = 0; i < n; i++) {
    double best = INFINITY;
    int32_t b1 = 0, b2 = 0, b3 = 0;
    #pragma omp parallel
    {
      double lbest = INFINITY;
      int32_t l1 = 0, l2 = 0, l3 = 0;
      #pragma omp for schedule(static)
      for (int a = 0; a < ORC_K; a++) {
        for (int b = 0; b < ORC_K; b++) {
          double p[ORC_D];
          for (int k = 0; k < ORC_D; k++)
            p[k] = (double)r[i * ORC_D + k] - ((double)C1[a * ORC_D + k] + (double)C2[b * ORC_D + k]);
          for (int c = 0; c < ORC_K; c++) {
            double e = 0.0;
            for (int k = 0; k < ORC_D; k++) {
              double t = p[k] - (double)C3[c * ORC_D + k];
              e = e + t * t;
            }
            if (e < lbest) { lbest = e; l1 = a; l2 = b; l3 = c; }
          }
        }
      }
      #pragma omp critical
      {
        if (lbest < best || (lbest == best && (l1 < b1 || (l1 == b1 && (l2 < b2 || (l2 == b2 && l3 < b3)))))) {
          best = lbest; b1 = l1; b2 = l2; b3 = l3;
        }
      }
    }
    best_idx[i * 3 + 0] = b1; best_idx[i * 3 + 1] = b2; best_idx[i * 3 + 2] = b3;
    best_err[i] = best;
  }
}

/* ---------------- VQ4P (page §5): 4 stages x 64 entries, 6-bit packed indices ---------------- */
/*
 * The page names VQ4P as VQ3R's sibling at the same 3.00 bits/weight: four
 * stages of 64-entry codebooks, 6-bit indices packed so that the container is
 * byte-for-byte the size of VQ3R's.  The page gives no packing, scale or
 * arithmetic details; the readings taken here keep everything of VQ3R that
 * applies and add the packing:
 *   - the same per-row binary16 RMS scale and normalisation;
 *   - stage s (s = 1..4) picks the nearest of 64 codewords to the running
 *     residual with VQ3R's distance (binary32, every operation rounded, k
 *     ascending) and tie rule (lowest index); r -= C_s[i_s];
 *   - the four indices of a vector form the 24-bit word
 *     i1 | i2 << 6 | i3 << 12 | i4 << 18, stored as three byte planes:
 *     plane p of [3][rows][cols/8] holds byte p of each vector's word;
 *   - decode: (float)scale * (((C1 + C2) + C3) + C4) in binary32;
 *   - Lloyd per stage as for VQ3R with 64 centroids (init = first 64
 *     vectors).
 */
#define ORC_K4 64
#define ORC_S4 4

static int nearest_k(const float* r, const float* C, int K) {
  float best = INFINITY;
  int bi = 0;
  for (int j = 0; j < K; j++) {
    const float* c = C + ORC_D * j;
    float e = r[0] - c[0];
    float d = e * e;
    for (int k = 1; k < ORC_D; k++) {
      float ek = r[k] - c[k];
      float sq = ek * ek;
      d = d + sq;
    }
    if (d < best) { best = d; bi = j; }
  }
  return bi;
}

/* idx4 [4][n] (one byte per index, values < 64) <-> planes [3][n]. */
void orc_vq4p_pack(const uint8_t* idx4, int64_t n, uint8_t* planes) {
  for (int64_t i = 0; i < n; i++) {
    uint32_t w = (uint32_t)(idx4[i] & 63) | ((uint32_t)(idx4[n + i] & 63) << 6) |
                 ((uint32_t)(idx4[2 * n + i] & 63) << 12) | ((uint32_t)(idx4[3 * n + i] & 63) << 18);
    planes[i] = (uint8_t)(w & 0xFF);
    planes[n + i] = (uint8_t)((w >> 8) & 0xFF);
    planes[2 * n + i] = (uint8_t)((w >> 16) & 0xFF);
  }
}

void orc_vq4p_unpack(const uint8_t* planes, int64_t n, uint8_t* idx4) {
  for (int64_t i = 0; i < n; i++) {
    uint32_t w = (uint32_t)planes[i] | ((uint32_t)planes[n + i] << 8) | ((uint32_t)planes[2 * n + i] << 16);
    for (int s = 0; s < ORC_S4; s++) idx4[(int64_t)s * n + i] = (uint8_t)((w >> (6 * s)) & 63);
  }
}

/* Greedy 4-stage assignment of n normalised vectors: idx4 [n][4] (vector-major),
 * resid_out (optional) the final residuals. */
void orc_vq4p_encode_vectors(const float* r_in, int64_t n, const float* codebooks, uint8_t* idx4, float* resid_out) {
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; i++) {
    float r[ORC_D];
    for (int k = 0; k < ORC_D; k++) r[k] = r_in[i * ORC_D + k];
    for (int s = 0; s < ORC_S4; s++) {
      const float* C = codebooks + (int64_t)s * ORC_K4 * ORC_D;
      int j = nearest_k(r, C, ORC_K4);
      idx4[i * ORC_S4 + s] = (uint8_t)j;
      for (int k = 0; k < ORC_D; k++) r[k] = r[k] - C[ORC_D * j + k];
    }
    if (resid_out)
      for (int k = 0; k < ORC_D; k++) resid_out[i * ORC_D + k] = r[k];
  }
}

/* Encode a rows x cols matrix: scales[rows] and the packed planes [3][rows][cols/8]. */
int orc_vq4p_encode(const void* W, int dtype, int64_t rows, int64_t cols, const float* codebooks, uint8_t* planes,
                    uint16_t* scales) {
  if (rows < 0 || cols < ORC_D || cols % ORC_D) return 2;
  int64_t V = cols / ORC_D, n = rows * V;
  #pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < rows; i++) {
    uint16_t s = orc_row_scale(W, dtype, i, cols);
    scales[i] = s;
    for (int64_t v = 0; v < V; v++) {
      float r[ORC_D];
      normalise(W, dtype, cols, i, v, s, r);
      uint32_t w = 0;
      for (int st = 0; st < ORC_S4; st++) {
        const float* C = codebooks + (int64_t)st * ORC_K4 * ORC_D;
        int j = nearest_k(r, C, ORC_K4);
        w |= (uint32_t)j << (6 * st);
        for (int k = 0; k < ORC_D; k++) r[k] = r[k] - C[ORC_D * j + k];
      }
      planes[i * V + v] = (uint8_t)(w & 0xFF);
      planes[n + i * V + v] = (uint8_t)((w >> 8) & 0xFF);
      planes[2 * n + i * V + v] = (uint8_t)((w >> 16) & 0xFF);
    }
  }
  return 0;
}

/* w_hat = (float)scale * (((C1 + C2) + C3) + C4), binary32; out_dtype as orc_decode. */
int orc_vq4p_decode(const uint8_t* planes, const uint16_t* scales, const float* codebooks, int64_t rows, int64_t cols,
                    void* out, int out_dtype) {
  if (rows < 0 || cols < ORC_D || cols % ORC_D) return 2;
  int64_t V = cols / ORC_D, n = rows * V;
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; i++) {
    float sf = (float)orc_fp16_to_double(scales[i]);
    for (int64_t v = 0; v < V; v++) {
      int64_t e = i * V + v;
      uint32_t w = (uint32_t)planes[e] | ((uint32_t)planes[n + e] << 8) | ((uint32_t)planes[2 * n + e] << 16);
      for (int k = 0; k < ORC_D; k++) {
        float acc = codebooks[(int64_t)(w & 63) * ORC_D + k];
        for (int st = 1; st < ORC_S4; st++) {
          int j = (int)((w >> (6 * st)) & 63);
          acc = acc + codebooks[((int64_t)st * ORC_K4 + j) * ORC_D + k];
        }
        float x = sf * acc;
        int64_t o = i * cols + v * ORC_D + k;
        if (out_dtype == ORC_F16) ((uint16_t*)out)[o] = orc_fp16_from_float(x);
        else if (out_dtype == ORC_BF16) ((uint16_t*)out)[o] = orc_bf16_from_float(x);
        else ((float*)out)[o] = x;
      }
    }
  }
  return 0;
}

/* Lloyd per stage with 64 centroids; as orc_lloyd_train otherwise. */
int orc_vq4p_train(const float* vecs, int64_t n, int iters, float* codebooks, double* trace) {
  if (n < ORC_K4 || iters < 0) return 2;
  float* R = (float*)malloc(sizeof(float) * (size_t)n * ORC_D);
  int* a = (int*)malloc(sizeof(int) * (size_t)n);
  double* sum = (double*)malloc(sizeof(double) * ORC_K4 * ORC_D);
  int64_t* cnt = (int64_t*)malloc(sizeof(int64_t) * ORC_K4);
  if (!R || !a || !sum || !cnt) { free(R); free(a); free(sum); free(cnt); return 3; }
  memcpy(R, vecs, sizeof(float) * (size_t)n * ORC_D);
  for (int s = 0; s < ORC_S4; s++) {
    float* C = codebooks + (int64_t)s * ORC_K4 * ORC_D;
    memcpy(C, R, sizeof(float) * ORC_K4 * ORC_D);
    for (int it = 0; it <= iters; it++) {
      double dist = 0.0;
      #pragma omp parallel for schedule(static)
      for (int64_t i = 0; i < n; i++) a[i] = nearest_k(R + i * ORC_D, C, ORC_K4);
      for (int64_t i = 0; i < n; i++)
        for (int k = 0; k < ORC_D; k++) {
          double e = (double)R[i * ORC_D + k] - (double)C[a[i] * ORC_D + k];
          dist = dist + e * e;
        }
      if (trace) trace[(int64_t)s * (iters + 1) + it] = dist;
      if (it == iters) break;
      memset(sum, 0, sizeof(double) * ORC_K4 * ORC_D);
      memset(cnt, 0, sizeof(int64_t) * ORC_K4);
      for (int64_t i = 0; i < n; i++) {
        cnt[a[i]]++;
        for (int k = 0; k < ORC_D; k++) sum[a[i] * ORC_D + k] = sum[a[i] * ORC_D + k] + (double)R[i * ORC_D + k];
      }
      for (int j = 0; j < ORC_K4; j++)
        if (cnt[j] > 0)
          for (int k = 0; k < ORC_D; k++) C[j * ORC_D + k] = (float)(sum[j * ORC_D + k] / (double)cnt[j]);
    }
    for (int64_t i = 0; i < n; i++)
      for (int k = 0; k < ORC_D; k++) R[i * ORC_D + k] = R[i * ORC_D + k] - C[a[i] * ORC_D + k];
  }
  free(R); free(a); free(sum); free(cnt);
  return 0;
}

/* Exhaustive joint search over all 64^4 quadruples (binary64), per vector. */
void orc_vq4p_bruteforce(const float* r, int64_t n, const float* codebooks, int32_t* best_idx, double* best_err) {
  const float* C = codebooks;
  for (int64_t i = 0; i < n; i++) {
    double best = INFINITY;
    int32_t bb[4] = {0, 0, 0, 0};
    #pragma omp parallel
    {
      double lbest = INFINITY;
      int32_t lb[4] = {0, 0, 0, 0};
      #pragma omp for schedule(static)
      for (int a = 0; a < ORC_K4; a++)
        for (int b = 0; b < ORC_K4; b++)
          for (int c = 0; c < ORC_K4; c++) {
            double p[ORC_D];
            for (int k = 0; k < ORC_D; k++)
              p[k] = (double)r[i * ORC_D + k] - (((double)C[a * ORC_D + k] + (double)C[(ORC_K4 + b) * ORC_D + k]) +
                                                 (double)C[(2 * ORC_K4 + c) * ORC_D + k]);
            for (int d = 0; d < ORC_K4; d++) {
              double e = 0.0;
              for (int k = 0; k < ORC_D; k++) {
                double t = p[k] - (double)C[(3 * ORC_K4 + d) * ORC_D + k];
                e = e + t * t;
              }
              if (e < lbest) { lbest = e; lb[0] = a; lb[1] = b; lb[2] = c; lb[3] = d; }
            }
          }
      #pragma omp critical
      {
        int better = lbest < best;
        if (lbest == best)
          for (int q = 0; q < 4; q++) {
            if (lb[q] != bb[q]) { better = lb[q] < bb[q]; break; }
          }
        if (better) {
          best = lbest;
          for (int q = 0; q < 4; q++) bb[q] = lb[q];
        }
      }
    }
    for (int q = 0; q < 4; q++) best_idx[i * 4 + q] = bb[q];
    best_err[i] = best;
  }
}

/* ---------------- outlier-aware variant: sparse FP16 residual on top of VQ3R ---------------- */
/*
 * Page "XFP：质量目标驱动的自适应码本量化" (zingnex.cn/forum/thread/xfp-llm),
 * 技术实现 / 权重分解: a weight matrix is split into a dense index tensor
 * into learned codebooks and a sparse FP16 outlier residual kept at full
 * precision; the outlier budget is a parameter of the format.  The page
 * gives no selection rule, layout or combination order; readings:
 *   - the dense part is the VQ3R encoding of W and w_hat its binary32 decode;
 *   - e = (double)w - (double)w_hat (one binary64 subtraction);
 *   - per row, the k positions with the largest |e| are the outliers (|e|
 *     ordered by its binary64 bit pattern, so a NaN ranks first), ties to
 *     the lower column;
 *   - each outlier stores its column (uint16) and o = fp16(e) (round to
 *     nearest even, saturating at +-65504), the k entries of a row in
 *     ascending column order;
 *   - the decode adds (float)o to w_hat in binary32.
 */
typedef struct { uint64_t key; int64_t col; } orc_outlier_cand;

static int orc_outlier_rank(const void* a, const void* b) {
  const orc_outlier_cand* x = (const orc_outlier_cand*)a;
  const orc_outlier_cand* y = (const orc_outlier_cand*)b;
  if (x->key != y->key) return x->key > y->key ? -1 : 1; /* larger |e| first */
  return x->col < y->col ? -1 : (x->col > y->col);       /* then lower column */
}

static int orc_col_order(const void* a, const void* b) {
  const orc_outlier_cand* x = (const orc_outlier_cand*)a;
  const orc_outlier_cand* y = (const orc_outlier_cand*)b;
  return x->col < y->col ? -1 : (x->col > y->col);
}

/* ocols, ovals: [rows][k].  Returns 2 on a bad shape (cols > 65536, k > cols). */
int orc_outliers_select(const void* W, int dtype, const float* What, int64_t rows, int64_t cols, int64_t k,
                        uint16_t* ocols, uint16_t* ovals) {
  if (rows < 0 || cols < 1 || cols > 65536 || k < 0 || k > cols) return 2;
  if (k == 0) return 0;
  #pragma omp parallel
  {
    orc_outlier_cand* c = (orc_outlier_cand*)malloc(sizeof(orc_outlier_cand) * (size_t)cols);
    #pragma omp for schedule(dynamic, 16)
    for (int64_t i = 0; i < rows; i++) {
      for (int64_t j = 0; j < cols; j++) {
        double e = (double)load_w(W, dtype, i * cols + j) - (double)What[i * cols + j];
        double a = fabs(e);
        uint64_t bits;
        memcpy(&bits, &a, sizeof bits);
        c[j].key = bits;
        c[j].col = j;
      }
      qsort(c, (size_t)cols, sizeof *c, orc_outlier_rank);
      qsort(c, (size_t)k, sizeof *c, orc_col_order);
      for (int64_t q = 0; q < k; q++) {
        int64_t j = c[q].col;
        double e = (double)load_w(W, dtype, i * cols + j) - (double)What[i * cols + j];
        ocols[i * k + q] = (uint16_t)j;
        ovals[i * k + q] = fp16_from_double(e, 1);
      }
    }
    free(c);
  }
  return 0;
}

/* What[i][col] += (float)o for each stored outlier, in binary32. */
int orc_outliers_apply(float* What, int64_t rows, int64_t cols, int64_t k, const uint16_t* ocols,
                       const uint16_t* ovals) {
  if (rows < 0 || cols < 1 || k < 0 || k > cols) return 2;
  for (int64_t i = 0; i < rows; i++)
    for (int64_t q = 0; q < k; q++) {
      int64_t j = ocols[i * k + q];
      if (j >= cols) return 3;
      float o = (float)orc_fp16_to_double(ovals[i * k + q]);
      What[i * cols + j] = What[i * cols + j] + o;
    }
  return 0;
}
