// VQ3R encoder: per-row FP16 scale and greedy 3-stage residual assignment.
//
// Page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验", §2: one FP16
// scale per row; three stages of 256-entry codebooks of 8-dim vectors; stage
// s quantises the residual left by stage s-1.  §4: a single pass over the
// three stages that writes only the winning indices.
//
// The work is FP32-pipe bound: per 8-weight vector and stage, 256 codewords.
// The definition's distance d_j = sum_k (r_k - c_jk)^2 has every operation
// rounded in k order (no fused multiply-add); the kernel screens all
// codewords with a cheaper fused form and a proven error margin, and takes
// the definition's arithmetic only where the margin cannot separate the best
// two (K2 below), so the indices are bit-identical to the definition.
// Packed f32x2 instructions evaluate two vectors per instruction.
#pragma once

#include "vq3r_common.cuh"

namespace vq3r {

// ---------------- K1: row scale ----------------
//
// scale_i = binary16(sqrt(ss_i / cols)) with ss_i in binary64 in the fixed
// order: thread p (of 128) sums q_v = ((w0^2 + w1^2) + ...) + w7^2 over
// v = p, p+128, ... ascending; then a halving tree t_p += t_{p+h},
// h = 64 .. 1.  __dmul_rn / __dadd_rn keep every product and sum rounded
// separately.
constexpr int kScaleThreads = 128;

template <int DT>
__global__ void __launch_bounds__(kScaleThreads) row_scale_kernel(const void* __restrict__ W, int64_t rows,
                                                                   int64_t cols, uint16_t* __restrict__ scales) {
  __shared__ double t[kScaleThreads];
  const int p = threadIdx.x;
  const int64_t V = cols / kDim;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    double acc = 0.0;
    for (int64_t v = p; v < V; v += kScaleThreads) {
      float w[8];
      load8<DT>(W, row * cols + v * kDim, w);
      double q = __dmul_rn((double)w[0], (double)w[0]);
#pragma unroll
      for (int k = 1; k < 8; k++) q = __dadd_rn(q, __dmul_rn((double)w[k], (double)w[k]));
      acc = __dadd_rn(acc, q);
    }
    t[p] = acc;
    __syncthreads();
#pragma unroll
    for (int h = 64; h >= 1; h >>= 1) {
      if (p < h) t[p] = __dadd_rn(t[p], t[p + h]);
      __syncthreads();
    }
    if (p == 0) {
      const double rms = __dsqrt_rn(__ddiv_rn(t[0], (double)cols));
      scales[row] = f64_to_f16_sat_rne(rms);
    }
    __syncthreads();
  }
}

// ---------------- K2: greedy 3-stage assignment ----------------
//
// Screen, then decide exactly.  For a residual r and codeword c let
//   D(c) = sum_k (r_k - c_k)^2            (real arithmetic),
//   d(c) = the definition's value: each subtraction, square and add rounded
//          to nearest binary32 in k order,
//   h(c) = ||c||^2 / 2 - r.c,  so  D(c) = ||r||^2 + 2 h(c).
// The screening value of c is L(c): the binary64 value (1/2 - 16u) ||c||^2
// rounded once to binary32, then fma(r_k, -c_k, acc) for k = 0..7, with
// u = 2^-24, R2 = ||r||^2, C(c) = ||c||^2.  Then:
//   (1) d has 10 roundings of non-negative terms: |d - D| <= 10.01 u D;
//   (2) every partial sum of L is at most C + R2/2 in magnitude and 9
//       roundings (start value included) touch it, so
//       |L(c) - (h(c) - 16u C(c))| <= 9.51 u C(c) + 4.51 u R2.
// Let j~ minimise L.  d(j) > d(j~) for every j != j~ (j~ is the unique
// winner) holds when h(j) - h(j~) > 10.02 u D(j~); with (2) and D(j~) = R2 +
// 2 h(j~) it suffices that, for every other j,
//   L(j) > L(j~) + 25.52 u C(j~) + 19.04 u R2 + 20.04 u |L(j~)|,
// which the kernel tests as  L2 - L1 > M = 2^-19 (C(j~) + R2 + |L1|) + 2^-126
// with L1 <= L2 the two smallest screening values (R2 computed with fused
// multiply-adds, relative error below 8.01 u, covered by the factor 32 u;
// 2^-126 covers subnormal rounding; M >= 2^100 is refused, which excludes
// overflow).  A vector that fails the test (near ties, exact ties, non-finite
// values) is re-scanned with the definition's arithmetic over all codewords,
// so the indices are bit-identical to the definition in every case.  The
// screen costs 8 fused multiply-adds and a few compares per codeword instead
// of 24 rounded operations; on trained codebooks about 1 vector-stage in
// 10^4 is re-scanned.

constexpr int kEncThreads = 256;
// Vector pairs per thread: 3 for VQ3R (2 measured 4.9% slower), 2 for VQ4P
// (whose packed index words leave no registers for a third pair).
template <int FMT>
__host__ __device__ constexpr int enc_pairs() {
  return FMT == FMT_VQ4P ? 2 : 3;
}
template <int FMT>
__host__ __device__ constexpr int enc_tile() {  // vectors per CTA iteration
  return kEncThreads * 2 * enc_pairs<FMT>();
}

struct __align__(16) EncSmem {
  float2 ncb[kStages][kCodewords][kDim];  // (-c, -c) duplicated for the packed operations (48 KiB)
  float2 nch[kStages][kCodewords];        // screening start values (1/2 - 16u) ||c||^2, duplicated (6 KiB)
  float c2[kStages][kCodewords];          // ||c||^2 rounded up (3 KiB)
  float raw[kCodebookFloats];              // TMA staging of the caller's codebooks (24 KiB)
  uint64_t mbar;
};

// Paired binary32 arithmetic for the distances, d = sum_k (r_k - c_k)^2 with
// every operation rounded to nearest even (no fused multiply-add).  A paired
// multiply followed by a paired add is contracted into a fused multiply-add
// even when both carry an explicit rounding modifier (measured: a vector
// whose two best codewords tie under the definition came out with the higher
// index ahead).  So each square is a paired fused multiply-add whose addend
// is a zero the compiler cannot see (a kernel argument): fma(e, e, +0) rounds
// e * e once, exactly like a rounded multiply, and a fused multiply-add's
// result cannot be fused into the add that follows.
__device__ __forceinline__ float2 f2add(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// e * e rounded once (z holds +0 in both lanes).
__device__ __forceinline__ float2 f2sq(float2 e, float2 z) {
  float2 d;
  asm("{\n\t.reg .b64 re, rz, rd;\n\t"
      "mov.b64 re, {%2, %3};\n\t"
      "mov.b64 rz, {%4, %5};\n\t"
      "fma.rn.f32x2 rd, re, re, rz;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(e.x), "f"(e.y), "f"(z.x), "f"(z.y));
  return d;
}
// a * b + c, paired, one rounding each (the screening arithmetic).
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// Running smallest screening value (best, its codeword bi; strict <, so the
// lowest index keeps a tie) and second smallest (second).
__device__ __forceinline__ void screen_update(float h, int j, float& best, float& second, int& bi) {
  second = fminf(second, fmaxf(best, h));
  const bool lt = h < best;
  bi = lt ? j : bi;
  best = lt ? h : best;
}

// The definition's argmin over the K codewords of stage cw for the vector pair r
// (both lanes), lowest index on ties.
template <int K>
__device__ __forceinline__ void exact_scan(const float2 (&r)[kDim], const float4* cw, float2 z2, int& b0, int& b1) {
  float best0 = __int_as_float(0x7F800000), best1 = __int_as_float(0x7F800000);
  b0 = 0;
  b1 = 0;
#pragma unroll 2
  for (int j = 0; j < K; j++) {
    float2 c[kDim];
#pragma unroll
    for (int k2 = 0; k2 < 4; k2++) {
      const float4 t = cw[j * 4 + k2];
      c[2 * k2] = make_float2(t.x, t.y);
      c[2 * k2 + 1] = make_float2(t.z, t.w);
    }
    float2 e = f2add(r[0], c[0]);
    float2 d = f2sq(e, z2);
#pragma unroll
    for (int k = 1; k < kDim; k++) {
      e = f2add(r[k], c[k]);
      d = f2add(d, f2sq(e, z2));
    }
    if (d.x < best0) { best0 = d.x; b0 = j; }
    if (d.y < best1) { best1 = d.y; b1 = j; }
  }
}

// FMT 0 (VQ3R): 3 stages x 256 codewords, index byte of stage s in plane s.
// FMT 1 (VQ4P, page §5): 4 stages x 64 codewords, the 6-bit indices packed
// into the 24-bit word i1 | i2 << 6 | i3 << 12 | i4 << 18, byte p in plane p.
template <int DT, int FMT>
__global__ void __launch_bounds__(kEncThreads, 2)
    encode_kernel(const void* __restrict__ W, int64_t cols, int64_t nvec, const float* __restrict__ codebooks,
                  const uint16_t* __restrict__ scales, uint8_t* __restrict__ idx, float zero) {
  constexpr int S = FMT ? 4 : kStages, K = FMT ? 64 : kCodewords;
  constexpr int kEncPairs = enc_pairs<FMT>(), kEncVecPerThread = 2 * kEncPairs, kEncTile = enc_tile<FMT>();
  constexpr int kFloats = S * K * kDim;  // the caller's codebooks: 24 KiB (VQ3R), 8 KiB (VQ4P)
  extern __shared__ __align__(16) unsigned char enc_smem_raw[];
  EncSmem& sm = *reinterpret_cast<EncSmem*>(enc_smem_raw);
  float2* const ncb = &sm.ncb[0][0][0];  // [S][K][8]
  float2* const nch = &sm.nch[0][0];     // [S][K]
  float* const c2 = &sm.c2[0][0];        // [S][K]
  const int tid = threadIdx.x;

  // Stage the codebooks with one bulk asynchronous copy, then expand to
  // negated, lane-duplicated pairs and the screening constants.
  if (tid == 0) {
    mbar_init(&sm.mbar, 1);
    mbar_arrive_expect_tx(&sm.mbar, kFloats * 4);
    bulk_copy_g2s(sm.raw, codebooks, kFloats * 4, &sm.mbar);
  }
  __syncthreads();
  if (!mbar_wait_bounded(&sm.mbar, 0)) return;
  for (int i = tid; i < kFloats; i += kEncThreads) {
    const float c = -sm.raw[i];
    ncb[i] = make_float2(c, c);
  }
  for (int j = tid; j < S * K; j += kEncThreads) {
    double n = 0.0;  // ||c||^2: each square exact in binary64
#pragma unroll
    for (int k = 0; k < kDim; k++) n += (double)sm.raw[j * kDim + k] * (double)sm.raw[j * kDim + k];
    const float h = __double2float_rn((0.5 - 0x1p-20) * n);
    nch[j] = make_float2(h, h);
    c2[j] = __double2float_ru(n);
  }
  __syncthreads();

  const int64_t V = cols / kDim;
  const int64_t ntiles = (nvec + kEncTile - 1) / kEncTile;
  const float2 z2 = make_float2(zero, zero);  // +0, unknown to the compiler
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    // Vector q of this thread: g = tile * kEncTile + q * kEncThreads + tid.
    float2 r[kEncPairs][kDim];
    int64_t g[kEncVecPerThread];
#pragma unroll
    for (int q = 0; q < kEncVecPerThread; q++) {
      g[q] = tile * kEncTile + (int64_t)q * kEncThreads + tid;
      float w[8];
      float rq[8];
      if (g[q] < nvec) {
        const int64_t row = g[q] / V;
        const int64_t v = g[q] - row * V;
        load8<DT>(W, row * cols + v * kDim, w);
        const float s = f16_bits_to_f32(scales[row]);
#pragma unroll
        for (int k = 0; k < 8; k++) rq[k] = (s == 0.0f) ? 0.0f : __fdiv_rn(w[k], s);
      } else {
#pragma unroll
        for (int k = 0; k < 8; k++) rq[k] = 0.0f;
      }
#pragma unroll
      for (int k = 0; k < 8; k++) {
        if (q & 1) r[q >> 1][k].y = rq[k];
        else r[q >> 1][k].x = rq[k];
      }
    }

    uint32_t word[kEncVecPerThread] = {};  // VQ4P: packed indices
#pragma unroll 1
    for (int s = 0; s < S; s++) {
      float best[kEncVecPerThread], second[kEncVecPerThread];
      int bi[kEncVecPerThread];
#pragma unroll
      for (int q = 0; q < kEncVecPerThread; q++) {
        best[q] = __int_as_float(0x7F800000);
        second[q] = __int_as_float(0x7F800000);
        bi[q] = 0;
      }
      const float4* cw = reinterpret_cast<const float4*>(ncb + (size_t)s * K * kDim);
      const float2* hs = nch + (size_t)s * K;
#pragma unroll 16  // measured against 4, 8 and 32: 16 is fastest
      for (int j = 0; j < K; j++) {
        // (-c_k, -c_k) for k = 0..7: four broadcast 16-byte shared loads
        float2 c[kDim];
#pragma unroll
        for (int k2 = 0; k2 < 4; k2++) {
          const float4 t = cw[j * 4 + k2];
          c[2 * k2] = make_float2(t.x, t.y);
          c[2 * k2 + 1] = make_float2(t.z, t.w);
        }
        const float2 h0 = hs[j];
#pragma unroll
        for (int pr = 0; pr < kEncPairs; pr++) {
          float2 h = f2fma(r[pr][0], c[0], h0);
#pragma unroll
          for (int k = 1; k < kDim; k++) h = f2fma(r[pr][k], c[k], h);
          screen_update(h.x, j, best[2 * pr], second[2 * pr], bi[2 * pr]);
          screen_update(h.y, j, best[2 * pr + 1], second[2 * pr + 1], bi[2 * pr + 1]);
        }
      }
      // accept the screened winners whose gap is provably above the margin; re-scan the rest exactly
      const float* c2s = c2 + (size_t)s * K;
#pragma unroll
      for (int pr = 0; pr < kEncPairs; pr++) {
        float2 r2 = f2fma(r[pr][0], r[pr][0], z2);
#pragma unroll
        for (int k = 1; k < kDim; k++) r2 = f2fma(r[pr][k], r[pr][k], r2);
        const int q0 = 2 * pr, q1 = 2 * pr + 1;
        const float m0 = fmaf(c2s[bi[q0]] + r2.x + fabsf(best[q0]), 0x1p-19f, 0x1p-126f);
        const float m1 = fmaf(c2s[bi[q1]] + r2.y + fabsf(best[q1]), 0x1p-19f, 0x1p-126f);
        const bool ok0 = (second[q0] - best[q0]) > m0 && m0 < 0x1p100f;
        const bool ok1 = (second[q1] - best[q1]) > m1 && m1 < 0x1p100f;
        if (!(ok0 && ok1)) {
          int e0, e1;
          exact_scan<K>(r[pr], cw, z2, e0, e1);
          if (!ok0) bi[q0] = e0;
          if (!ok1) bi[q1] = e1;
        }
      }
      // write the winning indices and update the residuals
#pragma unroll
      for (int q = 0; q < kEncVecPerThread; q++) {
        if constexpr (FMT == 0) {
          if (g[q] < nvec) idx[(int64_t)s * nvec + g[q]] = (uint8_t)bi[q];
        } else {
          word[q] |= (uint32_t)bi[q] << (6 * s);
        }
        const float2* cwin = ncb + ((size_t)s * K + bi[q]) * kDim;
#pragma unroll
        for (int k = 0; k < kDim; k++) {
          if (q & 1) r[q >> 1][k].y = __fadd_rn(r[q >> 1][k].y, cwin[k].x);
          else r[q >> 1][k].x = __fadd_rn(r[q >> 1][k].x, cwin[k].x);
        }
      }
    }
    if constexpr (FMT != 0) {  // the packed word's three bytes, one per plane
#pragma unroll
      for (int q = 0; q < kEncVecPerThread; q++) {
        if (g[q] < nvec) {
          idx[g[q]] = (uint8_t)(word[q] & 0xFFu);
          idx[nvec + g[q]] = (uint8_t)((word[q] >> 8) & 0xFFu);
          idx[2 * nvec + g[q]] = (uint8_t)(word[q] >> 16);
        }
      }
    }
  }
}

}  // namespace vq3r
