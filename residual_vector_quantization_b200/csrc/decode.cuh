// VQ3R decode and the relative-Frobenius error reduction.
//
// Page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验", §2: the
// reconstruction W ~ scale x (C1[i1] + C2[i2] + C3[i3]); §3.1: the relative
// Frobenius error ||W - W_hat||_F / ||W||_F of the Gate 3 table; §4: the
// container is dequantised and compared record by record with the source.
//
// Both kernels are HBM-bound.  Decode reads 0.375 B/weight of indices plus
// the row scales and writes 4 (fp32) or 2 (fp16) B/weight.  The error
// kernel reads the original weights (2 or 4 B/weight) and the indices,
// decodes in registers and keeps two binary64 sums.
#pragma once

#include "vq3r_common.cuh"

namespace vq3r {

constexpr int kDecThreads = 256;

// Codebooks staged in shared memory (plain loads: 24 KiB, once per CTA).
__device__ __forceinline__ void load_codebooks_smem(float* cb, const float* __restrict__ codebooks) {
  const float4* src = reinterpret_cast<const float4*>(codebooks);
  float4* dst = reinterpret_cast<float4*>(cb);
  for (int i = threadIdx.x; i < kCodebookFloats / 4; i += blockDim.x) dst[i] = __ldg(src + i);
  __syncthreads();
}

// w_hat of one vector: (float)scale * ((C1 + C2) + C3), each operation rounded.
__device__ __forceinline__ void decode_vector(const float* cb, uint32_t i1, uint32_t i2, uint32_t i3, float s,
                                              float out[8]) {
  const float4* c1 = reinterpret_cast<const float4*>(cb + (0 * kCodewords + i1) * kDim);
  const float4* c2 = reinterpret_cast<const float4*>(cb + (1 * kCodewords + i2) * kDim);
  const float4* c3 = reinterpret_cast<const float4*>(cb + (2 * kCodewords + i3) * kDim);
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const float4 a = c1[h], b = c2[h], c = c3[h];
    out[4 * h + 0] = __fmul_rn(s, __fadd_rn(__fadd_rn(a.x, b.x), c.x));
    out[4 * h + 1] = __fmul_rn(s, __fadd_rn(__fadd_rn(a.y, b.y), c.y));
    out[4 * h + 2] = __fmul_rn(s, __fadd_rn(__fadd_rn(a.z, b.z), c.z));
    out[4 * h + 3] = __fmul_rn(s, __fadd_rn(__fadd_rn(a.w, b.w), c.w));
  }
}

template <int OUT_DT>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const uint8_t* __restrict__ idx,
                                                              const uint16_t* __restrict__ scales,
                                                              const float* __restrict__ codebooks, int64_t cols,
                                                              int64_t nvec, void* __restrict__ out) {
  __shared__ __align__(16) float cb[kCodebookFloats];
  load_codebooks_smem(cb, codebooks);
  const int64_t V = cols / kDim;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nvec; g += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t i1 = __ldcs(idx + g), i2 = __ldcs(idx + nvec + g), i3 = __ldcs(idx + 2 * nvec + g);
    const int64_t row = g / V;
    const float s = f16_bits_to_f32(__ldg(scales + row));
    float w[8];
    decode_vector(cb, i1, i2, i3, s, w);
    if constexpr (OUT_DT == VQ3R_F32) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + g * kDim);
      __stcs(o, make_float4(w[0], w[1], w[2], w[3]));
      __stcs(o + 1, make_float4(w[4], w[5], w[6], w[7]));
    } else {
      uint32_t u[4];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const uint32_t lo = __half_as_ushort(__float2half_rn(w[2 * i]));
        const uint32_t hi = __half_as_ushort(__float2half_rn(w[2 * i + 1]));
        u[i] = lo | (hi << 16);
      }
      __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + g * kDim), make_uint4(u[0], u[1], u[2], u[3]));
    }
  }
}

// ---- relative Frobenius error: per-CTA binary64 partials, then one CTA ----

constexpr int kErrThreads = 256;

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, o);
  return v;
}

template <int DT>
__global__ void __launch_bounds__(kErrThreads) relfro_partial_kernel(const void* __restrict__ W,
                                                                      const uint8_t* __restrict__ idx,
                                                                      const uint16_t* __restrict__ scales,
                                                                      const float* __restrict__ codebooks,
                                                                      int64_t cols, int64_t nvec,
                                                                      double* __restrict__ partial) {
  __shared__ __align__(16) float cb[kCodebookFloats];
  __shared__ double red[2][kErrThreads / 32];
  load_codebooks_smem(cb, codebooks);
  const int64_t V = cols / kDim;
  double num = 0.0, den = 0.0;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nvec; g += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t i1 = __ldcs(idx + g), i2 = __ldcs(idx + nvec + g), i3 = __ldcs(idx + 2 * nvec + g);
    const int64_t row = g / V;
    const float s = f16_bits_to_f32(__ldg(scales + row));
    float wh[8], w[8];
    decode_vector(cb, i1, i2, i3, s, wh);
    load8<DT>(W, g * kDim, w);
#pragma unroll
    for (int k = 0; k < 8; k++) {
      const double e = (double)w[k] - (double)wh[k];
      num = fma(e, e, num);
      den = fma((double)w[k], (double)w[k], den);
    }
  }
  num = warp_sum_f64(num);
  den = warp_sum_f64(den);
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { red[0][wid] = num; red[1][wid] = den; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0;
    for (int i = 0; i < kErrThreads / 32; i++) { a += red[0][i]; b += red[1][i]; }
    partial[2 * blockIdx.x] = a;
    partial[2 * blockIdx.x + 1] = b;
  }
}

__global__ void __launch_bounds__(256) relfro_final_kernel(const double* __restrict__ partial, int n,
                                                            double* __restrict__ err_out) {
  __shared__ double red[2][8];
  double a = 0.0, b = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) { a += partial[2 * i]; b += partial[2 * i + 1]; }
  a = warp_sum_f64(a);
  b = warp_sum_f64(b);
  if ((threadIdx.x & 31) == 0) { red[0][threadIdx.x >> 5] = a; red[1][threadIdx.x >> 5] = b; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double x = 0.0, y = 0.0;
    for (int i = 0; i < 8; i++) { x += red[0][i]; y += red[1][i]; }
    *err_out = sqrt(x / y);
  }
}

}  // namespace vq3r
