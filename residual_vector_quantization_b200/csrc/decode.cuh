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

constexpr int kDecThreads = 512;

template <int FMT>
__host__ __device__ constexpr int fmt_codewords_total() {
  return FMT == FMT_VQ4P ? 4 * 64 : kStages * kCodewords;
}

// Codebooks for gathers by 32 lanes: every codeword stored four times side by
// side in a 128-byte row, cbr[row][copy][8] with row = stage * K + j.  Lane L
// reads copy (L >> 1) & 3, half L & 1, so the eight lanes of a quarter-warp
// hit eight distinct 16-byte bank groups whatever the indices are.  96 KiB
// for VQ3R, 32 KiB for VQ4P.
template <int FMT>
__host__ __device__ constexpr int fmt_cbr_floats() {
  return fmt_codewords_total<FMT>() * 4 * kDim;
}
constexpr int kCbrFloats = fmt_cbr_floats<FMT_VQ3R>();
template <int FMT>
__device__ __forceinline__ void load_codebooks_replicated(float* cbr, const float* __restrict__ codebooks) {
  const float4* src = reinterpret_cast<const float4*>(codebooks);
  float4* dst = reinterpret_cast<float4*>(cbr);
  for (int i = threadIdx.x; i < fmt_codewords_total<FMT>() * kDim / 4; i += blockDim.x) {  // i: half of codeword i >> 1
    const float4 v = __ldg(src + i);
#pragma unroll
    for (int c = 0; c < 4; c++) dst[((i >> 1) * 4 + c) * 2 + (i & 1)] = v;
  }
  __syncthreads();
}

// Codebook rows of a vector from its three plane bytes e0, e1, e2.
template <int FMT>
__device__ __forceinline__ void fmt_rows(uint32_t e0, uint32_t e1, uint32_t e2, uint32_t r[4]) {
  if constexpr (FMT == FMT_VQ4P) {
    const uint32_t w = e0 | (e1 << 8) | (e2 << 16);
    r[0] = w & 63u;
    r[1] = 64u + ((w >> 6) & 63u);
    r[2] = 128u + ((w >> 12) & 63u);
    r[3] = 192u + (w >> 18);
  } else {
    r[0] = e0;
    r[1] = kCodewords + e1;
    r[2] = 2 * kCodewords + e2;
    r[3] = 0;
  }
}

// scale * (sum of the stage codewords, added in stage order), each operation rounded.
template <int FMT>
__device__ __forceinline__ float4 combine4(float s, const float4& a, const float4& b, const float4& c, const float4& d) {
  if constexpr (FMT == FMT_VQ4P) {
    return make_float4(__fmul_rn(s, __fadd_rn(__fadd_rn(__fadd_rn(a.x, b.x), c.x), d.x)),
                       __fmul_rn(s, __fadd_rn(__fadd_rn(__fadd_rn(a.y, b.y), c.y), d.y)),
                       __fmul_rn(s, __fadd_rn(__fadd_rn(__fadd_rn(a.z, b.z), c.z), d.z)),
                       __fmul_rn(s, __fadd_rn(__fadd_rn(__fadd_rn(a.w, b.w), c.w), d.w)));
  } else {
    return make_float4(__fmul_rn(s, __fadd_rn(__fadd_rn(a.x, b.x), c.x)), __fmul_rn(s, __fadd_rn(__fadd_rn(a.y, b.y), c.y)),
                       __fmul_rn(s, __fadd_rn(__fadd_rn(a.z, b.z), c.z)), __fmul_rn(s, __fadd_rn(__fadd_rn(a.w, b.w), c.w)));
  }
}

// Half h = L & 1 (elements 4h .. 4h + 3) of w_hat for one vector:
// (float)scale * ((C1 + C2) + C3) (VQ3R) or (((C1 + C2) + C3) + C4) (VQ4P),
// each operation rounded.
template <int FMT>
__device__ __forceinline__ float4 decode_half_r(const float* cbr, uint32_t e0, uint32_t e1, uint32_t e2, float s,
                                                int lane) {
  const int off = ((lane >> 1) & 3) * kDim + 4 * (lane & 1);
  uint32_t r[4];
  fmt_rows<FMT>(e0, e1, e2, r);
  const float4 a = *reinterpret_cast<const float4*>(cbr + r[0] * 4 * kDim + off);
  const float4 b = *reinterpret_cast<const float4*>(cbr + r[1] * 4 * kDim + off);
  const float4 c = *reinterpret_cast<const float4*>(cbr + r[2] * 4 * kDim + off);
  float4 d = make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (FMT == FMT_VQ4P) d = *reinterpret_cast<const float4*>(cbr + r[3] * 4 * kDim + off);
  return combine4<FMT>(s, a, b, c, d);
}

// Traversal shared by decode and the error kernel.  Rows are split evenly over
// the CTAs.  Two lanes take one vector (lane parity = half), so a warp covers
// 16 consecutive vectors and its 16-byte stores form one 512-byte span.  The
// CTA's threads / 2 vectors per step walk its rows in order; (row, v) advance
// by that many vectors per step with no division.
struct RowWalk {
  int64_t row, v;     // current vector of this thread
  int64_t V, dq, dr;  // vectors per row; step = dq * V + dr
  __device__ __forceinline__ void init(int64_t r0, int64_t V_, int tid, int threads) {
    V = V_;
    const int64_t step = threads / 2, v0 = tid >> 1;
    row = r0 + v0 / V;
    v = v0 - (v0 / V) * V;
    dq = step / V;
    dr = step - dq * V;
  }
  __device__ __forceinline__ void next() {
    row += dq;
    v += dr;
    if (v >= V) {
      v -= V;
      row++;
    }
  }
};

constexpr int kWalkUnroll = 4;  // walk positions per thread whose loads are issued together

// The next kWalkUnroll positions of a walk (rows at or past r1 are marked
// invalid) with their index bytes and row scales, all loads issued before use.
struct WalkBatch {
  int64_t g[kWalkUnroll];
  uint32_t e[kWalkUnroll][3];
  float s[kWalkUnroll];
  bool ok[kWalkUnroll];
};
__device__ __forceinline__ bool walk_batch(RowWalk& it, int64_t r1, const uint8_t* __restrict__ idx, int64_t nvec,
                                           const uint16_t* __restrict__ scales, WalkBatch& wb) {
  if (it.row >= r1) return false;
#pragma unroll
  for (int u = 0; u < kWalkUnroll; u++) {
    wb.ok[u] = it.row < r1;
    const int64_t row = wb.ok[u] ? it.row : r1 - 1, v = wb.ok[u] ? it.v : 0;  // clamped: always a valid address
    wb.g[u] = row * it.V + v;
    wb.e[u][0] = __ldcs(idx + wb.g[u]);
    wb.e[u][1] = __ldcs(idx + nvec + wb.g[u]);
    wb.e[u][2] = __ldcs(idx + 2 * nvec + wb.g[u]);
    wb.s[u] = f16_bits_to_f32(__ldg(scales + row));
    it.next();
  }
  return true;
}

template <int OUT_DT, int FMT>
__global__ void __launch_bounds__(kDecThreads, 2) decode_kernel(const uint8_t* __restrict__ idx,
                                                                 const uint16_t* __restrict__ scales,
                                                                 const float* __restrict__ codebooks, int64_t rows,
                                                                 int64_t cols, void* __restrict__ out) {
  extern __shared__ __align__(16) float cbr[];
  load_codebooks_replicated<FMT>(cbr, codebooks);
  const int lane = threadIdx.x & 31, h = lane & 1;
  const int64_t V = cols / kDim, nvec = rows * V;
  const int64_t r0 = (int64_t)blockIdx.x * rows / gridDim.x, r1 = (int64_t)(blockIdx.x + 1) * rows / gridDim.x;
  RowWalk it;
  it.init(r0, V, threadIdx.x, kDecThreads);
  WalkBatch wb;
  while (walk_batch(it, r1, idx, nvec, scales, wb)) {
#pragma unroll
    for (int u = 0; u < kWalkUnroll; u++) {
      if (!wb.ok[u]) continue;
      const int64_t g = wb.g[u];
      const float4 o = decode_half_r<FMT>(cbr, wb.e[u][0], wb.e[u][1], wb.e[u][2], wb.s[u], lane);
      if constexpr (OUT_DT == VQ3R_F32) {
        __stcs(reinterpret_cast<float4*>(static_cast<float*>(out) + g * kDim + 4 * h), o);
      } else {
        const uint32_t u0 = (uint32_t)__half_as_ushort(__float2half_rn(o.x)) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(o.y)) << 16);
        const uint32_t u1 = (uint32_t)__half_as_ushort(__float2half_rn(o.z)) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(o.w)) << 16);
        __stcs(reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + g * kDim + 4 * h), make_uint2(u0, u1));
      }
    }
  }
}

// Decode with the index bytes staged per tile: a CTA takes tiles of
// kDecTileV consecutive vectors (t = blockIdx.x, + gridDim.x, ...); thread 0
// copies a tile's three index planes into shared memory with bulk
// asynchronous copies (no multicast), two tiles in flight, and the threads
// decode from there.  Plane p of a tile starts at idx + p * nvec + t *
// kDecTileV: the host uses this kernel when nvec is a multiple of 16, so
// every copy starts on a 16-byte boundary and moves a multiple of 16 bytes.
constexpr int kDecTileV = 2048;
template <int FMT>
__host__ __device__ constexpr size_t decode_bulk_smem() {
  return fmt_cbr_floats<FMT>() * sizeof(float) + 2 * 3 * kDecTileV;
}

template <int OUT_DT, int FMT>
__global__ void __launch_bounds__(kDecThreads, 2) decode_bulk_kernel(const uint8_t* __restrict__ idx,
                                                                      const uint16_t* __restrict__ scales,
                                                                      const float* __restrict__ codebooks,
                                                                      int64_t rows, int64_t cols,
                                                                      void* __restrict__ out) {
  extern __shared__ __align__(16) float cbr[];
  uint8_t* const tiles = reinterpret_cast<uint8_t*>(cbr + fmt_cbr_floats<FMT>());  // [2][3][kDecTileV]
  __shared__ uint64_t mbar[2];
  const int tid = threadIdx.x, lane = tid & 31, h = lane & 1;
  const int64_t V = cols / kDim, nvec = rows * V;
  const int64_t ntiles = (nvec + kDecTileV - 1) / kDecTileV;
  auto issue = [&](int64_t t, int b) {  // thread 0: tile t into buffer b
    const int64_t g0 = t * kDecTileV;
    const uint32_t n = (uint32_t)(nvec - g0 < kDecTileV ? nvec - g0 : kDecTileV);
    mbar_arrive_expect_tx(&mbar[b], 3 * n);
#pragma unroll
    for (int p = 0; p < 3; p++) bulk_copy_g2s(tiles + (b * 3 + p) * kDecTileV, idx + p * nvec + g0, n, &mbar[b]);
  };
  if (tid == 0) {
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
    if (blockIdx.x < ntiles) issue(blockIdx.x, 0);
    if (blockIdx.x + gridDim.x < ntiles) issue(blockIdx.x + gridDim.x, 1);
  }
  load_codebooks_replicated<FMT>(cbr, codebooks);  // ends with a barrier: the barriers are initialised too
  const int64_t step = kDecThreads / 2, dq = step / V, dr = step - dq * V;
  bool ok = true;
  int it = 0;
  for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, it++) {
    const int b = it & 1;
    ok = mbar_wait_bounded(&mbar[b], (uint32_t)(it >> 1) & 1u) && ok;
    const int64_t g0 = t * kDecTileV;
    const int n = (int)(nvec - g0 < kDecTileV ? nvec - g0 : kDecTileV);
    const uint8_t* tp = tiles + b * 3 * kDecTileV;
    int64_t row = (g0 + (tid >> 1)) / V, v = g0 + (tid >> 1) - row * V;
    for (int j = tid >> 1; j < n; j += (int)step) {
      const float s = f16_bits_to_f32(__ldg(scales + row));
      const float4 o = decode_half_r<FMT>(cbr, tp[j], tp[kDecTileV + j], tp[2 * kDecTileV + j], s, lane);
      const int64_t g = g0 + j;
      if constexpr (OUT_DT == VQ3R_F32) {
        __stcs(reinterpret_cast<float4*>(static_cast<float*>(out) + g * kDim + 4 * h), o);
      } else {
        const uint32_t u0 = (uint32_t)__half_as_ushort(__float2half_rn(o.x)) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(o.y)) << 16);
        const uint32_t u1 = (uint32_t)__half_as_ushort(__float2half_rn(o.z)) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(o.w)) << 16);
        __stcs(reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + g * kDim + 4 * h), make_uint2(u0, u1));
      }
      row += dq;
      v += dr;
      if (v >= V) {
        v -= V;
        row++;
      }
    }
    __syncthreads();  // every thread is done with buffer b
    if (tid == 0 && t + 2 * (int64_t)gridDim.x < ntiles) {
      fence_proxy_async_smem();  // generic reads of the buffer precede its async refill
      issue(t + 2 * (int64_t)gridDim.x, b);
    }
  }
  (void)ok;  // a timed-out wait has recorded the device error word
}

// ---- relative Frobenius error: per-CTA binary64 partials, then one CTA ----

constexpr int kErrThreads = 512;

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Whole w_hat vector for one lane: both halves, the lane's copy of each
// codeword, half L & 1 first (conflict-free order for a quarter-warp).
template <int FMT>
__device__ __forceinline__ void decode_vector_r(const float* cbr, uint32_t e0, uint32_t e1, uint32_t e2, float s,
                                                int lane, float4& lo, float4& hi) {
  const int copy = (lane >> 1) & 3, h0 = lane & 1;
  uint32_t r[4];
  fmt_rows<FMT>(e0, e1, e2, r);
  const float4* c1 = reinterpret_cast<const float4*>(cbr + (r[0] * 4 + copy) * kDim);
  const float4* c2 = reinterpret_cast<const float4*>(cbr + (r[1] * 4 + copy) * kDim);
  const float4* c3 = reinterpret_cast<const float4*>(cbr + (r[2] * 4 + copy) * kDim);
  const float4* c4 = reinterpret_cast<const float4*>(cbr + (r[3] * 4 + copy) * kDim);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 first = combine4<FMT>(s, c1[h0], c2[h0], c3[h0], FMT == FMT_VQ4P ? c4[h0] : z);
  const float4 second = combine4<FMT>(s, c1[h0 ^ 1], c2[h0 ^ 1], c3[h0 ^ 1], FMT == FMT_VQ4P ? c4[h0 ^ 1] : z);
  lo = h0 ? second : first;
  hi = h0 ? first : second;
}

__device__ __forceinline__ void acc_err(double& num, double& den, float w, float wh) {
  const double e = (double)w - (double)wh;
  num = fma(e, e, num);
  den = fma((double)w, (double)w, den);
}

constexpr int kErrVecs = 4;  // consecutive vectors per thread and step

// Rows are split evenly over the CTAs.  A CTA numbers the 4-vector groups of
// its rows consecutively (row-major, at most 2^31 of them) and thread t takes
// groups t, t + 512, ...: the index bytes of a group are one 32-bit word per
// plane when V is a multiple of 4, and a warp's 16-byte W loads are 512
// contiguous bytes.  Each thread keeps two binary64 sums, reduced per CTA.
//
// OUT: the decode carries a sparse outlier residual (ocols / ovals [rows][k],
// columns ascending per row): each outlier's (float)o is added to its
// decoded value in binary32 before the sums, so the numerator is summed
// directly.  A thread finds the first outlier of its 32 columns by binary
// search in the row's columns.
template <int DT, int FMT, bool OUT = false>
__global__ void __launch_bounds__(kErrThreads, 2) relfro_partial_kernel(const void* __restrict__ W,
                                                                         const uint8_t* __restrict__ idx,
                                                                         const uint16_t* __restrict__ scales,
                                                                         const float* __restrict__ codebooks,
                                                                         int64_t rows, int64_t cols,
                                                                         double* __restrict__ partial,
                                                                         const uint16_t* __restrict__ ocols = nullptr,
                                                                         const uint16_t* __restrict__ ovals = nullptr,
                                                                         int k = 0) {
  extern __shared__ __align__(16) float cbr[];
  __shared__ double red[2][kErrThreads / 32];
  load_codebooks_replicated<FMT>(cbr, codebooks);
  const int lane = threadIdx.x & 31;
  const int64_t V = cols / kDim, nvec = rows * V;
  const uint32_t gpr = (uint32_t)((V + kErrVecs - 1) / kErrVecs);  // groups per row
  const bool vec4 = (V % kErrVecs) == 0;
  const int64_t r0 = (int64_t)blockIdx.x * rows / gridDim.x, r1 = (int64_t)(blockIdx.x + 1) * rows / gridDim.x;
  const uint32_t nf = (uint32_t)((r1 - r0) * gpr);
  double num = 0.0, den = 0.0;
  for (uint32_t f = threadIdx.x; f < nf; f += kErrThreads) {
    const uint32_t rl = f / gpr, q = f - rl * gpr;
    const int64_t row = r0 + rl;
    const int64_t g = row * V + (int64_t)q * kErrVecs;
    const int n = (int)((V - (int64_t)q * kErrVecs) < kErrVecs ? (V - (int64_t)q * kErrVecs) : kErrVecs);
    const float s = f16_bits_to_f32(__ldg(scales + row));
    uint32_t w3[3];
#pragma unroll
    for (int st = 0; st < kStages; st++) {
      if (vec4) {
        w3[st] = __ldcs(reinterpret_cast<const unsigned int*>(idx + st * nvec + g));
      } else {
        uint32_t x = 0;
        for (int i = 0; i < n; i++) x |= (uint32_t)__ldcs(idx + st * nvec + g + i) << (8 * i);
        w3[st] = x;
      }
    }
    int oq = 0;  // OUT: first outlier of the row at or after this group's first column
    const uint16_t* orow = nullptr;
    if constexpr (OUT) {
      orow = ocols + row * k;
      const int c_lo = q * kErrVecs * kDim;
      int lo = 0, hi = k;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((int)__ldg(orow + mid) < c_lo) lo = mid + 1;
        else hi = mid;
      }
      oq = lo;
    }
#pragma unroll
    for (int i = 0; i < kErrVecs; i++) {
      if (i < n) {
        float4 lo, hi;
        decode_vector_r<FMT>(cbr, (w3[0] >> (8 * i)) & 0xFFu, (w3[1] >> (8 * i)) & 0xFFu, (w3[2] >> (8 * i)) & 0xFFu, s, lane,
                        lo, hi);
        float wh[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        if constexpr (OUT) {
          const int cv = (q * kErrVecs + i) * kDim;
          while (oq < k) {
            const int c = (int)__ldg(orow + oq);
            if (c >= cv + kDim) break;
            const float o = f16_bits_to_f32(__ldg(ovals + row * k + oq));
#pragma unroll
            for (int j = 0; j < kDim; j++)
              if (c == cv + j) wh[j] = __fadd_rn(wh[j], o);
            oq++;
          }
        }
        float wv[8];
        load8<DT>(W, (g + i) * kDim, wv);
#pragma unroll
        for (int j = 0; j < kDim; j++) acc_err(num, den, wv[j], wh[j]);
      }
    }
  }
  num = warp_sum_f64(num);
  den = warp_sum_f64(den);
  const int wid = threadIdx.x >> 5;
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
