// Outlier-aware variant: a sparse FP16 residual on top of the VQ3R encoding.
//
// Page "XFP：质量目标驱动的自适应码本量化" (zingnex.cn/forum/thread/xfp-llm),
// 技术实现 / 权重分解: each weight matrix is split into a dense index tensor
// into learned codebooks and a sparse FP16 outlier residual kept at full
// precision, with an outlier budget.  The page fixes no rule; readings:
//   e = (double)w - (double)w_hat, w_hat the binary32 VQ3R decode;
//   per row, the k positions with the largest |e| (ordered by the binary64
//   bit pattern of |e|), ties to the lower column, are the outliers;
//   each stores its column (uint16) and fp16(e) (nearest even, saturating
//   at +-65504); a row's k entries are in ascending column order;
//   decode: w_hat + (float)o in binary32.
//
// Kernels:
//   outlier_select_kernel  one CTA per row: the row's e values in shared
//                          memory, an exact radix select of the k-th largest
//                          |e| (up to 8 passes of 8 bits over the 64-bit
//                          pattern, stopping once the bucket is decided),
//                          then a column-ordered compaction that takes every
//                          larger key and the lowest-column equal keys;
//   outlier_apply_kernel   adds the outliers onto a binary32 decode;
//   (the error with outliers is relfro_partial_kernel<DT, FMT, true>, which
//   adds the outliers to the decoded values before its sums);
//   outlier_gemv_kernel    y[b][i] += sum_q (float)o_iq * x[b][c_iq] over the
//                          matrices of a grouped call (after the dense GEMV).
#pragma once

#include "vq3r_common.cuh"

namespace vq3r {

constexpr int kOutThreads = 512;  // >= 256: one histogram bin per thread for the clearing
constexpr int64_t kOutMaxCols = 16384;  // a row's binary64 errors live in shared memory
constexpr int kOutGemvMaxMats = 32;

// Dynamic shared memory of the select kernel: plain codebooks, the row's e
// values, the digit histogram.
__host__ __device__ constexpr size_t outlier_select_smem(int64_t cols) {
  return (size_t)kCodebookBytes + (size_t)cols * sizeof(double) + 256 * sizeof(uint32_t);
}

// One element of the VQ3R decode: s * ((C1[i1][k] + C2[i2][k]) + C3[i3][k]), each operation rounded.
__device__ __forceinline__ float decode_elem(const float* cb, uint32_t i1, uint32_t i2, uint32_t i3, int k, float s) {
  const float a = cb[(0 * kCodewords + i1) * kDim + k];
  const float b = cb[(1 * kCodewords + i2) * kDim + k];
  const float c = cb[(2 * kCodewords + i3) * kDim + k];
  return __fmul_rn(s, __fadd_rn(__fadd_rn(a, b), c));
}

__device__ __forceinline__ uint64_t abs_key(double e) {
  return (uint64_t)__double_as_longlong(e) & 0x7FFFFFFFFFFFFFFFull;
}

template <int DT>
__global__ void __launch_bounds__(kOutThreads) outlier_select_kernel(const void* __restrict__ W,
                                                                      const uint8_t* __restrict__ idx,
                                                                      const uint16_t* __restrict__ scales,
                                                                      const float* __restrict__ codebooks,
                                                                      int64_t rows, int64_t cols, int k,
                                                                      uint16_t* __restrict__ ocols,
                                                                      uint16_t* __restrict__ ovals) {
  extern __shared__ __align__(16) unsigned char out_smem[];
  float* cb = reinterpret_cast<float*>(out_smem);
  double* ev = reinterpret_cast<double*>(out_smem + kCodebookBytes);
  uint32_t* hist = reinterpret_cast<uint32_t*>(out_smem + kCodebookBytes + (size_t)cols * sizeof(double));
  __shared__ uint32_t s_digit, s_remaining, s_whole;
  __shared__ uint32_t s_wsum[kOutThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kCodebookFloats; i += kOutThreads) cb[i] = __ldg(codebooks + i);
  __syncthreads();
  const int64_t V = cols / kDim, plane = rows * V;

  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    // (a) the row's errors e = (double)w - (double)w_hat; column 8v + q is kept at ev[q * V + v], so that
    // consecutive lanes (consecutive v) touch consecutive words in every phase
    const float s = f16_bits_to_f32(__ldg(scales + row));
    for (int64_t v = tid; v < V; v += kOutThreads) {
      const int64_t g = row * V + v;
      const uint32_t i1 = __ldg(idx + g), i2 = __ldg(idx + plane + g), i3 = __ldg(idx + 2 * plane + g);
      float w[8];
      load8<DT>(W, row * cols + v * kDim, w);
#pragma unroll
      for (int q = 0; q < kDim; q++) ev[q * V + v] = (double)w[q] - (double)decode_elem(cb, i1, i2, i3, q, s);
    }
    __syncthreads();

    // (b) the k-th largest key, 8 bits at a time from the top: after each
    // pass, prefix/mask select the bucket that holds it and `remaining` is how
    // many of that bucket's keys belong to the outliers.  Once the bucket is
    // taken whole the search stops (the compaction compares masked keys).
    uint64_t prefix = 0, mask = 0;
    uint32_t remaining = (uint32_t)k;
    for (int pass = 0; pass < 8; pass++) {
      const int shift = 56 - 8 * pass;
      if (tid < 256) hist[tid] = 0u;
      __syncthreads();
      for (int64_t c = tid; c < cols; c += kOutThreads) {
        const uint64_t key = abs_key(ev[c]);
        // most keys share the leading digits: one atomic per distinct digit of the warp
        const uint32_t d = (key & mask) == prefix ? (uint32_t)((key >> shift) & 255u) : 256u;
        const unsigned peers = __match_any_sync(__activemask(), d);
        if (d < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (uint32_t)__popc(peers));
      }
      __syncthreads();
      if (warp == 0) {
        // lane L holds bins 255 - 8L down to 248 - 8L; counts above a lane's bins: exclusive scan over lanes
        uint32_t tot = 0;
#pragma unroll
        for (int b = 0; b < 8; b++) tot += hist[255 - 8 * lane - b];
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += t;
        }
        const uint32_t above = incl - tot;
        if (above < remaining && remaining <= incl) {
          uint32_t cum = above;
          for (int b = 0; b < 8; b++) {
            const uint32_t h = hist[255 - 8 * lane - b];
            if (cum + h >= remaining) {
              s_digit = (uint32_t)(255 - 8 * lane - b);
              s_remaining = remaining - cum;
              s_whole = (remaining - cum == h) ? 1u : 0u;
              break;
            }
            cum += h;
          }
        }
      }
      __syncthreads();
      prefix |= (uint64_t)s_digit << shift;
      mask |= 255ull << shift;
      remaining = s_remaining;
      if (s_whole) break;  // uniform: every thread read the same value
    }
    const uint64_t T = prefix;  // compared with key & mask below
    const uint32_t need_eq = remaining;

    // (c) column-ordered compaction: position of a taken column = (# larger keys before it) + min(# equal keys
    // before it, need_eq); chunks of 8 columns per thread, 2048 per CTA step
    uint32_t gt_run = 0, eq_run = 0;
    for (int64_t base = 0; base < cols; base += 8 * kOutThreads) {
      const int64_t c0 = base + 8 * tid;
      uint32_t ngt = 0, neq = 0;
      const int64_t v0 = c0 / kDim;  // this thread's vector: columns c0 .. c0 + 7
#pragma unroll
      for (int j = 0; j < 8; j++) {
        if (c0 + j < cols) {
          const uint64_t key = abs_key(ev[j * V + v0]) & mask;
          ngt += key > T;
          neq += key == T;
        }
      }
      // block exclusive scan of (gt << 16 | eq); each count <= 8 * kOutThreads
      const uint32_t packed = (ngt << 16) | neq;
      uint32_t incl = packed;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += t;
      }
      if (lane == 31) s_wsum[warp] = incl;
      __syncthreads();
      uint32_t wbase = 0, total = 0;
#pragma unroll
      for (int w8 = 0; w8 < kOutThreads / 32; w8++) {
        const uint32_t x = s_wsum[w8];
        if (w8 < warp) wbase += x;
        total += x;
      }
      const uint32_t excl = wbase + incl - packed;
      uint32_t gt_before = gt_run + (excl >> 16), eq_before = eq_run + (excl & 0xFFFFu);
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const int64_t c = c0 + j;
        if (c < cols) {
          const double e = ev[j * V + v0];
          const uint64_t key = abs_key(e) & mask;
          bool take = false;
          uint32_t pos = 0;
          if (key > T) {
            take = true;
            pos = gt_before + (eq_before < need_eq ? eq_before : need_eq);
            gt_before++;
          } else if (key == T) {
            if (eq_before < need_eq) {
              take = true;
              pos = gt_before + eq_before;
            }
            eq_before++;
          }
          if (take) {
            ocols[row * k + pos] = (uint16_t)c;
            ovals[row * k + pos] = f64_to_f16_sat_rne(e);
          }
        }
      }
      gt_run += total >> 16;
      eq_run += total & 0xFFFFu;
      __syncthreads();  // s_wsum and (after the last chunk) ev are reused
    }
  }
}

// out[i][c] += (float)o for the k outliers of each row (binary32).
__global__ void __launch_bounds__(256) outlier_apply_kernel(float* __restrict__ out, int64_t rows, int64_t cols,
                                                            int64_t k, const uint16_t* __restrict__ ocols,
                                                            const uint16_t* __restrict__ ovals) {
  const int64_t n = rows * k;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = t / k;
    const int64_t c = __ldg(ocols + t);
    if (c < cols) out[i * cols + c] = __fadd_rn(out[i * cols + c], f16_bits_to_f32(__ldg(ovals + t)));
  }
}

// Matrices of a grouped sparse add, rows numbered consecutively across them.
struct OutGemvParams {
  const uint16_t* ocols[kOutGemvMaxMats];
  const uint16_t* ovals[kOutGemvMaxMats];
  const void* x[kOutGemvMaxMats];
  float* y[kOutGemvMaxMats];
  int64_t rows[kOutGemvMaxMats], k[kOutGemvMaxMats], cols[kOutGemvMaxMats];
  int64_t row_begin[kOutGemvMaxMats + 1];
  int n_mats, B;
};

// One thread per row: y[b][i] += sum_q (float)o_iq * x[b][c_iq] in binary32, q ascending.  The row's
// columns and values are loaded 8 at a time before any use, so their loads overlap.
template <int XDT>
__global__ void __launch_bounds__(256) outlier_gemv_kernel(const __grid_constant__ OutGemvParams P) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= P.row_begin[P.n_mats]) return;
  int m = 0;
  while (t >= P.row_begin[m + 1]) m++;
  const int64_t i = t - P.row_begin[m], k = P.k[m], cols = P.cols[m], rows = P.rows[m];
  const uint16_t* oc = P.ocols[m] + i * k;
  const uint16_t* ov = P.ovals[m] + i * k;
  const void* x = P.x[m];
  float* y = P.y[m];
  for (int b = 0; b < P.B; b++) {
    float acc = 0.0f;
    for (int64_t q0 = 0; q0 < k; q0 += 8) {
      uint32_t c8[8];
      float o8[8];
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const bool ok = q0 + u < k;
        c8[u] = ok ? (uint32_t)__ldg(oc + q0 + u) : 0u;
        o8[u] = ok ? f16_bits_to_f32(__ldg(ov + q0 + u)) : 0.0f;
      }
      float x8[8];
#pragma unroll
      for (int u = 0; u < 8; u++) x8[u] = (int64_t)c8[u] < cols ? load1<XDT>(x, (int64_t)b * cols + c8[u]) : 0.0f;
#pragma unroll
      for (int u = 0; u < 8; u++) acc = fmaf(o8[u], x8[u], acc);
    }
    y[(int64_t)b * rows + i] += acc;
  }
}

// Outlier tiles: per 512-row tile t of a matrix and outlier number q, 512
// words ocols[512 t + r][q] | ovals[512 t + r][q] << 16 (r = 0..511; rows past
// the end hold kNoOutlierWord), so that the q-th outliers of a tile's rows are
// one contiguous 2 KiB block.  One thread per output word.
constexpr int kOutTileRows = 512;
constexpr uint32_t kNoOutlierWord = 0xFFFFFFFFu;  // column field 0xFFFF: no column (cols <= 16384)

__global__ void __launch_bounds__(256) pack_outliers_kernel(const uint16_t* __restrict__ ocols,
                                                            const uint16_t* __restrict__ ovals, int64_t rows,
                                                            int64_t k, int64_t n_tiles, uint32_t* __restrict__ out) {
  const int64_t n = n_tiles * k * kOutTileRows;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = t % kOutTileRows, tq = t / kOutTileRows;
    const int64_t tile = tq / k, q = tq - tile * k;
    const int64_t row = tile * kOutTileRows + r;
    out[t] = row < rows ? (uint32_t)__ldg(ocols + row * k + q) | ((uint32_t)__ldg(ovals + row * k + q) << 16)
                        : kNoOutlierWord;
  }
}

// Grouped sparse add over outlier tiles (the calls the tiled GEMV does not
// fuse): one thread per row, y[b][i] += sum_q (float)o_iq * x[b][c_iq] in
// binary32, q ascending; a warp's reads of one q are 128 contiguous bytes.
struct OutTilesParams {
  const uint32_t* ot[kOutGemvMaxMats];
  const void* x[kOutGemvMaxMats];
  float* y[kOutGemvMaxMats];
  int64_t rows[kOutGemvMaxMats], k[kOutGemvMaxMats], cols[kOutGemvMaxMats];
  int64_t row_begin[kOutGemvMaxMats + 1];
  int n_mats, B;
};

template <int XDT>
__global__ void __launch_bounds__(256) outlier_tiles_add_kernel(const __grid_constant__ OutTilesParams P) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= P.row_begin[P.n_mats]) return;
  int m = 0;
  while (t >= P.row_begin[m + 1]) m++;
  const int64_t i = t - P.row_begin[m], k = P.k[m], cols = P.cols[m], rows = P.rows[m];
  const uint32_t* p = P.ot[m] + (i / kOutTileRows) * k * kOutTileRows + i % kOutTileRows;
  for (int b = 0; b < P.B; b++) {
    float acc = 0.0f;
    for (int64_t q0 = 0; q0 < k; q0 += 8) {
      uint32_t w8[8];
#pragma unroll
      for (int u = 0; u < 8; u++) w8[u] = q0 + u < k ? __ldg(p + (q0 + u) * kOutTileRows) : kNoOutlierWord;
      float x8[8];
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const int64_t c = w8[u] & 0xFFFFu;
        x8[u] = c < cols ? load1<XDT>(P.x[m], (int64_t)b * cols + c) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 8; u++)
        if ((w8[u] & 0xFFFFu) < cols) acc = fmaf(f16_bits_to_f32((uint16_t)(w8[u] >> 16)), x8[u], acc);
    }
    P.y[m][(int64_t)b * rows + i] += acc;
  }
}

}  // namespace vq3r
