// VQ3R decode-GEMV for the MoE decode step: y[b] = W_hat . x[b], 1..32 tokens.
//
// Page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验", §1: each token
// activates a few experts, so decoding streams a few expert matrices per
// token and is bound by the bytes read; §2: W ~ scale x (C1[i1] + C2[i2] +
// C3[i3]) per 8-vector.
//
// x-projected tables.  For one token and one 8-vector column v,
//   W[i, 8v:8v+8] . x[8v:8v+8] = scale_i * sum_s C_s[i_s] . x[8v:8v+8]
//                               = scale_i * sum_s T_s[v][i_s],
//   T_s[v][j] = sum_k C_s[j][k] * x[8v+k].
// A row's dot product is then 3 table reads and 3 adds per 8 weights instead
// of gathering 3 x 32 bytes of codewords, so shared memory (4 B per lookup)
// keeps pace with HBM (0.375 B of indices per weight).
//
// Tables are built per slab of 64 vector columns (192 KiB: 3 stages x 256 x
// 64 fp32) into the workspace (lut_build_kernel) and bulk-copied into shared
// memory by the CTA that consumes them (gemv_lut_kernel).  Inside a slab the
// table of column v lives in one shared-memory bank, chosen so that the 32
// lanes of a warp always read 32 different banks whatever the indices are:
// lanes 0-15 take row 2p, lanes 16-31 row 2p+1, lane l owns columns
// 4(l mod 16) + {0..3}, and the upper half-warp walks its four columns
// rotated by two.  Partial sums per (slab, row) go to the workspace and a
// last kernel adds the slabs in order and applies the row scale.
#pragma once

#include "vq3r_common.cuh"

namespace vq3r {

constexpr int kSlabV = 64;                                  // vector columns per slab
constexpr int kSlabWords = kStages * kCodewords * kSlabV;   // 49152 floats
constexpr uint32_t kSlabBytes = kSlabWords * 4u;            // 192 KiB
constexpr int kGvThreads = 512;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvRowPairs = 4;                              // row pairs per warp per unit
constexpr int kGvTileRows = kGvWarps * kGvRowPairs * 2;     // 128 rows per unit
constexpr int kLutBuildBlocksPerImage = 12;                 // 64 (stage, codeword) rows per block

// Word offset of T_s[v][j] inside a slab image:
//   s * 16384 + j * 64 + (v & 1) * 32 + bank(v),  bank(v) = 16 * ((v >> 1) & 1) + (v >> 2).
__host__ __device__ __forceinline__ int slab_word(int s, int v, int j) {
  return s * (kCodewords * kSlabV) + j * kSlabV + (v & 1) * 32 + 16 * ((v >> 1) & 1) + (v >> 2);
}

struct GvMat {
  const uint8_t* idx;
  const uint16_t* scales;
  float* y;
  float* partial;     // [B][n_slabs][rows]
  int64_t rows;
  int64_t plane_stride;  // bytes between index planes
  int32_t group;
  int32_t n_tiles;     // ceil(rows / kGvTileRows)
  int32_t tile_prefix; // tiles of the earlier matrices of the same group
  int32_t pad_;
};

struct GvGroup {
  const float* codebooks;
  const void* x;       // [B][cols]
  float* lut;          // [B][n_slabs] slab images
  int64_t cols;
  int64_t unit_begin;  // first work unit of this group
  int32_t n_slabs;
  int32_t tiles;       // tiles of all matrices of the group (units per (slab, token))
  int32_t image_begin; // first slab image (for the build kernel)
  int32_t pad_;
};

struct GvParams {
  GvMat m[VQ3R_GEMV_MAX_MATS];
  GvGroup g[VQ3R_GEMV_MAX_MATS];
  int32_t n_mats, n_groups, B, x_dtype;
  int64_t total_units;
  int32_t total_images;
  int32_t pad_;
};

// ---------------- table build ----------------

template <int XDT>
__global__ void __launch_bounds__(kGvThreads) lut_build_kernel(const __grid_constant__ GvParams P) {
  __shared__ float xs[kSlabV][kDim];
  const int image = blockIdx.x / kLutBuildBlocksPerImage;
  const int part = blockIdx.x - image * kLutBuildBlocksPerImage;
  int gi = 0;
  while (gi + 1 < P.n_groups && P.g[gi + 1].image_begin <= image) gi++;
  const GvGroup& G = P.g[gi];
  const int local = image - G.image_begin;  // = b * n_slabs + slab
  const int b = local / G.n_slabs, slab = local - b * G.n_slabs;
  const int64_t V = G.cols / kDim;
  for (int i = threadIdx.x; i < kSlabV * kDim; i += blockDim.x) {
    const int v = i / kDim, k = i - v * kDim;
    const int64_t vg = (int64_t)slab * kSlabV + v;
    xs[v][k] = (vg < V) ? load1<XDT>(G.x, (int64_t)b * G.cols + vg * kDim + k) : 0.0f;
  }
  __syncthreads();
  float* img = G.lut + (size_t)local * kSlabWords;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kRowsPerBlock = kStages * kCodewords / kLutBuildBlocksPerImage;  // 64
  for (int rr = warp; rr < kRowsPerBlock; rr += kGvWarps) {
    const int e = part * kRowsPerBlock + rr;  // (stage, codeword) row
    const int s = e / kCodewords, j = e - s * kCodewords;
    const float4* cp = reinterpret_cast<const float4*>(G.codebooks + (size_t)e * kDim);
    const float4 c0 = __ldg(cp), c1 = __ldg(cp + 1);
#pragma unroll
    for (int half = 0; half < 2; half++) {
      const int v = lane + 32 * half;
      const float* xv = xs[v];
      float t = c0.x * xv[0];
      t = fmaf(c0.y, xv[1], t);
      t = fmaf(c0.z, xv[2], t);
      t = fmaf(c0.w, xv[3], t);
      t = fmaf(c1.x, xv[4], t);
      t = fmaf(c1.y, xv[5], t);
      t = fmaf(c1.z, xv[6], t);
      t = fmaf(c1.w, xv[7], t);
      img[slab_word(s, v, j)] = t;
    }
  }
}

// ---------------- main kernel ----------------

// Unit u of the schedule: (group, slab, token, matrix, row tile), ordered so
// that consecutive units share a slab image.
struct GvUnit {
  int g, slab, b, m, tile;
};

__device__ __forceinline__ GvUnit decode_unit(const GvParams& P, int64_t u) {
  GvUnit r;
  int g = 0;
  while (g + 1 < P.n_groups && P.g[g + 1].unit_begin <= u) g++;
  const GvGroup& G = P.g[g];
  const int64_t lu = u - G.unit_begin;
  const int64_t sb = lu / G.tiles;  // slab * B + b
  int t = (int)(lu - sb * G.tiles);
  r.g = g;
  r.slab = (int)(sb / P.B);
  r.b = (int)(sb - (int64_t)r.slab * P.B);
  int m = 0;
  while (m < P.n_mats && !(P.m[m].group == g && t >= P.m[m].tile_prefix && t < P.m[m].tile_prefix + P.m[m].n_tiles))
    m++;
  r.m = m;
  r.tile = t - P.m[m].tile_prefix;
  return r;
}

template <bool ALIGNED4>
__device__ __forceinline__ uint32_t load_idx_word(const uint8_t* plane, int64_t off, int64_t v0, int64_t V) {
  if (ALIGNED4) {
    return (v0 < V) ? __ldcs(reinterpret_cast<const unsigned int*>(plane + off)) : 0u;
  } else {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 4; i++)
      if (v0 + i < V) w |= (uint32_t)__ldcs(plane + off + i) << (8 * i);
    return w;
  }
}

template <bool ALIGNED4>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_lut_kernel(const __grid_constant__ GvParams P) {
  extern __shared__ __align__(128) unsigned char gv_smem[];
  unsigned char* lut_s = gv_smem;                                  // kSlabBytes
  uint64_t* mbar = reinterpret_cast<uint64_t*>(gv_smem + kSlabBytes);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = lane >> 4, l16 = lane & 15;
  // PRMT operands: byte 0 = bank byte offset of this lane's column, byte 1 = index byte.
  const uint32_t lc0 = 64u * h + 4u * l16;        // steps m = 0, 1
  const uint32_t lc1 = 64u * (1 - h) + 4u * l16;  // steps m = 2, 3
  uint32_t sel[4];
#pragma unroll
  for (int m = 0; m < 4; m++) sel[m] = 0x5504u | ((uint32_t)((m + 2 * h) & 3) << 4);

  const int64_t u0 = (int64_t)blockIdx.x * P.total_units / gridDim.x;
  const int64_t u1 = (int64_t)(blockIdx.x + 1) * P.total_units / gridDim.x;
  if (tid == 0) mbar_init(mbar, 1);
  __syncthreads();

  const float* cur = nullptr;
  uint32_t phase = 0;
  for (int64_t u = u0; u < u1; u++) {
    const GvUnit U = decode_unit(P, u);
    const GvGroup& G = P.g[U.g];
    const GvMat& M = P.m[U.m];
    const float* img = G.lut + ((size_t)U.b * G.n_slabs + U.slab) * kSlabWords;
    if (img != cur) {
      __syncthreads();  // every warp is done with the previous image
      if (tid == 0) {
        mbar_arrive_expect_tx(mbar, kSlabBytes);
#pragma unroll
        for (int c = 0; c < 4; c++)
          bulk_copy_g2s(lut_s + c * (kSlabBytes / 4), reinterpret_cast<const unsigned char*>(img) + c * (kSlabBytes / 4),
                        kSlabBytes / 4, mbar);
      }
      if (!mbar_wait_bounded(mbar, phase)) return;
      phase ^= 1u;
      cur = img;
    }
    const int64_t V = G.cols / kDim;
    const int64_t v0 = (int64_t)U.slab * kSlabV + 4 * l16;
    const int64_t row0 = (int64_t)U.tile * kGvTileRows + warp * (2 * kGvRowPairs) + h;
    const int64_t plane_stride = M.plane_stride;

    uint32_t wd[kGvRowPairs][kStages];
#pragma unroll
    for (int p = 0; p < kGvRowPairs; p++) {
      const int64_t row = row0 + 2 * p;
#pragma unroll
      for (int s = 0; s < kStages; s++)
        wd[p][s] = (row < M.rows) ? load_idx_word<ALIGNED4>(M.idx + s * plane_stride, row * V + v0, v0, V) : 0u;
    }
    float acc[kGvRowPairs];
#pragma unroll
    for (int p = 0; p < kGvRowPairs; p++) {
      float a = 0.0f;
#pragma unroll
      for (int m = 0; m < 4; m++) {
        const uint32_t lc = (m < 2) ? lc0 : lc1;
#pragma unroll
        for (int s = 0; s < kStages; s++) {
          const uint32_t off = __byte_perm(wd[p][s], lc, sel[m]);
          a += *reinterpret_cast<const float*>(lut_s + off + s * 65536 + (m & 1) * 128);
        }
      }
      acc[p] = a;
    }
#pragma unroll
    for (int p = 0; p < kGvRowPairs; p++) {
      float a = acc[p];
      a += __shfl_xor_sync(0xFFFFFFFFu, a, 8);
      a += __shfl_xor_sync(0xFFFFFFFFu, a, 4);
      a += __shfl_xor_sync(0xFFFFFFFFu, a, 2);
      a += __shfl_xor_sync(0xFFFFFFFFu, a, 1);
      const int64_t row = row0 + 2 * p;
      if (l16 == 0 && row < M.rows) M.partial[((int64_t)U.b * G.n_slabs + U.slab) * M.rows + row] = a;
    }
  }
}

// y[b][i] = scale_i * sum_slab partial[b][slab][i], slabs in ascending order.
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const __grid_constant__ GvParams P) {
  // blockIdx.y = matrix
  const GvMat& M = P.m[blockIdx.y];
  const GvGroup& G = P.g[M.group];
  const int64_t n = (int64_t)P.B * M.rows;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = i / M.rows, row = i - b * M.rows;
    const float* pp = M.partial + b * G.n_slabs * M.rows + row;
    float a = 0.0f;
    for (int s = 0; s < G.n_slabs; s++) a += pp[(int64_t)s * M.rows];
    M.y[i] = f16_bits_to_f32(__ldg(M.scales + row)) * a;
  }
}

}  // namespace vq3r
