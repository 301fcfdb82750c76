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
constexpr int kGvRowsPerWarp = 8;                           // 4 lanes per row, 16 columns per lane
constexpr int kGvTileRows = kGvWarps * kGvRowsPerWarp;      // 128 rows per unit
constexpr int kGvRing = 3;                                  // units of index words held per lane
constexpr int kSlabGroup = 2;                               // CTAs walking adjacent slabs in step
constexpr int kLutBuildBlocksPerImage = 12;                 // 64 (stage, codeword) rows per block

// Word offset of T_s[v][j] inside a slab image (v = column within the slab):
//   s * 16384 + j * 64 + slot(v) * 32 + bank(v),
//   slot(v) = (v >> 2) & 1,  bank(v) = 8 * (v >> 4) + (v & 3) + 4 * ((v >> 3) & 1).
// Lane (g, a) of a warp (g = lane / 4 picks one of 8 rows, a = lane % 4 the
// 16 columns [16a, 16a + 16)) visits its columns in the order o = m ^ d(g),
// d(g) = (g & 3) | ((g >> 2) << 3), m = 0..15.  At step m its bank is
// 8a + ((m ^ g) & 3) + 4 * ((m >> 3) ^ (g >> 2)), so the 32 lanes hit 32
// distinct banks whatever the indices, and the slot ((m >> 2) & 1) is the
// same for all lanes.  The column's index byte sits in register m >> 2 when
// the lane loads its two 8-byte halves in the order (g >> 2, 1 - (g >> 2)).
__host__ __device__ __forceinline__ int slab_word(int s, int v, int j) {
  return s * (kCodewords * kSlabV) + j * kSlabV + ((v >> 2) & 1) * 32 + 8 * (v >> 4) + (v & 3) + 4 * ((v >> 3) & 1);
}

struct GvMat {
  const uint8_t* idx;
  const uint16_t* scales;
  float* y;
  float* partial;        // [B][n_slabs][rows]
  int64_t rows;
  int64_t plane_stride;  // bytes between index planes
  int32_t group;
  int32_t n_tiles;       // ceil(rows / kGvTileRows) >= 1
  int32_t tile_prefix;   // tiles of the earlier matrices of the same group
  int32_t pad_;
};

struct GvGroup {
  const float* codebooks;
  const void* x;         // [B][cols]
  float* lut;            // [B][n_slabs] slab images
  int64_t cols;
  int64_t unit_begin;    // first work unit of this group
  int32_t n_slabs;
  int32_t n_sgroups;     // ceil(n_slabs / kSlabGroup)
  int32_t tiles;         // tiles of all matrices of the group (units per (slab, token))
  int32_t image_begin;   // first slab image (for the build kernel)
  int16_t mat_begin, mat_end;  // the group's matrices are P.m[mat_begin .. mat_end)
  int32_t pad_;
};

struct GvParams {
  GvMat m[VQ3R_GEMV_MAX_MATS];
  GvGroup g[VQ3R_GEMV_MAX_MATS];
  int32_t n_mats, n_groups, B, x_dtype;
  int64_t total_units;
  int32_t total_images;
  int32_t vec8;          // 1: index rows and planes are 8-byte aligned (64-bit loads)
};

// Programmatic dependent launch: wait until the preceding kernel in the
// stream has completed and its writes are visible / let the next kernel's
// CTAs launch early (they wait at their own griddep_wait).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------- table build ----------------

template <int XDT>
__global__ void __launch_bounds__(kGvThreads) lut_build_kernel(const __grid_constant__ GvParams P) {
  __shared__ float xs[kSlabV][kDim];
  griddep_launch_dependents();
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

// Work unit: (group, slab group, token, matrix, row tile of 128 rows),
// ordered so that consecutive units share a slab image.  The kSlabGroup CTAs
// of a CTA group take the same units, each its own slab of the slab group:
// they read adjacent 64-byte pieces of the same index rows at about the same
// time, so each 128-byte line fetched from DRAM serves both.
struct GvCursor {
  int g, sg, b, m, tile;
};

__device__ __forceinline__ GvCursor unit_cursor(const GvParams& P, int64_t u) {
  GvCursor c;
  int g = 0;
  while (g + 1 < P.n_groups && P.g[g + 1].unit_begin <= u) g++;
  const GvGroup& G = P.g[g];
  const int64_t lu = u - G.unit_begin;
  const int64_t sb = lu / G.tiles;  // slab * B + b
  const int t = (int)(lu - sb * G.tiles);
  c.g = g;
  c.sg = (int)(sb / P.B);
  c.b = (int)(sb - (int64_t)c.sg * P.B);
  int m = G.mat_begin;
  while (m + 1 < G.mat_end && P.m[m + 1].tile_prefix <= t) m++;
  c.m = m;
  c.tile = t - P.m[m].tile_prefix;
  return c;
}

__device__ __forceinline__ void unit_advance(const GvParams& P, GvCursor& c) {
  if (++c.tile < P.m[c.m].n_tiles) return;
  c.tile = 0;
  if (++c.m < P.g[c.g].mat_end) return;
  c.m = P.g[c.g].mat_begin;
  if (++c.b < P.B) return;
  c.b = 0;
  if (++c.sg < P.g[c.g].n_sgroups) return;
  c.sg = 0;
  if (++c.g < P.n_groups) c.m = P.g[c.g].mat_begin;
}

// The 12 index words of one lane for one unit: for plane s, registers 0-1
// hold bytes [8h, 8h + 8) and registers 2-3 bytes [8(1-h), 8(1-h) + 8) of the
// lane's 16 columns, h = g >> 2 (zero past the matrix's end).
__device__ __forceinline__ void load_unit_words(const GvParams& P, const GvCursor& c, int member, int warp, int g,
                                                int a, uint32_t wd[kStages][4]) {
  const GvMat& M = P.m[c.m];
  const int64_t V = P.g[c.g].cols / kDim;
  const int64_t row0 = (int64_t)c.tile * kGvTileRows;
  const int64_t row = row0 + warp * kGvRowsPerWarp + g;
  const int64_t col0 = (int64_t)(c.sg * kSlabGroup + member) * kSlabV;
  const int h = g >> 2;
  const uint8_t* base = M.idx + row * V + col0 + 16 * a;
  if (P.vec8 && row0 + kGvTileRows <= M.rows && col0 + kSlabV <= V) {
#pragma unroll
    for (int s = 0; s < kStages; s++) {
      const uint8_t* p = base + s * M.plane_stride;
      const uint2 x0 = __ldg(reinterpret_cast<const uint2*>(p + 8 * h));
      const uint2 x1 = __ldg(reinterpret_cast<const uint2*>(p + 8 * (1 - h)));
      wd[s][0] = x0.x;
      wd[s][1] = x0.y;
      wd[s][2] = x1.x;
      wd[s][3] = x1.y;
    }
  } else {  // edge of the matrix or unaligned rows: byte loads with bounds checks
    const bool row_ok = row < M.rows;
#pragma unroll
    for (int s = 0; s < kStages; s++) {
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const int cw = 4 * (k ^ (2 * h));  // first column of the word held in register k
        uint32_t x = 0;
#pragma unroll 1
        for (int i = 0; i < 4; i++)
          if (row_ok && col0 + 16 * a + cw + i < V) x |= (uint32_t)__ldg(base + s * M.plane_stride + cw + i) << (8 * i);
        wd[s][k] = x;
      }
    }
  }
}

__global__ void __launch_bounds__(kGvThreads, 1) gemv_lut_kernel(const __grid_constant__ GvParams P) {
  extern __shared__ __align__(128) unsigned char gv_smem[];
  unsigned char* lut_s = gv_smem;  // kSlabBytes
  uint64_t* mbar = reinterpret_cast<uint64_t*>(gv_smem + kSlabBytes);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, a = lane & 3;
  // PRMT operands: byte 0 = byte offset of the bank of the current column, byte 1 = its index.
  // lc[q], q = (m & 3) | ((m >> 3) << 2); sel[m & 3] picks the index byte (m ^ g) & 3.
  uint32_t lc[8];
#pragma unroll
  for (int q = 0; q < 8; q++)
    lc[q] = 4u * (8u * a + (uint32_t)((q & 3) ^ (g & 3)) + 4u * (uint32_t)((q >> 2) ^ (g >> 2)));
  uint32_t sel[4];
#pragma unroll
  for (int q = 0; q < 4; q++) sel[q] = 0x5504u | ((uint32_t)((q ^ g) & 3) << 4);

  const int member = blockIdx.x % kSlabGroup;  // which slab of each slab group
  const int64_t cg = blockIdx.x / kSlabGroup, ncg = gridDim.x / kSlabGroup;
  const int64_t u0 = cg * P.total_units / ncg;
  const int64_t u1 = (cg + 1) * P.total_units / ncg;
  griddep_launch_dependents();  // the reduction kernel may be scheduled now; it waits for us
  if (u0 >= u1) return;
  if (tid == 0) mbar_init(mbar, 1);
  __syncthreads();

  // Ring of kGvRing units of index words: while unit u is looked up, the
  // loads of units u+1 .. u+kGvRing-1 are in flight.
  GvCursor c0 = unit_cursor(P, u0), c1 = c0, c2;
  unit_advance(P, c1);
  c2 = c1;
  unit_advance(P, c2);
  uint32_t w0[kStages][4], w1[kStages][4], w2[kStages][4];
  load_unit_words(P, c0, member, warp, g, a, w0);
  if (u0 + 1 < u1) load_unit_words(P, c1, member, warp, g, a, w1);
  if (u0 + 2 < u1) load_unit_words(P, c2, member, warp, g, a, w2);

  griddep_wait();  // the slab tables written by the build kernel are complete

  const float* loaded = nullptr;
  uint32_t phase = 0;
  auto step = [&](int64_t u, GvCursor& c, uint32_t (&wa)[kStages][4]) -> bool {
    const GvGroup& G = P.g[c.g];
    const int slab = c.sg * kSlabGroup + member;
    if (slab >= G.n_slabs) {  // odd slab count: this CTA has no slab in the last group
#pragma unroll
      for (int i = 0; i < kGvRing; i++) unit_advance(P, c);
      if (u + kGvRing < u1) load_unit_words(P, c, member, warp, g, a, wa);
      return true;
    }
    const float* img = G.lut + ((size_t)c.b * G.n_slabs + slab) * kSlabWords;
    if (img != loaded) {
      __syncthreads();  // every warp is done with the previous image
      if (tid == 0) {
        mbar_arrive_expect_tx(mbar, kSlabBytes);
#pragma unroll
        for (int q = 0; q < 4; q++)
          bulk_copy_g2s(lut_s + q * (kSlabBytes / 4),
                        reinterpret_cast<const unsigned char*>(img) + q * (kSlabBytes / 4), kSlabBytes / 4, mbar);
      }
      if (!mbar_wait_bounded(mbar, phase)) return false;
      phase ^= 1u;
      loaded = img;
    }
    float acc = 0.0f;
#pragma unroll
    for (int m = 0; m < 16; m++) {
#pragma unroll
      for (int s = 0; s < kStages; s++) {
        const uint32_t off = __byte_perm(wa[s][m >> 2], lc[(m & 3) | ((m >> 3) << 2)], sel[m & 3]);
        acc += *reinterpret_cast<const float*>(lut_s + off + s * 65536 + ((m >> 2) & 1) * 128);
      }
    }
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 1);
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 2);
    const GvMat& M = P.m[c.m];
    const int64_t row = (int64_t)c.tile * kGvTileRows + warp * kGvRowsPerWarp + g;
    if (a == 0 && row < M.rows) M.partial[((int64_t)c.b * G.n_slabs + slab) * M.rows + row] = acc;
    // this buffer now takes unit u + kGvRing
#pragma unroll
    for (int i = 0; i < kGvRing; i++) unit_advance(P, c);
    if (u + kGvRing < u1) load_unit_words(P, c, member, warp, g, a, wa);
    return true;
  };
  for (int64_t u = u0; u < u1; u += kGvRing) {
    if (!step(u, c0, w0)) return;
    if (u + 1 < u1 && !step(u + 1, c1, w1)) return;
    if (u + 2 < u1 && !step(u + 2, c2, w2)) return;
  }
}

// y[b][i] = scale_i * sum_slab partial[b][slab][i], slabs in ascending order.
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const __grid_constant__ GvParams P) {
  // blockIdx.y = matrix
  griddep_wait();
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
