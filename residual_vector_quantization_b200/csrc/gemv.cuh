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
// A row's dot product is then one 4-byte table read and one add per stage
// and 8 weights instead of a 32-byte codeword gather, so shared memory keeps
// pace with HBM (0.375 B of indices per weight).
//
// Work is split into units of (stage s, slab of 64 columns, token b, matrix,
// tile of 256 rows).  A CTA builds the 64 KiB table T_s[slab][.] of its
// current units in shared memory; two CTAs share an SM.  Each lane loads the
// 16 index bytes of its two rows straight into registers and keeps the loads
// of the next three units in flight (about 128 KiB per SM), so index bytes
// never pass through shared memory, which is left to the lookups.
// Per-(stage, slab, row) partial sums go to the workspace; the reduction
// kernel adds them in a fixed order and applies the row scale, so results do
// not depend on scheduling.
#pragma once

#include "vq3r_common.cuh"

namespace vq3r {

constexpr int kSlabV = 64;                        // vector columns per slab
constexpr int kTabWords = kCodewords * kSlabV;    // 16384 floats: one stage, one slab
constexpr uint32_t kTabBytes = kTabWords * 4u;    // 64 KiB
constexpr int kGvThreads = 512;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvRowsPerWarp = 16;                // rows g and g + 8 of the warp's 16 (4 lanes per row)
constexpr int kGvTileRows = kGvWarps * kGvRowsPerWarp;  // 256 rows per unit
constexpr int kGvRing = 4;                        // units of index words in flight per lane
constexpr size_t kGvSmemBytes = kTabBytes + (size_t)(kSlabV * kDim + kCodewords * kDim) * 4;

// Tiled index layout (VQ3R_LAYOUT_TILES): per (stage s, slab, tile of
// kTileRows rows) one contiguous block of kTileRows x 64 bytes, blocks ordered
// ((s * n_slabs + slab) * n_tiles + tile); row r of a block at r * 64, column
// c at 16 (c >> 4) + 8 (((c >> 3) & 1) ^ ((r >> 2) & 1)) + (c & 7); rows and
// columns past the matrix are zero.  The swapped halves are the register
// order the lookup schedule wants, so a 16-byte load needs no shuffling.
constexpr int kTileRows = 512;
constexpr int kTileBytes = kTileRows * kSlabV;  // 32 KiB
__host__ __device__ __forceinline__ int tile_byte(int r, int c) {
  return r * kSlabV + 16 * (c >> 4) + 8 * (((c >> 3) & 1) ^ ((r >> 2) & 1)) + (c & 7);
}

// Word offset of T[v][j] inside a table (v = column within the slab):
//   j * 64 + slot(v) * 32 + bank(v),
//   slot(v) = (v >> 2) & 1,  bank(v) = 8 * (v >> 4) + (v & 3) + 4 * ((v >> 3) & 1).
// Lane (g, a) of a warp (g = lane / 4 picks one of 8 rows, a = lane % 4 the
// 16 columns [16a, 16a + 16)) visits its columns in the order o = m ^ d(g),
// d(g) = (g & 3) | ((g >> 2) << 3), m = 0..15.  At step m its bank is
// 8a + ((m ^ g) & 3) + 4 * ((m >> 3) ^ (g >> 2)), so the 32 lanes hit 32
// distinct banks whatever the indices, and the slot ((m >> 2) & 1) is the
// same for all lanes.  The column's index byte is in register m >> 2 when
// registers 0-1 hold the 8-byte half h = g >> 2 of the lane's 16 index bytes
// and registers 2-3 the other half.
__host__ __device__ __forceinline__ int tab_word(int v, int j) {
  return j * kSlabV + ((v >> 2) & 1) * 32 + 8 * (v >> 4) + (v & 3) + 4 * ((v >> 3) & 1);
}

struct GvMat {
  const uint8_t* idx;
  const uint16_t* scales;
  float* y;
  float* partial;        // [B][3][n_slabs][rows]
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
  int64_t cols;
  int64_t unit_begin;    // first work unit of this group
  int32_t n_slabs;
  int32_t tiles;         // tiles of all matrices of the group (units per table)
  int16_t mat_begin, mat_end;  // the group's matrices are P.m[mat_begin .. mat_end)
  int32_t pad_;
};

struct GvParams {
  GvMat m[VQ3R_GEMV_MAX_MATS];
  GvGroup g[VQ3R_GEMV_MAX_MATS];
  int32_t n_mats, n_groups, B, vec8;  // vec8: rows and planes 8-byte aligned (64-bit index loads)
  int64_t total_units;
  int32_t tile_rows;     // rows per work unit: kGvTileRows (planes) or kTileRows (tiles)
  int32_t layout;        // VQ3R_LAYOUT_PLANES or VQ3R_LAYOUT_TILES
};

// Programmatic dependent launch: wait until the preceding kernel in the
// stream has completed and its writes are visible / let the next kernel's
// CTAs launch early (they wait at their own griddep_wait).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Work unit cursor: group, table (slab, stage, token), matrix, row tile.
// Units are ordered (group, slab, stage, token, matrix, tile) so that
// consecutive units share a table.  Decoded once per CTA, then advanced
// with carries (no divisions in the loop).
struct GvCursor {
  int g, slab, s, b, m, tile;
};

__device__ __forceinline__ GvCursor unit_cursor(const GvParams& P, int64_t u) {
  GvCursor c;
  int g = 0;
  while (g + 1 < P.n_groups && P.g[g + 1].unit_begin <= u) g++;
  const GvGroup& G = P.g[g];
  const int64_t lu = u - G.unit_begin;
  c.g = g;
  const int tab = (int)(lu / G.tiles);
  const int t = (int)(lu - (int64_t)tab * G.tiles);
  c.b = tab % P.B;
  c.s = (tab / P.B) % kStages;
  c.slab = tab / (P.B * kStages);
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
  if (++c.s < kStages) return;
  c.s = 0;
  if (++c.slab < P.g[c.g].n_slabs) return;
  c.slab = 0;
  if (++c.g < P.n_groups) c.m = P.g[c.g].mat_begin;
}

// The 8 index words of one lane for one unit: for each of its two rows,
// registers 0-1 hold bytes [8h, 8h + 8) and registers 2-3 bytes
// [8(1-h), 8(1-h) + 8) of the lane's 16 columns, h = g >> 2 (zero past the
// matrix's end).
__device__ __forceinline__ void load_unit_words(const GvParams& P, const GvCursor& c, int warp, int g, int a,
                                                uint32_t wd[2][4]) {
  const GvGroup& G = P.g[c.g];
  const GvMat& M = P.m[c.m];
  const int64_t V = G.cols / kDim;
  const int64_t row0 = (int64_t)c.tile * kGvTileRows;
  const int64_t col0 = (int64_t)c.slab * kSlabV;
  const int h = g >> 2;
  const int64_t r = row0 + warp * kGvRowsPerWarp + g;
  const uint8_t* p = M.idx + (int64_t)c.s * M.plane_stride + r * V + col0 + 16 * a;
  if (P.vec8 && row0 + kGvTileRows <= M.rows && col0 + kSlabV <= V) {
#pragma unroll
    for (int q = 0; q < 2; q++) {
      const uint8_t* pr = p + (int64_t)(8 * q) * V;
      const uint2 x0 = __ldg(reinterpret_cast<const uint2*>(pr + 8 * h));
      const uint2 x1 = __ldg(reinterpret_cast<const uint2*>(pr + 8 * (1 - h)));
      wd[q][0] = x0.x;
      wd[q][1] = x0.y;
      wd[q][2] = x1.x;
      wd[q][3] = x1.y;
    }
  } else {  // edge of the matrix or unaligned rows: byte loads with bounds checks
#pragma unroll
    for (int q = 0; q < 2; q++) {
      const bool row_ok = r + 8 * q < M.rows;
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const int cw = 4 * (k ^ (2 * h));  // first column of the word held in register k
        uint32_t x = 0;
#pragma unroll 1
        for (int i = 0; i < 4; i++)
              if (row_ok && col0 + 16 * a + cw + i < V) x |= (uint32_t)__ldg(p + (int64_t)(8 * q) * V + cw + i) << (8 * i);
        wd[q][k] = x;
      }
    }
  }
}

// Build T[v][j] = C_s[j] . x_b[8(slab*64 + v) .. +8] (zero past the row end).
// The stage's codebook (8 KiB) and the x slab (2 KiB) are first copied to
// shared memory by one load per thread, so the build costs one round trip.
template <int XDT>
__device__ __forceinline__ void build_table(const GvGroup& G, const GvCursor& T, float* tab, float* xs, float* cbs,
                                            int tid) {
  const int64_t V = G.cols / kDim;
  __syncthreads();  // every warp is done with the previous table
  for (int i = tid; i < kSlabV * kDim; i += kGvThreads) {
    const int v = i >> 3, k = i & 7;
    const int64_t vg = (int64_t)T.slab * kSlabV + v;
    xs[i] = (vg < V) ? load1<XDT>(G.x, (int64_t)T.b * G.cols + vg * kDim + k) : 0.0f;
  }
  for (int i = tid; i < kCodewords * kDim / 4; i += kGvThreads)
    reinterpret_cast<float4*>(cbs)[i] =
        __ldg(reinterpret_cast<const float4*>(G.codebooks + (size_t)T.s * kCodewords * kDim) + i);
  __syncthreads();
  const int lane = tid & 31, warp = tid >> 5;
  const float4* xa = reinterpret_cast<const float4*>(xs + lane * kDim);
  const float4* xb = reinterpret_cast<const float4*>(xs + (lane + 32) * kDim);
  const float4 xa0 = xa[0], xa1 = xa[1], xb0 = xb[0], xb1 = xb[1];
  const float4* cb = reinterpret_cast<const float4*>(cbs);
#pragma unroll 2
  for (int j = warp; j < kCodewords; j += kGvWarps) {
    const float4 c0 = cb[2 * j], c1 = cb[2 * j + 1];
    float ta = c0.x * xa0.x, tb = c0.x * xb0.x;
    ta = fmaf(c0.y, xa0.y, ta); tb = fmaf(c0.y, xb0.y, tb);
    ta = fmaf(c0.z, xa0.z, ta); tb = fmaf(c0.z, xb0.z, tb);
    ta = fmaf(c0.w, xa0.w, ta); tb = fmaf(c0.w, xb0.w, tb);
    ta = fmaf(c1.x, xa1.x, ta); tb = fmaf(c1.x, xb1.x, tb);
    ta = fmaf(c1.y, xa1.y, ta); tb = fmaf(c1.y, xb1.y, tb);
    ta = fmaf(c1.z, xa1.z, ta); tb = fmaf(c1.z, xb1.z, tb);
    ta = fmaf(c1.w, xa1.w, ta); tb = fmaf(c1.w, xb1.w, tb);
    tab[tab_word(lane, j)] = ta;
    tab[tab_word(lane + 32, j)] = tb;
  }
  __syncthreads();
}

template <int XDT>
__global__ void __launch_bounds__(kGvThreads, 2) gemv_lut_kernel(const __grid_constant__ GvParams P) {
  extern __shared__ __align__(128) unsigned char gv_smem[];
  float* tab = reinterpret_cast<float*>(gv_smem);                  // kTabBytes
  float* xs = reinterpret_cast<float*>(gv_smem + kTabBytes);       // 64 x 8 floats
  float* cbs = xs + kSlabV * kDim;                                 // 256 x 8 floats

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

  const int64_t u0 = (int64_t)blockIdx.x * P.total_units / gridDim.x;
  const int64_t u1 = (int64_t)(blockIdx.x + 1) * P.total_units / gridDim.x;
  griddep_launch_dependents();  // the reduction kernel may be scheduled; it waits for this grid
  if (u0 >= u1) return;

  // Ring of kGvRing units of index words: while unit u is looked up, the
  // loads of units u+1 .. u+3 are in flight.  ci is the next unit to load.
  GvCursor ci = unit_cursor(P, u0);
  GvCursor c0 = ci, c1, c2, c3;
  uint32_t w0[2][4], w1[2][4], w2[2][4], w3[2][4];
  load_unit_words(P, ci, warp, g, a, w0);
  unit_advance(P, ci);
  c1 = ci;
  if (u0 + 1 < u1) load_unit_words(P, ci, warp, g, a, w1);
  unit_advance(P, ci);
  c2 = ci;
  if (u0 + 2 < u1) load_unit_words(P, ci, warp, g, a, w2);
  unit_advance(P, ci);
  c3 = ci;
  if (u0 + 3 < u1) load_unit_words(P, ci, warp, g, a, w3);
  unit_advance(P, ci);

  int loaded_g = -1, loaded_tab = -1;
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(tab);
  auto step = [&](int64_t u, GvCursor& c, uint32_t (&wa)[2][4]) {
    const GvGroup& G = P.g[c.g];
    const int tab_id = (c.slab * kStages + c.s) * P.B + c.b;
    if (c.g != loaded_g || tab_id != loaded_tab) {
      build_table<XDT>(G, c, tab, xs, cbs, tid);
      loaded_g = c.g;
      loaded_tab = tab_id;
    }
    const GvMat& M = P.m[c.m];
    const int row = c.tile * kGvTileRows + warp * kGvRowsPerWarp + g;
    float* part = M.partial + (((int64_t)c.b * kStages + c.s) * G.n_slabs + c.slab) * M.rows + row;
    const bool w_ok0 = a == 0 && row < M.rows, w_ok1 = a == 0 && row + 8 < M.rows;
#pragma unroll
    for (int q = 0; q < 2; q++) {
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int m = 0; m < 16; m += 2) {
        const uint32_t o0 = __byte_perm(wa[q][m >> 2], lc[(m & 3) | ((m >> 3) << 2)], sel[m & 3]);
        const uint32_t o1 = __byte_perm(wa[q][(m + 1) >> 2], lc[((m + 1) & 3) | (((m + 1) >> 3) << 2)], sel[(m + 1) & 3]);
        const float t0 = *reinterpret_cast<const float*>(tb + o0 + ((m >> 2) & 1) * 128);
        const float t1 = *reinterpret_cast<const float*>(tb + o1 + (((m + 1) >> 2) & 1) * 128);
        acc = __fadd2_rn(acc, make_float2(t0, t1));
      }
      float sum = acc.x + acc.y;
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
      if (q == 0 ? w_ok0 : w_ok1) part[8 * q] = sum;
    }
    // this buffer now takes the next unit to load
    c = ci;
    if (u + kGvRing < u1) load_unit_words(P, ci, warp, g, a, wa);
    unit_advance(P, ci);
  };
  for (int64_t u = u0; u < u1; u += kGvRing) {
    step(u, c0, w0);
    if (u + 1 < u1) step(u + 1, c1, w1);
    if (u + 2 < u1) step(u + 2, c2, w2);
    if (u + 3 < u1) step(u + 3, c3, w3);
  }
}

// Decode-GEMV over the tiled index layout: the 32 KiB block of a unit is
// contiguous, so each lane reads the 16 bytes of its 4 rows with four 16-byte
// loads and keeps the next unit's loads in flight (two-deep register ring).
template <int XDT>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_tiles_kernel(const __grid_constant__ GvParams P) {
  extern __shared__ __align__(128) unsigned char gv_smem[];
  float* tab = reinterpret_cast<float*>(gv_smem);
  float* xs = reinterpret_cast<float*>(gv_smem + kTabBytes);
  float* cbs = xs + kSlabV * kDim;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, a = lane & 3;
  uint32_t lc[8];
#pragma unroll
  for (int q = 0; q < 8; q++)
    lc[q] = 4u * (8u * a + (uint32_t)((q & 3) ^ (g & 3)) + 4u * (uint32_t)((q >> 2) ^ (g >> 2)));
  uint32_t sel[4];
#pragma unroll
  for (int q = 0; q < 4; q++) sel[q] = 0x5504u | ((uint32_t)((q ^ g) & 3) << 4);
  constexpr int kRowsPerWarpT = kTileRows / kGvWarps;  // 32: rows warp*32 + 8t + g, t = 0..3
  const int lane_off = (warp * kRowsPerWarpT + g) * kSlabV + 16 * a;

  const int64_t u0 = (int64_t)blockIdx.x * P.total_units / gridDim.x;
  const int64_t u1 = (int64_t)(blockIdx.x + 1) * P.total_units / gridDim.x;
  griddep_launch_dependents();
  if (u0 >= u1) return;

  auto load = [&](const GvCursor& c, uint4 (&w)[4]) {
    const GvMat& M = P.m[c.m];
    const uint8_t* base = M.idx + ((int64_t)c.s * P.g[c.g].n_slabs + c.slab) * M.plane_stride +
                          (int64_t)c.tile * kTileBytes + lane_off;
#pragma unroll
    for (int t = 0; t < 4; t++) w[t] = __ldg(reinterpret_cast<const uint4*>(base + t * 8 * kSlabV));
  };
  GvCursor ci = unit_cursor(P, u0);
  GvCursor c0 = ci, c1;
  uint4 r0[4], r1[4];
  load(ci, r0);
  unit_advance(P, ci);
  c1 = ci;
  if (u0 + 1 < u1) load(ci, r1);
  unit_advance(P, ci);

  int loaded_g = -1, loaded_tab = -1;
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(tab);
  auto step = [&](int64_t u, GvCursor& c, uint4 (&wr)[4]) {
    const GvGroup& G = P.g[c.g];
    const int tab_id = (c.slab * kStages + c.s) * P.B + c.b;
    if (c.g != loaded_g || tab_id != loaded_tab) {
      build_table<XDT>(G, c, tab, xs, cbs, tid);
      loaded_g = c.g;
      loaded_tab = tab_id;
    }
    const GvMat& M = P.m[c.m];
    const int row = c.tile * kTileRows + warp * kRowsPerWarpT + g;
    float* part = M.partial + (((int64_t)c.b * kStages + c.s) * G.n_slabs + c.slab) * M.rows + row;
#pragma unroll
    for (int t = 0; t < 4; t++) {
      const uint32_t w[4] = {wr[t].x, wr[t].y, wr[t].z, wr[t].w};
      float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
      for (int m = 0; m < 16; m++) {
        const uint32_t off = __byte_perm(w[m >> 2], lc[(m & 3) | ((m >> 3) << 2)], sel[m & 3]);
        const float tv = *reinterpret_cast<const float*>(tb + off + ((m >> 2) & 1) * 128);
        if (m & 1) acc1 += tv;
        else acc0 += tv;
      }
      float sum = acc0 + acc1;
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
      if (a == 0 && row + 8 * t < M.rows) part[8 * t] = sum;
    }
    c = ci;
    if (u + 2 < u1) load(ci, wr);
    unit_advance(P, ci);
  };
  for (int64_t u = u0; u < u1; u += 2) {
    step(u, c0, r0);
    if (u + 1 < u1) step(u + 1, c1, r1);
  }
}

// Repack the index planes [3][rows][cols/8] (plane_stride bytes apart) into
// the tiled layout; one thread per 16-byte chunk of the output.
__global__ void __launch_bounds__(256) pack_tiles_kernel(const uint8_t* __restrict__ idx, int64_t rows, int64_t V,
                                                          int64_t plane_stride, int32_t n_slabs, int64_t n_tiles,
                                                          uint8_t* __restrict__ out) {
  const int64_t n_chunks = (int64_t)kStages * n_slabs * n_tiles * (kTileBytes / 16);
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < n_chunks; q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = q / (kTileBytes / 16);
    const int within = (int)(q - blk * (kTileBytes / 16));
    const int r = within >> 2, ch = within & 3;  // packed row, 16-byte chunk
    const int64_t tile = blk % n_tiles;
    const int64_t sc = blk / n_tiles;
    const int slab = (int)(sc % n_slabs), s = (int)(sc / n_slabs);
    const int64_t row = tile * kTileRows + r;
    uint32_t h[4] = {0u, 0u, 0u, 0u};  // the chunk's 16 columns in source order
    if (row < rows) {
      const uint8_t* src = idx + s * plane_stride + row * V;
#pragma unroll
      for (int i = 0; i < 16; i++) {
        const int64_t col = (int64_t)slab * kSlabV + 16 * ch + i;
        const uint32_t v = col < V ? (uint32_t)__ldg(src + col) : 0u;
        h[i >> 2] |= v << (8 * (i & 3));
      }
    }
    const bool swap = (r >> 2) & 1;  // rows whose two 8-byte halves are stored swapped
    reinterpret_cast<uint4*>(out)[q] = swap ? make_uint4(h[2], h[3], h[0], h[1]) : make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// y[b][i] = scale_i * sum_s sum_slab partial[b][s][slab][i].  Four lanes share
// an output: lane k of the group adds partials k, k+4, k+8, ... in order, then
// two butterfly steps combine the four sums, so the order is fixed.
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const __grid_constant__ GvParams P) {
  griddep_wait();  // the partial sums of the main kernel are complete
  const GvMat& M = P.m[blockIdx.y];
  const GvGroup& G = P.g[M.group];
  const int64_t n = (int64_t)P.B * M.rows;
  const int np = kStages * G.n_slabs;
  const int sub = threadIdx.x & 3;
  const int64_t per_pass = (int64_t)gridDim.x * (blockDim.x / 4);
  for (int64_t base = (int64_t)blockIdx.x * (blockDim.x / 4); base < n; base += per_pass) {
    const int64_t i = base + (threadIdx.x >> 2);
    float acc = 0.0f;
    if (i < n) {
      const int64_t b = i / M.rows, row = i - b * M.rows;
      const float* pp = M.partial + b * np * M.rows + row;
#pragma unroll 4
      for (int k = sub; k < np; k += 4) acc += __ldg(pp + (int64_t)k * M.rows);
    }
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 1);
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 2);
    if (i < n && sub == 0) {
      const int64_t row = i - (i / M.rows) * M.rows;
      M.y[i] = f16_bits_to_f32(__ldg(M.scales + row)) * acc;
    }
  }
}

}  // namespace vq3r
