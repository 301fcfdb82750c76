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
// row tile).  A CTA builds the 64 KiB table T_s[slab][.] of its current units
// in shared memory.  Each lane loads the 16 index bytes of its rows straight
// into registers and keeps the next units' loads in flight, so index bytes
// never pass through shared memory, which is left to the lookups.
// Two kernels: gemv_lut_kernel reads the encoder's plane layout (256-row
// tiles, two CTAs per SM) and leaves per-(stage, slab, row) partial sums that
// gemv_reduce_kernel adds in a fixed order, so its results do not depend on
// scheduling; gemv_tiles_kernel reads the tiled layout (512-row tiles, one
// CTA per SM) and adds each unit's scaled row sums straight into y.
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
constexpr int kTileSlots = 2;                   // units of index registers per lane in the tiled kernel
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
  void* partial;         // planes: [B][3][n_slabs][rows] float partial sums (unused by the tiled kernel)
  int64_t rows;
  int64_t plane_stride;  // bytes between index planes
  int32_t group;
  int32_t n_tiles;       // ceil(rows / kGvTileRows) >= 1
  int32_t tile_prefix;   // tiles of the earlier matrices of the same group
  int32_t blk_begin;     // first row block of this matrix in the tensor-core kernel's grid
  // sparse outlier residual added by the tiled kernel (n_out = 0: none), in the outlier-tile layout
  // (per 512-row tile and outlier number q, 512 words column | value << 16)
  const uint32_t* otiles;
  int32_t n_out;
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

constexpr int kMaxSplit = 256;  // CTAs whose unit ranges the host can set (tiled kernel)

struct GvParams {
  GvMat m[VQ3R_GEMV_MAX_MATS];
  GvGroup g[VQ3R_GEMV_MAX_MATS];
  int64_t cta_begin[kMaxSplit + 1];  // tiles: CTA c takes units [cta_begin[c], cta_begin[c + 1]) when n_split == grid
  // tiles, when n_split == grid: where CTA c starts (table key, matrix and
  // tile of its first unit) and the table key of its last unit, so that a
  // CTA need not search the descriptors for them
  uint32_t cta_key0[kMaxSplit], cta_key_last[kMaxSplit];
  int32_t cta_m0[kMaxSplit], cta_tile0[kMaxSplit];
  int32_t n_mats, n_groups, B, vec8;  // vec8: rows and planes 8-byte aligned (64-bit index loads)
  int32_t nb;            // table tokens: B, or ceil(B / 2) when the tiled kernel looks up two tokens per table pair
  int32_t tokm;          // tokens per table token (1 or 2): table token b covers tokens tokm * b ..
  int32_t nst;           // table stages per slab: 3 (VQ3R, one table per stage), 1 (VQ4P, one table for all four)
  int64_t total_units;
  int32_t has_out;       // some matrix has outliers (tiled kernel with OUTL)
  int32_t tile_rows;     // rows per work unit: kGvTileRows (planes) or kTileRows (tiles)
  int32_t layout;        // VQ3R_LAYOUT_PLANES or VQ3R_LAYOUT_TILES
  unsigned long long* hdr;  // workspace header: [0] arrival count at the start of the call, [1] arrival count
  int32_t n_split;       // tiles: entries of cta_begin in use minus one (0: equal split)
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

__host__ __device__ __forceinline__ GvCursor unit_cursor(const GvParams& P, int64_t u) {
  GvCursor c;
  int g = 0;
  while (g + 1 < P.n_groups && P.g[g + 1].unit_begin <= u) g++;
  const GvGroup& G = P.g[g];
  const int64_t lu = u - G.unit_begin;
  c.g = g;
  const int tab = (int)(lu / G.tiles);
  const int t = (int)(lu - (int64_t)tab * G.tiles);
  c.b = tab % P.nb;
  c.s = (tab / P.nb) % P.nst;
  c.slab = tab / (P.nb * P.nst);
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
  if (++c.b < P.nb) return;
  c.b = 0;
  if (++c.s < P.nst) return;
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
    const int tab_id = (c.slab * kStages + c.s) * P.nb + c.b;
    if (c.g != loaded_g || tab_id != loaded_tab) {
      build_table<XDT>(G, c, tab, xs, cbs, tid);
      loaded_g = c.g;
      loaded_tab = tab_id;
    }
    const GvMat& M = P.m[c.m];
    const int row = c.tile * kGvTileRows + warp * kGvRowsPerWarp + g;
    float* part = static_cast<float*>(M.partial) + (((int64_t)c.b * kStages + c.s) * G.n_slabs + c.slab) * M.rows + row;
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

// ---------------------------------------------------------------------------
// Decode-GEMV over the tiled index layout.
//
// A unit is one 32 KiB block (stage s, slab, 512-row tile); lane (warp, g, a)
// owns rows warp*32 + 8t + g, t = 0..3, and the lane's 16 index bytes of each
// row arrive as one 16-byte load.  Each slot of the register ring holds one
// unit; a slot is refilled quarter by quarter (one row t at a time) as soon as
// that quarter has been looked up, so about NSLOT - 1/2 units per SM stay in
// flight while the lookups run.
//
// Table key of a unit: slab | s << 20 | b << 22 | group << 27 (slab < 2^20,
// s < 3, b < 32, group < 32), so one 32-bit compare detects a table switch.
__host__ __device__ __forceinline__ uint32_t table_key(int g, int slab, int s, int b) {
  return (uint32_t)slab | ((uint32_t)s << 20) | ((uint32_t)b << 22) | ((uint32_t)g << 27);
}

// Position of the next unit to load: the index block, y and the scales at the
// tile's first row, the matrix rows from that row on, the table key, and the
// coordinates needed for the carry to the next matrix or table.
struct TileCursor {
  const uint8_t* p;
  float* q;             // y of the unit's (first) token, at the tile's first row
  const uint16_t* sc;   // scales, at the tile's first row
  int32_t rows_left;
  int32_t mrows;        // rows of the matrix: y's stride from one token to the next
  int64_t pst;          // bytes from one byte plane's blocks to the next (n_slabs * plane_stride)
  uint32_t tkey;
  int32_t m, tile, ntiles;
};

__device__ __forceinline__ void tcur_fill(const GvParams& P, TileCursor& c) {
  const uint32_t k = c.tkey;
  const int slab = (int)(k & 0xFFFFFu), s = (int)((k >> 20) & 3u), b = (int)((k >> 22) & 31u), g = (int)(k >> 27);
  const GvMat& M = P.m[c.m];
  const int64_t n_slabs = P.g[g].n_slabs;
  c.ntiles = M.n_tiles;
  c.p = M.idx + ((int64_t)s * n_slabs + slab) * M.plane_stride + (int64_t)c.tile * kTileBytes;
  c.q = M.y + (int64_t)b * P.tokm * M.rows + (int64_t)c.tile * kTileRows;
  c.sc = M.scales + (int64_t)c.tile * kTileRows;
  c.rows_left = (int32_t)(M.rows - (int64_t)c.tile * kTileRows);
  c.mrows = (int32_t)M.rows;
  c.pst = n_slabs * M.plane_stride;
}

__device__ __forceinline__ TileCursor tcur_at(const GvParams& P, int64_t u) {
  const GvCursor g = unit_cursor(P, u);
  TileCursor c;
  c.tkey = table_key(g.g, g.slab, g.s, g.b);
  c.m = g.m;
  c.tile = g.tile;
  tcur_fill(P, c);
  return c;
}

// Next unit in (group, slab, stage, token, matrix, tile) order.  The common
// case, the next tile of the same matrix, is three increments.
__device__ __forceinline__ void tcur_next(const GvParams& P, TileCursor& c) {
  if (++c.tile < c.ntiles) {
    c.p += kTileBytes;
    c.q += kTileRows;
    c.sc += kTileRows;
    c.rows_left -= kTileRows;
    return;
  }
  c.tile = 0;
  int g = (int)(c.tkey >> 27);
  if (++c.m >= P.g[g].mat_end) {
    int slab = (int)(c.tkey & 0xFFFFFu), s = (int)((c.tkey >> 20) & 3u), b = (int)((c.tkey >> 22) & 31u);
    if (++b >= P.nb) {
      b = 0;
      if (++s >= P.nst) {
        s = 0;
        if (++slab >= P.g[g].n_slabs) {
          slab = 0;
          if (++g >= P.n_groups) return;  // past the last unit: never loaded
        }
      }
    }
    c.m = P.g[g].mat_begin;
    c.tkey = table_key(g, slab, s, b);
  }
  tcur_fill(P, c);
}

// Table pipeline of the tiled kernel.  A CTA walks its units table by table
// (table = group, slab, stage, token).  Table t lives in table buffer t & 1;
// its inputs (the x slab as stored and the stage's 8 KiB codebook) are
// brought into xraw[t & 1] / cb[t & 1] by bulk asynchronous copies
// completing on mbar[t & 1], issued one table ahead, so they never wait
// behind the index stream.  At the switch to table t + 1 all warps build it
// at once (each its share of the codewords, kBuildChunks pieces): spread over
// the units of table t instead, one piece per unit, the build's dependent
// chains held every warp back at the same time and cost about three times
// as much.
constexpr int kBuildChunks = 8;
constexpr int kChunkCw = kCodewords / kBuildChunks;  // 32 codewords per piece
constexpr uint32_t kNoTable = 0xFFFFFFFFu;           // no key has all bits set (group < 32, s < 3)

// Staging area of the tiled kernel's tables (inputs and barriers).
struct TilesSmem {
  float cb[2][kCodewords * kDim];                // 2 x 8 KiB
  unsigned char xraw[2][2][kSlabV * kDim * 4];   // [buffer][token of the pair] 2 KiB each (f32; 16-bit types use half)
  uint64_t mbar[2];
};
// The two 64 KiB table buffers start on a 64 KiB boundary of the shared
// address space, so that a lookup's byte permute (index byte in byte 1, bank
// offset in byte 0, table number in byte 2) is its full shared address.  The
// staging area sits below the tables when it fits there, else after them;
// 64 KiB of slack covers any placement of the dynamic shared memory.
constexpr size_t kTilesSmemBytes = 0x10000 + 2 * (size_t)kTabBytes;
// Index blocks prefetched into L2 ahead of the register ring.
constexpr int kPrefetchUnits = 2;

template <int XDT>
__host__ __device__ constexpr int x_elt_bytes() {
  return XDT == VQ3R_F32 ? 4 : 2;
}

__device__ __forceinline__ uint32_t next_table_key(const GvParams& P, uint32_t k) {
  int slab = (int)(k & 0xFFFFFu), s = (int)((k >> 20) & 3u), b = (int)((k >> 22) & 31u), g = (int)(k >> 27);
  if (++b < P.nb) return table_key(g, slab, s, b);
  b = 0;
  if (++s < P.nst) return table_key(g, slab, s, b);
  s = 0;
  if (++slab < P.g[g].n_slabs) return table_key(g, slab, s, b);
  return table_key(g + 1, 0, 0, 0);
}

// Vector columns of the slab that exist in the matrix (the last slab may be short).
__device__ __forceinline__ int slab_columns(const GvParams& P, uint32_t k) {
  const GvGroup& G = P.g[k >> 27];
  const int64_t left = G.cols / kDim - (int64_t)(k & 0xFFFFFu) * kSlabV;
  return left < kSlabV ? (int)left : kSlabV;
}

// Issued by one thread: copy table k's inputs into staging buffer i.
// Where a table's inputs come from: the x slab as stored (xbytes) and the
// stage's codebook.  Kernel parameters only, so it may run before
// griddep_wait.
struct TableSrc {
  const unsigned char* x;
  const unsigned char* x2;  // the pair's second token (two-token tables), else null
  const float* cb;
  uint32_t xbytes;
};

template <int XDT>
__device__ __forceinline__ TableSrc table_src(const GvParams& P, uint32_t k) {
  const GvGroup& G = P.g[k >> 27];
  const int slab = (int)(k & 0xFFFFFu), s = (int)((k >> 20) & 3u), b = (int)((k >> 22) & 31u);
  const int tok = b * P.tokm;
  TableSrc t;
  t.xbytes = (uint32_t)(slab_columns(P, k) * kDim * x_elt_bytes<XDT>());
  const unsigned char* xs = static_cast<const unsigned char*>(G.x) + (int64_t)slab * kSlabV * kDim * x_elt_bytes<XDT>();
  t.x = xs + (int64_t)tok * G.cols * x_elt_bytes<XDT>();
  // an odd token count leaves the last pair with one token: its second table repeats the first (never added)
  t.x2 = P.tokm == 2 ? xs + (int64_t)(tok + 1 < P.B ? tok + 1 : tok) * G.cols * x_elt_bytes<XDT>() : nullptr;
  t.cb = G.codebooks + (size_t)s * kCodewords * kDim;
  return t;
}

// Bulk copies of a table's inputs into xraw[i][..] / cb[i], completing on mbar[i].
__device__ __forceinline__ void stage_src(const TableSrc& t, TilesSmem& S, int i) {
  mbar_arrive_expect_tx(&S.mbar[i], t.xbytes * (t.x2 ? 2u : 1u) + (uint32_t)(kCodewords * kDim * 4));
  bulk_copy_g2s(S.xraw[i][0], t.x, t.xbytes, &S.mbar[i]);
  if (t.x2) bulk_copy_g2s(S.xraw[i][1], t.x2, t.xbytes, &S.mbar[i]);
  bulk_copy_g2s(S.cb[i], t.cb, kCodewords * kDim * 4, &S.mbar[i]);
}

template <int XDT>
__device__ __forceinline__ void stage_table(const GvParams& P, uint32_t k, TilesSmem& S, int i) {
  stage_src(table_src<XDT>(P, k), S, i);
}

// The 8 x values of slab column v widened to float (zero for columns past the row end).
template <int XDT>
__device__ __forceinline__ void staged_x(const unsigned char* xr, int v, int nv, float x[8]) {
  if (v >= nv) {
#pragma unroll
    for (int k = 0; k < 8; k++) x[k] = 0.0f;
    return;
  }
  if constexpr (XDT == VQ3R_F32) {
    const float4 a = reinterpret_cast<const float4*>(xr)[2 * v], b = reinterpret_cast<const float4*>(xr)[2 * v + 1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    const uint4 w = reinterpret_cast<const uint4*>(xr)[v];
    const uint32_t h[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; q++) {
      if constexpr (XDT == VQ3R_BF16) {
        x[2 * q] = bf16_bits_to_f32(h[q] & 0xFFFFu);
        x[2 * q + 1] = bf16_bits_to_f32(h[q] >> 16);
      } else {
        x[2 * q] = f16_bits_to_f32(h[q] & 0xFFFFu);
        x[2 * q + 1] = f16_bits_to_f32(h[q] >> 16);
      }
    }
  }
}

// Piece c of a table: warp w computes codewords 32c + w and 32c + w + 16 for
// slab columns lane and lane + 32 (x values xa, xb), T[v][j] = C[j] . x[v] in
// k order.
__device__ __forceinline__ void build_piece_x(float* tab, const float* cb, const float xa[8], const float xb[8],
                                              int c, int warp, int lane) {
  const float4* c4 = reinterpret_cast<const float4*>(cb);
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const int j = c * kChunkCw + warp + 16 * h;
    const float4 c0 = c4[2 * j], c1 = c4[2 * j + 1];
    const float cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    float ta = cw[0] * xa[0], tb = cw[0] * xb[0];
#pragma unroll
    for (int k = 1; k < 8; k++) {
      ta = fmaf(cw[k], xa[k], ta);
      tb = fmaf(cw[k], xb[k], tb);
    }
    tab[tab_word(lane, j)] = ta;
    tab[tab_word(lane + 32, j)] = tb;
  }
}

// Pieces c0 .. kBuildChunks - 1 of a table, the lane's x values read once.
template <int XDT>
__device__ __forceinline__ void build_pieces_from(float* tab, const float* cb, const unsigned char* xr, int nv,
                                                  int c0, int warp, int lane) {
  if (c0 >= kBuildChunks) return;
  float xa[8], xb[8];
  staged_x<XDT>(xr, lane, nv, xa);
  staged_x<XDT>(xr, lane + 32, nv, xb);
#pragma unroll 2
  for (int c = c0; c < kBuildChunks; c++) build_piece_x(tab, cb, xa, xb, c, warp, lane);
}

// ---------------------------------------------------------------------------
// Accumulation into y inside the tiled kernel.
//
// Each unit adds scale_i x (its partial sum of row i) to y[b][i] with one
// fire-and-forget atomic add in L2 (red.add.f32), so no partial sums are
// stored and no reduction pass follows the units; the order of the adds,
// and so the rounding of y, depends on scheduling.  y must be zero before the
// first add: every CTA zeroes a share of the outputs, then arrives on a grid
// barrier that is waited for only after the first table build, by when it
// has normally completed.  Every CTA of the grid must be resident at once
// (one CTA per SM, grid <= SMs), or the wait's 1 s bound fires and the call
// reports kDevErrBarrierTimeout.
//
// The barrier uses the workspace header: hdr[1] counts arrivals over all
// calls on the workspace, hdr[0] holds its value at the start of the current
// call, and the call's barrier is complete once hdr[1] - hdr[0] reaches the
// grid size.  The last CTA to arrive moves hdr[0] on for the next call (which
// starts after this grid has completed).  A zeroed header is a valid start.

// This CTA's share of the outputs to zero.  Zeroing jobs are (matrix, part)
// pairs, parts = grid / n_mats pieces of a matrix's B x rows floats (at least
// one); CTA c takes jobs c, c + grid, ...  A job touches one descriptor, so no
// CTA walks the whole descriptor list.  When the grid has at least as many
// CTAs as matrices (the usual case) a CTA has at most one job, which zero_job
// describes from the kernel parameters alone (so before griddep_wait);
// zero_rest does any further jobs.
struct ZeroJob {
  float* y;
  int64_t lo, hi;
  int m;  // the matrix
};

__device__ __forceinline__ ZeroJob zero_job(const GvParams& P, int j) {
  const int n_mats = P.n_mats, grid = (int)gridDim.x;
  const int parts = grid >= n_mats ? grid / n_mats : 1;
  ZeroJob z = {nullptr, 0, 0, 0};
  if (j < n_mats * parts) {
    const int m = j % n_mats, part = j / n_mats;
    const int64_t n = (int64_t)P.B * P.m[m].rows;
    z.y = P.m[m].y;
    z.m = m;
    z.lo = n * part / parts;
    z.hi = n * (part + 1) / parts;
  }
  return z;
}

__device__ __forceinline__ void zero_run(const ZeroJob& z, int tid) {
  for (int64_t i = z.lo + tid; i < z.hi; i += kGvThreads) z.y[i] = 0.0f;
}

__device__ __forceinline__ void zero_rest(const GvParams& P, int tid) {
  for (int j = blockIdx.x + gridDim.x; j < P.n_mats; j += gridDim.x) zero_run(zero_job(P, j), tid);
}

// Outliers (OUTL): instead of zero, y[b][i] starts as its row's outlier sum
// sum_q (float)o_iq * x[b][c_iq] (binary32, q ascending), written by the CTA
// that would zero it before the grid barrier; the lookup units then add into
// it, and the lookup loop is that of the kernel without outliers.  Eight
// words are loaded before their x values are gathered.  The words come from
// the outlier tiles (a warp's words of one q for consecutive rows are
// contiguous).  On the 8-expert decode step (14 or 4 outliers per row) this
// costs 1.16x the step without outliers; measured and slower: the same sums
// added after the CTA's last unit (1.22x, also with x staged in shared
// memory, the words prefetched into L2 and the code warmed before
// griddepcontrol.wait), one outlier per row in each lookup unit (1.25x), per
// warp chunks between units (2.4x), a second launch (1.29x), and passes over
// up to four outputs at once (all their words requested before any gather:
// inline they spill the kernel, out of line 1.27x).
template <int XDT>
__device__ __forceinline__ void outlier_init_run(const GvParams& P, const ZeroJob& z, int tid) {
  const GvMat& M = P.m[z.m];
  const int k = M.n_out;
  if (k == 0) {
    zero_run(z, tid);
    return;
  }
  const GvGroup& G = P.g[M.group];
  for (int64_t i = z.lo + tid; i < z.hi; i += kGvThreads) {
    const int64_t b = i / M.rows, row = i - b * M.rows;
    const uint32_t* p = M.otiles + (row / kTileRows) * k * kTileRows + row % kTileRows;
    float acc = 0.0f;
    for (int q0 = 0; q0 < k; q0 += 8) {
      uint32_t w8[8];
#pragma unroll
      for (int u = 0; u < 8; u++) w8[u] = q0 + u < k ? __ldg(p + (int64_t)(q0 + u) * kTileRows) : 0xFFFFFFFFu;
      float x8[8];
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const int64_t c = w8[u] & 0xFFFFu;
        x8[u] = c < G.cols ? load1<XDT>(G.x, b * G.cols + c) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 8; u++)
        if ((int64_t)(w8[u] & 0xFFFFu) < G.cols) acc = fmaf(f16_bits_to_f32((uint16_t)(w8[u] >> 16)), x8[u], acc);
    }
    z.y[i] = acc;
  }
}

// The CTA's share of y: zeros, or with OUTL the outlier sums.
template <int XDT, bool OUTL>
__device__ __forceinline__ void init_y(const GvParams& P, const ZeroJob& zj, int tid) {
  if (OUTL && P.has_out) {
    if (zj.y) outlier_init_run<XDT>(P, zj, tid);
    for (int j = blockIdx.x + gridDim.x; j < P.n_mats; j += gridDim.x) outlier_init_run<XDT>(P, zero_job(P, j), tid);
  } else {
    zero_run(zj, tid);
    zero_rest(P, tid);
  }
}

struct Arrival {
  unsigned long long start, seq;  // count at the start of the call, this CTA's place in it
};

// Arrival of this CTA, by one thread after a __syncthreads that follows the
// CTA's zeros.  The add is a release (it publishes those zeros; the acquire
// is the waiter's load), so the thread goes on without waiting for it; the
// count it returns is used only later.
__device__ __forceinline__ Arrival barrier_arrive(unsigned long long* hdr) {
  Arrival t;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(t.start) : "l"(hdr) : "memory");
  asm volatile("atom.release.gpu.global.add.u64 %0, [%1], 1;" : "=l"(t.seq) : "l"(hdr + 1) : "memory");
  return t;
}

// The last CTA to arrive (every CTA read hdr[0] before its own arrival)
// moves hdr[0] on for the next call.
__device__ __forceinline__ void barrier_close(unsigned long long* hdr, Arrival t) {
  if (t.seq - t.start == (unsigned long long)gridDim.x - 1)
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(hdr), "l"(t.start + gridDim.x) : "memory");
}

// Waits, with a 1 s bound, until all CTAs of the grid have arrived; the
// acquire load pairs with their releases.
__device__ __forceinline__ void barrier_wait(unsigned long long* hdr, Arrival t) {
  const unsigned long long grid = gridDim.x;
  barrier_close(hdr, t);
  uint64_t t0 = 0;
  for (;;) {
    unsigned long long n;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(n) : "l"(hdr + 1) : "memory");
    if (n - t.start >= grid) break;
    const uint64_t now = global_timer_ns();
    if (t0 == 0) {
      t0 = now;
    } else if (now - t0 > 1000000000ull) {
      set_device_error(kDevErrBarrierTimeout);
      break;
    }
    __nanosleep(32);
  }
}

// One table entry at a 32-bit shared address (plus 128 bytes for the second
// column slot).
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_f32_128(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+128];" : "=f"(v) : "r"(a));
  return v;
}
// The same entries of table buffer 1 (64 KiB further): the pair's second token.
__device__ __forceinline__ float lds_f32_t1(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+65536];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_f32_t1_128(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+65664];" : "=f"(v) : "r"(a));
  return v;
}

// VQ4P table entries: one 256-row table holds the four stages' 64 codewords
// (row 64 s + i), so stage s is 16 KiB further; plus 128 bytes for the second
// column slot and 64 KiB for the pair's second token.  off is a constant
// once the lookup loop is unrolled.
template <int OFF>
__device__ __forceinline__ float lds_at(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF));
  return v;
}
__device__ __forceinline__ float lds_vq4p(uint32_t a, int stage, int slot, int buf) {
  switch (buf * 8 + stage * 2 + slot) {
#define VQ4P_LDS_CASE(k) \
  case k: return lds_at<65536 * ((k) >> 3) + 16384 * (((k) >> 1) & 3) + 128 * ((k) & 1)>(a);
    VQ4P_LDS_CASE(0) VQ4P_LDS_CASE(1) VQ4P_LDS_CASE(2) VQ4P_LDS_CASE(3)
    VQ4P_LDS_CASE(4) VQ4P_LDS_CASE(5) VQ4P_LDS_CASE(6) VQ4P_LDS_CASE(7)
    VQ4P_LDS_CASE(8) VQ4P_LDS_CASE(9) VQ4P_LDS_CASE(10) VQ4P_LDS_CASE(11)
    VQ4P_LDS_CASE(12) VQ4P_LDS_CASE(13) VQ4P_LDS_CASE(14)
#undef VQ4P_LDS_CASE
    default: return lds_at<65536 + 3 * 16384 + 128>(a);
  }
}

// Shared addresses of the four table entries of one VQ4P vector.  v holds
// the vector's plane-0 byte in byte 0 and its plane-1 byte in byte 1, v2 its
// plane-1 and plane-2 bytes; with the 24-bit word w = e0 | e1 << 8 | e2 << 16
// the indices are i1 = w[0:6), i2 = w[6:12), i3 = w[12:18), i4 = w[18:24),
// so i_s << 8 is one shift and mask away: i1 = v[0:6), i2 = v[6:12),
// i3 = v2[4:10), i4 = v2[10:16).  l supplies the bank offset and the table
// base (bytes 0 and 2).
__device__ __forceinline__ void vq4p_addrs(uint32_t v, uint32_t v2, uint32_t l, uint32_t (&ad)[4]) {
  ad[0] = ((v << 8) & 0x3F00u) | l;
  ad[1] = ((v << 2) & 0x3F00u) | l;
  ad[2] = ((v2 << 4) & 0x3F00u) | l;
  ad[3] = ((v2 >> 2) & 0x3F00u) | l;
}

// Bulk prefetch of one 32 KiB index block into L2 (a hint: it reads, writes
// nothing, and may be issued before the inputs are final).
__device__ __forceinline__ void prefetch_block_l2(const void* p) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"((uint32_t)kTileBytes) : "memory");
}

__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// Table key of unit u (divisions; used once per CTA).
__device__ __forceinline__ uint32_t unit_table_key(const GvParams& P, int64_t u) {
  const GvCursor c = unit_cursor(P, u);
  return table_key(c.g, c.slab, c.s, c.b);
}

// A warp's exchange: four lanes (a = 0..3) hold partial sums of rows t = 0..3
// over their column quarters; two exchange steps leave lane a with the full
// sum of row t = a.
__device__ __forceinline__ float rows_exchange(const float (&acc)[4], bool hi2, bool hi1) {
  float k0 = hi2 ? acc[2] : acc[0], k1 = hi2 ? acc[3] : acc[1];
  const float s0 = hi2 ? acc[0] : acc[2], s1 = hi2 ? acc[1] : acc[3];
  k0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 2);
  k1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 2);
  float kk = hi1 ? k1 : k0;
  kk += __shfl_xor_sync(0xFFFFFFFFu, hi1 ? k0 : k1, 1);
  return kk;
}

// TOKS = 1: table buffers t & 1 double-buffer the tables of consecutive
// (slab, stage, token) keys.  TOKS = 2 (2 or more tokens): a key is (slab,
// stage, token pair); buffer 0 holds the pair's first token's table and
// buffer 1 the second's, so every index byte is looked up for both tokens at
// the same offset (+ 64 KiB) and the index stream is read once per pair
// instead of once per token.
// FMT = FMT_VQ4P: a slab has one table (the four stages' 64 codewords seen as
// 256 rows, built exactly as a VQ3R stage table), a unit reads the three
// byte planes of its (slab, tile) and makes four lookups per vector.
template <int XDT, int NSLOT, int TOKS, int FMT = FMT_VQ3R, bool OUTL = false>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_tiles_kernel(const __grid_constant__ GvParams P) {
  constexpr int PL = FMT == FMT_VQ4P ? 3 : 1;  // byte planes read per unit
  extern __shared__ __align__(128) unsigned char gv_smem[];
  const uint32_t sbase = smem_u32(gv_smem);
  const uint32_t tab_addr = (sbase + 0xFFFFu) & ~0xFFFFu;  // table buffer 0; buffer 1 follows at + 64 KiB
  const uint32_t pad = tab_addr - sbase;
  float* const tabp = reinterpret_cast<float*>(gv_smem + pad);
  TilesSmem& S = *reinterpret_cast<TilesSmem*>(pad >= sizeof(TilesSmem) ? gv_smem : gv_smem + pad + 2 * kTabBytes);
  const uint32_t tk = tab_addr >> 16;
  const uint32_t tab_toggle = (tk ^ (tk + 1u)) << 16;  // flips byte 2 between buffers 0 and 1

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, a = lane & 3;
  // PRMT operands: byte 0 = byte offset of the bank of the current column,
  // byte 2 = shared address of the current table buffer >> 16; the index
  // byte lands in byte 1, i.e. at j * 256.
  uint32_t lc[8];
#pragma unroll
  for (int q = 0; q < 8; q++)
    lc[q] = (tk << 16) | (4u * (8u * a + (uint32_t)((q & 3) ^ (g & 3)) + 4u * (uint32_t)((q >> 2) ^ (g >> 2))));
  uint32_t sel[4];
#pragma unroll
  for (int q = 0; q < 4; q++) sel[q] = 0x7604u | ((uint32_t)((q ^ g) & 3) << 4);
  // VQ4P: byte (q ^ g) & 3 of the first register in byte 0, of the second in byte 1
  uint32_t sel2[4];
#pragma unroll
  for (int q = 0; q < 4; q++) sel2[q] = (uint32_t)((q ^ g) & 3) | ((4u + (uint32_t)((q ^ g) & 3)) << 4);
  constexpr int kRowsPerWarpT = kTileRows / kGvWarps;  // 32: rows warp*32 + 8t + g, t = 0..3
  const int lane_off = (warp * kRowsPerWarpT + g) * kSlabV + 16 * a;
  const int out_row = warp * kRowsPerWarpT + 8 * a + g;  // row whose sum this lane holds after the reduction
  const bool hi2 = (a & 2) != 0, hi1 = (a & 1) != 0;
  const uint64_t pol = l2_policy_evict_first();

  int64_t u0 = (int64_t)blockIdx.x * P.total_units / gridDim.x;
  int64_t u1 = (int64_t)(blockIdx.x + 1) * P.total_units / gridDim.x;
  if (P.n_split == (int)gridDim.x) {  // ranges balanced by the host for units and table builds
    u0 = P.cta_begin[blockIdx.x];
    u1 = P.cta_begin[blockIdx.x + 1];
  }
  griddep_launch_dependents();
  const ZeroJob zj = zero_job(P, blockIdx.x);
  if (u0 >= u1) {  // no units: only the share of y to zero
    griddep_wait();
    init_y<XDT, OUTL>(P, zj, tid);
    __syncthreads();
    if (tid == 0) barrier_close(P.hdr, barrier_arrive(P.hdr));  // adds nothing, so it need not wait
    return;
  }
  TileCursor ci;
  uint32_t key_last;
  if (P.n_split == (int)gridDim.x) {  // start position precomputed by the host
    ci.tkey = P.cta_key0[blockIdx.x];
    ci.m = P.cta_m0[blockIdx.x];
    ci.tile = P.cta_tile0[blockIdx.x];
    tcur_fill(P, ci);
    key_last = P.cta_key_last[blockIdx.x];
  } else {
    ci = tcur_at(P, u0);
    key_last = unit_table_key(P, u1 - 1);
  }
  uint32_t key_cur = ci.tkey;
  uint32_t key_next = key_cur == key_last ? kNoTable : next_table_key(P, key_cur);
  // Everything that reads only the kernel parameters is done before
  // griddep_wait, while the preceding kernel drains.
  TableSrc src0 = {nullptr, nullptr, 0u}, src1 = {nullptr, nullptr, 0u};
  if (tid == 0) {
    mbar_init(&S.mbar[0], 1);
    mbar_init(&S.mbar[1], 1);
    src0 = table_src<XDT>(P, key_cur);
    if (key_next != kNoTable) src1 = table_src<XDT>(P, key_next);
  }
  __syncthreads();
  griddep_wait();  // inputs may be written by the preceding kernel in the stream

  // The first table's inputs arrive before the index stream is started (so
  // they do not queue behind it); its build then overlaps the first loads.
  // The outputs are zeroed while they are in flight.
  if (tid == 0) {
    stage_src(src0, S, 0);
    if (key_next != kNoTable) stage_src(src1, S, 1);
  }
  init_y<XDT, OUTL>(P, zj, tid);
  __syncthreads();  // the CTA's zeros precede its count
  Arrival arrival = {0ull, 0ull};
  if (tid == 0) arrival = barrier_arrive(P.hdr);
  bool ok = mbar_wait_bounded(&S.mbar[0], 0);

  uint4 r[NSLOT][PL][4];
  float* sq[NSLOT];
  uint32_t ssc[NSLOT];  // binary16 bits of the lane's row scale, converted when the unit's sum is added
  int32_t srows[NSLOT];
  uint32_t skey[NSLOT];
  int32_t smr[NSLOT];  // the unit's matrix rows (y's stride between the pair's tokens)
#pragma unroll
  for (int i = 0; i < NSLOT; i++) {
    if (u0 + i < u1) {
#pragma unroll
      for (int t = 0; t < 4; t++)
#pragma unroll
        for (int pl = 0; pl < PL; pl++) r[i][pl][t] = ldg_stream16(ci.p + pl * ci.pst + lane_off + t * 8 * kSlabV, pol);
      sq[i] = ci.q;
      ssc[i] = out_row < ci.rows_left ? (uint32_t)__ldg(ci.sc + out_row) : 0u;
      srows[i] = ci.rows_left;
      skey[i] = ci.tkey;
      smr[i] = ci.mrows;
      tcur_next(P, ci);
    } else {
      sq[i] = nullptr;
      ssc[i] = 0u;
      srows[i] = 0;
      skey[i] = kNoTable;
      smr[i] = 0;
    }
  }
  // L2 prefetch of the kPrefetchUnits index blocks beyond the ring; one more
  // is requested per unit after this, so the distance stays the same.
  TileCursor cpf = ci;
  int64_t upf = u0 + NSLOT;
  if (tid == 0) {
    for (int k = 0; k < kPrefetchUnits && upf < u1; k++, upf++) {
      for (int pl = 0; pl < PL; pl++) prefetch_block_l2(cpf.p + pl * cpf.pst);
      tcur_next(P, cpf);
    }
  }

  // The first table is built at once, while the first index loads are in flight.
  build_pieces_from<XDT>(tabp, S.cb[0], S.xraw[0][0], slab_columns(P, key_cur), 0, warp, lane);
  if constexpr (TOKS == 2) build_pieces_from<XDT>(tabp + kTabWords, S.cb[0], S.xraw[0][1], slab_columns(P, key_cur), 0, warp, lane);
  if (tid == 0) barrier_wait(P.hdr, arrival);  // every y is zeroed before the first add
  __syncthreads();
  int tno = 0;  // number of the current table within this CTA; it lives in table buffer tno & 1
  for (int64_t u = u0; u < u1; u += NSLOT) {
#pragma unroll
    for (int i = 0; i < NSLOT; i++) {
      if (u + i < u1) {
        if (skey[i] != key_cur) {  // switch to table tno + 1 (= key_next)
          const int nb = (tno + 1) & 1;
          ok = mbar_wait_bounded(&S.mbar[nb], (uint32_t)((tno + 1) >> 1) & 1u) && ok;
          if constexpr (TOKS == 1) {
            build_pieces_from<XDT>(tabp + nb * kTabWords, S.cb[nb], S.xraw[nb][0], slab_columns(P, key_next), 0, warp,
                                   lane);
          } else {
            __syncthreads();  // every warp is done with both buffers (the pair's tables of key_cur)
            build_pieces_from<XDT>(tabp, S.cb[nb], S.xraw[nb][0], slab_columns(P, key_next), 0, warp, lane);
            build_pieces_from<XDT>(tabp + kTabWords, S.cb[nb], S.xraw[nb][1], slab_columns(P, key_next), 0, warp, lane);
          }
          __syncthreads();  // table complete; every warp is done with table tno - 1's buffers
          tno++;
          key_cur = key_next;
          key_next = key_cur == key_last ? kNoTable : next_table_key(P, key_cur);
          if constexpr (TOKS == 1) {
#pragma unroll
            for (int q = 0; q < 8; q++) lc[q] ^= tab_toggle;
          }
          if (tid == 0 && key_next != kNoTable) {
            fence_proxy_async_smem();  // generic reads of the staging buffer precede the async refill
            stage_table<XDT>(P, key_next, S, (tno + 1) & 1);
          }
        }
        float* const q = sq[i];
        const uint32_t scale_bits = ssc[i];
        const int32_t rows_valid = srows[i];
        const bool refill = u + i + NSLOT < u1;
        const uint8_t* const pn = ci.p + lane_off;
        const int64_t pstn = ci.pst;
        const int32_t mrows = smr[i];
        const uint32_t ukey = skey[i];
        float acc[4], acc2[4];
#pragma unroll
        for (int t = 0; t < 4; t++) {
          const uint32_t w[4] = {r[i][0][t].x, r[i][0][t].y, r[i][0][t].z, r[i][0][t].w};
          float2 s2 = make_float2(0.0f, 0.0f);
          if constexpr (FMT == FMT_VQ4P) {
            const uint32_t wb[4] = {r[i][PL - 2][t].x, r[i][PL - 2][t].y, r[i][PL - 2][t].z, r[i][PL - 2][t].w};
            const uint32_t wc[4] = {r[i][PL - 1][t].x, r[i][PL - 1][t].y, r[i][PL - 1][t].z, r[i][PL - 1][t].w};
#pragma unroll
            for (int m = 0; m < 16; m++) {
              const int k = m >> 2, slot = (m >> 2) & 1;
              uint32_t ad[4];
              vq4p_addrs(__byte_perm(w[k], wb[k], sel2[m & 3]), __byte_perm(wb[k], wc[k], sel2[m & 3]),
                         lc[(m & 3) | ((m >> 3) << 2)], ad);
              if constexpr (TOKS == 1) {  // stages 1 and 3 in one half of the pair sum, 2 and 4 in the other
                s2 = __fadd2_rn(s2, make_float2(lds_vq4p(ad[0], 0, slot, 0), lds_vq4p(ad[1], 1, slot, 0)));
                s2 = __fadd2_rn(s2, make_float2(lds_vq4p(ad[2], 2, slot, 0), lds_vq4p(ad[3], 3, slot, 0)));
              } else {  // (first token, second token)
#pragma unroll
                for (int st = 0; st < 4; st++)
                  s2 = __fadd2_rn(s2, make_float2(lds_vq4p(ad[st], st, slot, 0), lds_vq4p(ad[st], st, slot, 1)));
              }
            }
            if constexpr (TOKS == 1) {
              acc[t] = s2.x + s2.y;
            } else {
              acc[t] = s2.x;
              acc2[t] = s2.y;
            }
          } else if constexpr (TOKS == 1) {
#pragma unroll
            for (int m = 0; m < 16; m += 2) {
              const uint32_t o0 = __byte_perm(w[m >> 2], lc[(m & 3) | ((m >> 3) << 2)], sel[m & 3]);
              const uint32_t o1 = __byte_perm(w[(m + 1) >> 2], lc[((m + 1) & 3) | (((m + 1) >> 3) << 2)], sel[(m + 1) & 3]);
              const float t0 = ((m >> 2) & 1) ? lds_f32_128(o0) : lds_f32(o0);
              const float t1 = (((m + 1) >> 2) & 1) ? lds_f32_128(o1) : lds_f32(o1);
              s2 = __fadd2_rn(s2, make_float2(t0, t1));
            }
            acc[t] = s2.x + s2.y;
          } else {  // (first token, second token) of the pair, summed in pairs
#pragma unroll
            for (int m = 0; m < 16; m++) {
              const uint32_t o = __byte_perm(w[m >> 2], lc[(m & 3) | ((m >> 3) << 2)], sel[m & 3]);
              const float t0 = ((m >> 2) & 1) ? lds_f32_128(o) : lds_f32(o);
              const float t1 = ((m >> 2) & 1) ? lds_f32_t1_128(o) : lds_f32_t1(o);
              s2 = __fadd2_rn(s2, make_float2(t0, t1));
            }
            acc[t] = s2.x;
            acc2[t] = s2.y;
          }
          if (refill) {
#pragma unroll
            for (int pl = 0; pl < PL; pl++) r[i][pl][t] = ldg_stream16(pn + pl * pstn + t * 8 * kSlabV, pol);
          }
        }
        if (tid == 0 && upf < u1) {  // keep kPrefetchUnits units prefetched beyond the ring
          for (int pl = 0; pl < PL; pl++) prefetch_block_l2(cpf.p + pl * cpf.pst);
          tcur_next(P, cpf);
          upf++;
        }
        if (refill) {
          sq[i] = ci.q;
          ssc[i] = out_row < ci.rows_left ? (uint32_t)__ldg(ci.sc + out_row) : 0u;
          srows[i] = ci.rows_left;
          skey[i] = ci.tkey;
          smr[i] = ci.mrows;
          tcur_next(P, ci);
        }
        const float sc = f16_bits_to_f32((uint16_t)scale_bits);
        const float kk = rows_exchange(acc, hi2, hi1);
        if (out_row < rows_valid) red_add_f32(q + out_row, sc * kk);
        if constexpr (TOKS == 2) {
          const float kk2 = rows_exchange(acc2, hi2, hi1);
          const int tok2 = 2 * (int)((ukey >> 22) & 31u) + 1;  // the pair's second token
          if (out_row < rows_valid && tok2 < P.B) red_add_f32(q + mrows + out_row, sc * kk2);
        }
      }
    }
  }
  (void)ok;  // a timed-out wait has recorded kDevErrMbarTimeout in the device error word
}

// Repack the index planes [3][rows][cols/8] (plane_stride bytes apart) into
// the tiled layout; one thread per 16-byte chunk of the output.  The chunk's 16
// source columns are contiguous in the plane: one aligned 16-byte load when V
// and plane_stride are multiples of 16 and the chunk lies inside the row,
// byte loads otherwise.  Blocks are numbered below 2^32.
__global__ void __launch_bounds__(256) pack_tiles_kernel(const uint8_t* __restrict__ idx, int64_t rows, int64_t V,
                                                          int64_t plane_stride, int32_t n_slabs, int64_t n_tiles,
                                                          uint8_t* __restrict__ out) {
  const int64_t n_chunks = (int64_t)kStages * n_slabs * n_tiles * (kTileBytes / 16);
  const bool vec = (V % 16) == 0 && (plane_stride % 16) == 0 && (reinterpret_cast<uintptr_t>(idx) % 16) == 0;
  const uint32_t nt = (uint32_t)n_tiles, ns = (uint32_t)n_slabs;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < n_chunks; q += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t blk = (uint32_t)(q >> 11);  // kTileBytes / 16 = 2048 chunks per block
    const int within = (int)(q & 2047);
    const int r = within >> 2, ch = within & 3;  // packed row, 16-byte chunk
    const uint32_t sc = blk / nt, tile = blk - sc * nt;
    const uint32_t s = sc / ns, slab = sc - s * ns;
    const int64_t row = (int64_t)tile * kTileRows + r;
    const int64_t col0 = (int64_t)slab * kSlabV + 16 * ch;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);  // the chunk's 16 columns in source order
    if (row < rows) {
      const uint8_t* src = idx + s * plane_stride + row * V + col0;
      if (vec && col0 + 16 <= V) {
        v = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        uint32_t h[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; i++) {
          const uint32_t b = col0 + i < V ? (uint32_t)__ldg(src + i) : 0u;
          h[i >> 2] |= b << (8 * (i & 3));
        }
        v = make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
    const bool swap = (r >> 2) & 1;  // rows whose two 8-byte halves are stored swapped
    reinterpret_cast<uint4*>(out)[q] = swap ? make_uint4(v.z, v.w, v.x, v.y) : v;
  }
}

// y[b][i] = scale_i * sum_s sum_slab partial[b][s][slab][i].  Two lanes share
// an output: lane k (k = 0, 1) adds partials k, k + 2, k + 4, ... in order and
// one butterfly step combines the two sums, so the order is fixed.  Each lane
// issues the loads of up to kRedPer partials before adding any, so an output
// with up to 2 * kRedPer partials costs one round trip to L2.  CTA (x, y)
// takes rows [128x, 128x + 128) of matrix y for every token.
constexpr int kRedPer = 24;
constexpr int kPlanesRedRows = 128;  // rows per CTA of the reduction kernel (256 threads)

// Sum, in order, of partials k0, k0 + 2, ... (N of them, those below np) of
// one output.  The loads are unconditional (past-the-end ones re-read the
// last partial) so that all N are in flight at once; the sum masks them.
template <int N>
__device__ __forceinline__ float sum_partials(const float* pp, int64_t stride, int np, int k0) {
  float v[N];
#pragma unroll
  for (int j = 0; j < N; j++) v[j] = __ldcg(pp + (int64_t)min(k0 + 2 * j, np - 1) * stride);
  float acc = 0.0f;
#pragma unroll
  for (int j = 0; j < N; j++)
    if (k0 + 2 * j < np) acc += v[j];
  return acc;
}

__global__ void __launch_bounds__(256) gemv_reduce_kernel(const __grid_constant__ GvParams P) {
  griddep_launch_dependents();
  const GvMat& M = P.m[blockIdx.y];
  const int64_t row = (int64_t)blockIdx.x * kPlanesRedRows + (threadIdx.x >> 1);
  if ((int64_t)blockIdx.x * kPlanesRedRows >= M.rows) return;  // past this matrix's rows (whole CTA)
  griddep_wait();  // the partial sums of the main kernel are complete
  const int sub = threadIdx.x & 1;
  const int np = kStages * P.g[M.group].n_slabs;
  const bool valid = row < M.rows;
  const float scale = valid ? f16_bits_to_f32(__ldg(M.scales + row)) : 0.0f;
  for (int b = 0; b < P.B; b++) {
    float acc = 0.0f;
    if (valid) {
      const float* pp = static_cast<const float*>(M.partial) + (int64_t)b * np * M.rows + row;
      if (np <= 16)
        acc = sum_partials<8>(pp, M.rows, np, sub);
      else
        for (int k0 = sub; k0 < np; k0 += 2 * kRedPer) acc += sum_partials<kRedPer>(pp, M.rows, np, k0);
    }
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 1);
    if (valid && sub == 0) M.y[(int64_t)b * M.rows + row] = scale * acc;
  }
}

}  // namespace vq3r
