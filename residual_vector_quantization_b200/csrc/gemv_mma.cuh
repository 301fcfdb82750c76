// VQ3R decode-GEMV for batches of tokens on the tensor cores: reconstruct the
// weight tile, then multiply.
//
// Page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验", §1 (the MoE decode
// step) and §2 (W ~ scale x (C1[i1] + C2[i2] + C3[i3]) per 8-vector).  With B
// tokens the x-projected tables cost one shared-memory lookup per index byte
// and token, so beyond a few tokens it is cheaper to rebuild the weights once
// and contract them with all B tokens at once: y^T = W_hat x^T is a dense
// (rows x cols) . (cols x B) product.
//
// Layout of the work.  A CTA of 16 warps owns 256 rows of one matrix and walks
// all its columns, so it writes y directly (no partial sums).  Warp w owns rows
// 16w .. 16w + 15 of the CTA's block; per 16 columns (two 8-vectors) it
// contracts a 16 x 16 tile of reconstructed weights with x on mma.sync
// m16n8k16 (bf16 inputs, fp32 accumulation), one instruction per 8 tokens.
//
// Reconstruction in registers.  Lane (g, t) of the m16n8k16 A fragment holds
// columns 2t, 2t+1 and 2t+8, 2t+9 of rows g and g+8, i.e. elements 2t, 2t+1 of
// the two 8-vectors of each of its two rows.  It reads exactly those two
// elements of each stage's codeword (one 8-byte shared load from the fp32
// codebook; the four lanes of a row read one whole 32-byte codeword between
// them) and adds the stages as decode does, ((C1 + C2) + C3) in fp32.  Each
// value w is then split into bf16 hi = rn(w) and lo = rn(w - hi); the two
// products hi.x + lo.x carry w to about 2^-16 relative, so the result keeps
// fp32-class accuracy.  x is bf16 and exact.  The row scale is applied to the
// fp32 sums at the end, as in the other kernels.
//
// Index bytes come from the tiled layout (512-row x 64-column blocks): the four
// lanes of a row group load the same 16 bytes (one sector for the warp), two
// rows and three stages per 16-vector chunk.
#pragma once

#include "gemv.cuh"

namespace vq3r {

constexpr int kMmaWarps = 16;
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kMmaRows = kMmaWarps * 16;            // rows per CTA
constexpr int kMmaMaxTok = VQ3R_GEMV_MAX_B;         // 32 tokens = 4 n-tiles
constexpr int kXCols = kSlabV * kDim;               // 512 columns of x per slab
constexpr int kXStride = kXCols + 8;                // bf16 per token row in shared memory (padding: no bank conflicts)
constexpr int kMmaMinB = 11;                        // smallest bf16 batch routed to the tensor cores (below: two-token tables)

// Codebooks: each codeword stored four times side by side in a 128-byte row,
// cb[s][j][r][k] = C_s[j][k].  Row group g reads copy g mod 4, so the 16 lanes
// of a half-warp (four row groups x four 8-byte pieces) hit 16 distinct bank
// pairs whatever the indices are.
struct MmaSmem {
  float cb[kStages][kCodewords][4][kDim];           // 96 KiB
  uint16_t xs[2][kMmaMaxTok][kXStride];             // 2 x 32 x 520 bf16 = 65 KiB, x of one slab (double buffer)
};
constexpr size_t kMmaSmemBytes = sizeof(MmaSmem);

// Pack two floats into bf16x2, low half = a.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

// hi = rn_bf16(a, b); returns lo = rn_bf16(a - hi.a, b - hi.b).
__device__ __forceinline__ uint32_t split_bf16x2(float2 w, uint32_t& hi) {
  hi = pack_bf16x2(w.x, w.y);
  const float2 r = __fadd2_rn(w, make_float2(-__uint_as_float(hi << 16), -__uint_as_float(hi & 0xFFFF0000u)));
  return pack_bf16x2(r.x, r.y);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Issue the asynchronous copies of x[b][col0 .. col0 + 512) for b < B into
// buffer xs (16 bytes per copy); columns past the row end are zeroed.
__device__ __forceinline__ void stage_x_slab(const uint16_t* x, int64_t cols, int B, int64_t col0, uint16_t (*xs)[kXStride],
                                             int tid) {
  const int64_t left = cols - col0;
  const int chunks = (int)((left < kXCols ? left : kXCols) / 8);  // 16-byte pieces per token row
  for (int i = tid; i < B * (kXCols / 8); i += kMmaThreads) {
    const int b = i / (kXCols / 8), c = i - b * (kXCols / 8);
    if (c < chunks) {
      const uint16_t* src = x + (int64_t)b * cols + col0 + 8 * c;
      const uint32_t dst = smem_u32(&xs[b][8 * c]);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    } else {  // past the row end (last slab): zero, whatever an earlier slab left there
      *reinterpret_cast<uint4*>(&xs[b][8 * c]) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Reconstructed weights of (row, vector) from one index byte per stage: the
// lane's two elements 2t, 2t+1 of ((C1[e0] + C2[e1]) + C3[e2]).
// The codebooks are written once, before the CTA barrier that precedes every
// call, so the loads need no ordering beyond their address inputs.
__device__ __forceinline__ float2 rebuild2(uint32_t cb_lane, uint32_t e0, uint32_t e1, uint32_t e2) {
  float2 c0, c1, c2;
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(c0.x), "=f"(c0.y) : "r"(cb_lane + e0 * 128u));
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(c1.x), "=f"(c1.y) : "r"(cb_lane + 32768u + e1 * 128u));
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(c2.x), "=f"(c2.y) : "r"(cb_lane + 65536u + e2 * 128u));
  return __fadd2_rn(__fadd2_rn(c0, c1), c2);
}

// Load the lane's index bytes of one 16-vector chunk: rows a (= g) and b (= g + 8)
// of the warp's 16, stages 0..2; halves put back in vector order.
__device__ __forceinline__ void load_chunk(const uint8_t* pa, int64_t plane_stride, bool swap, uint4 (&ia)[3],
                                           uint4 (&ib)[3]) {
#pragma unroll
  for (int s = 0; s < kStages; s++) {
    uint4 va = __ldg(reinterpret_cast<const uint4*>(pa + s * plane_stride));
    uint4 vb = __ldg(reinterpret_cast<const uint4*>(pa + s * plane_stride + 8 * kSlabV));
    ia[s] = swap ? make_uint4(va.z, va.w, va.x, va.y) : va;
    ib[s] = swap ? make_uint4(vb.z, vb.w, vb.x, vb.y) : vb;
  }
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int q) {
  return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

// Blocks of kMmaRows rows: matrix m owns blocks blk_begin[m] .. (filled by the host for this kernel).
template <int NT>
__global__ void __launch_bounds__(kMmaThreads, 1) gemv_mma_kernel(const __grid_constant__ GvParams P) {
  extern __shared__ __align__(128) unsigned char mma_smem[];
  MmaSmem& S = *reinterpret_cast<MmaSmem*>(mma_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const int blk = blockIdx.x;
  int m = 0;
  while (m + 1 < P.n_mats && P.m[m + 1].blk_begin <= blk) m++;
  const GvMat& M = P.m[m];
  const GvGroup& G = P.g[M.group];
  const int64_t row0 = (int64_t)(blk - M.blk_begin) * kMmaRows + warp * 16;  // the warp's 16 rows
  griddep_launch_dependents();
  griddep_wait();  // inputs may be written by the preceding kernel in the stream

  const int B = P.B;
  for (int i = tid; i < kStages * kCodewords * kDim / 4; i += kMmaThreads) {  // i: one half codeword
    const float4 v = __ldg(reinterpret_cast<const float4*>(G.codebooks) + i);
    const int sj = i >> 1, half = i & 1;
#pragma unroll
    for (int r = 0; r < 4; r++) reinterpret_cast<float4*>(&S.cb[0][0][0][0])[(sj * 4 + r) * 2 + half] = v;
  }
  for (int i = tid; i < (int)(sizeof(S.xs) / 16); i += kMmaThreads) reinterpret_cast<uint4*>(&S.xs[0][0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();  // zeros in place before any copy lands
  const uint16_t* x = static_cast<const uint16_t*>(G.x);
  const int n_slabs = G.n_slabs;
  stage_x_slab(x, G.cols, B, 0, S.xs[0], tid);

  // The warp's rows lie in one 512-row tile; lane rows a = row0 + g and b = a + 8.
  const int64_t tile = row0 / kTileRows;
  const int rin = (int)(row0 - tile * kTileRows) + g;
  const bool swap = ((rin >> 2) & 1) != 0;  // stored with halves swapped (same for rows a and b)
  const uint8_t* const rowp = M.idx + tile * kTileBytes + (int64_t)rin * kSlabV;
  const uint32_t cb_lane = smem_u32(&S.cb[0][0][0][0]) + 32u * (g & 3) + 8u * t;
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; n++) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;

  for (int slab = 0; slab < n_slabs; slab++) {
    const int buf = slab & 1;
    if (slab + 1 < n_slabs) stage_x_slab(x, G.cols, B, (int64_t)(slab + 1) * kXCols, S.xs[buf ^ 1], tid);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();  // x of this slab is in S.xs[buf]
    const uint8_t* pa = rowp + (int64_t)slab * M.plane_stride;  // stage 0 of this slab; stage s at + s * n_slabs * plane_stride
    const int64_t sstride = (int64_t)n_slabs * M.plane_stride;
    uint4 ia[3], ib[3], na[3], nb[3];
    load_chunk(pa, sstride, swap, ia, ib);
#pragma unroll 1
    for (int c = 0; c < 4; c++) {
      if (c + 1 < 4) load_chunk(pa + 16 * (c + 1), sstride, swap, na, nb);
#pragma unroll
      for (int kk = 0; kk < 8; kk++) {
        const int q = 2 * (kk >> 2) + ((kk & 3) >> 1), sh = 16 * (kk & 1);
        uint32_t e[2][3][2];  // [row a/b][stage][vector 0/1]
#pragma unroll
        for (int st = 0; st < kStages; st++) {
          const uint32_t wa = word_of(ia[st], q), wb = word_of(ib[st], q);
          e[0][st][0] = (wa >> sh) & 0xFFu;
          e[0][st][1] = (wa >> (sh + 8)) & 0xFFu;
          e[1][st][0] = (wb >> sh) & 0xFFu;
          e[1][st][1] = (wb >> (sh + 8)) & 0xFFu;
        }
        const float2 wa0 = rebuild2(cb_lane, e[0][0][0], e[0][1][0], e[0][2][0]);
        const float2 wb0 = rebuild2(cb_lane, e[1][0][0], e[1][1][0], e[1][2][0]);
        const float2 wa1 = rebuild2(cb_lane, e[0][0][1], e[0][1][1], e[0][2][1]);
        const float2 wb1 = rebuild2(cb_lane, e[1][0][1], e[1][1][1], e[1][2][1]);
        uint32_t hi[4], lo[4];
        lo[0] = split_bf16x2(wa0, hi[0]);  // row a, columns 2t, 2t+1
        lo[1] = split_bf16x2(wb0, hi[1]);  // row b
        lo[2] = split_bf16x2(wa1, hi[2]);  // row a, columns 2t+8, 2t+9
        lo[3] = split_bf16x2(wb1, hi[3]);  // row b
        const int kc = 128 * c + 16 * kk + 2 * t;   // column of x within the slab
#pragma unroll
        for (int n = 0; n < NT; n++) {
          const uint16_t* xr = &S.xs[buf][8 * n + g][kc];
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(xr), b1 = *reinterpret_cast<const uint32_t*>(xr + 8);
          mma_bf16_16816(acc[n], hi, b0, b1);
          mma_bf16_16816(acc[n], lo, b0, b1);
        }
      }
      if (c + 1 < 4) {
#pragma unroll
        for (int st = 0; st < kStages; st++) {
          ia[st] = na[st];
          ib[st] = nb[st];
        }
      }
    }
    __syncthreads();  // every warp is done with S.xs[buf] before it is refilled
  }

  // acc[n]: rows a (c0, c1) and b (c2, c3), tokens 8n + 2t and 8n + 2t + 1.
  const int64_t ra = row0 + g, rb = ra + 8;
  const float sa = ra < M.rows ? f16_bits_to_f32(__ldg(M.scales + ra)) : 0.0f;
  const float sb = rb < M.rows ? f16_bits_to_f32(__ldg(M.scales + rb)) : 0.0f;
#pragma unroll
  for (int n = 0; n < NT; n++) {
    const int b0 = 8 * n + 2 * t, b1 = b0 + 1;
    if (ra < M.rows) {
      if (b0 < B) M.y[(int64_t)b0 * M.rows + ra] = sa * acc[n][0];
      if (b1 < B) M.y[(int64_t)b1 * M.rows + ra] = sa * acc[n][1];
    }
    if (rb < M.rows) {
      if (b0 < B) M.y[(int64_t)b0 * M.rows + rb] = sb * acc[n][2];
      if (b1 < B) M.y[(int64_t)b1 * M.rows + rb] = sb * acc[n][3];
    }
  }
}

}  // namespace vq3r
