// VQ3R prefill product on the fifth-generation tensor cores (tcgen05):
//   Y[t][i] = sum_c bf16(w_hat[i][c]) * x[t][c],  x bf16 [T][cols], Y fp32 [T][rows],
// w_hat = scale_i * ((C1[i1] + C2[i2]) + C3[i3]) in binary32 (as vq3r_decode
// writes it), rounded to bfloat16 for the bf16 tensor-core product.
//
// Page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验", §1 (MoE
// expert weights stored at 3 bits) and §2 (the reconstruction rule).  The
// pages give no batched product; this is the many-token counterpart of the
// decode-step GEMV, for prompts (prefill), where the weights are rebuilt once
// per CTA and used for 256 tokens.
//
// One CTA computes 128 weight rows x 256 tokens over all columns, in steps
// of 64 columns (one 128-byte swizzle atom of bf16 per row):
//   - all 512 threads rebuild the step's 128 x 64 weights from the tiled
//     indices and the shared-memory codebooks, round them to bf16 and store
//     them in the K-major 128-byte-swizzled layout the tensor core reads
//     (operand A, two buffers);
//   - cp.async brings the step's 256 x 64 x tile into the same layout one
//     step ahead (operand B, three buffers; zeros past the token and column
//     ends);
//   - one thread issues four tcgen05.mma (M = 128, N = 256, K = 16, bf16 in,
//     fp32 accumulate) into tensor memory and commits them to the buffer's
//     mbarrier, which the rebuild of the step after next waits for;
//   - at the end, sixteen warps read the accumulators back (tcgen05.ld) and
//     store Y, one token per store instruction across 32 consecutive rows.
#pragma once

#include <cuda_bf16.h>

#include "gemv.cuh"
#include "vq3r_common.cuh"

namespace vq3r {

constexpr int kTcRows = 128;     // M: weight rows per CTA
constexpr int kTcTokens = 256;   // N: tokens per CTA
constexpr int kTcK = 64;         // columns per step
constexpr int kTcThreads = 512;
constexpr int kTcParts = kTcThreads / kTcRows;   // threads per weight row: 4
constexpr int kTcVecs = 8 / kTcParts;            // 8-vectors per thread and step: 2
constexpr int kTcBStages = 3;
constexpr int kTcTmemCols = 256;  // fp32 accumulator columns (one per token)

struct GmMat {
  const uint8_t* idx;       // tiled layout
  const uint16_t* scales;
  const float* codebooks;
  const uint16_t* x;        // bf16 [tokens][cols]
  float* y;                 // [tokens][rows]
  int64_t rows, cols, tokens, plane_stride;
  int64_t cta_begin;        // first CTA of this matrix
  int32_t n_slabs;          // ceil(cols / 512)
  int32_t tok_tiles;        // ceil(tokens / 256)
};

struct GemmParams {
  GmMat m[VQ3R_GEMV_MAX_MATS];
  int32_t n_mats;
  int64_t total_ctas;
};

struct TcSmem {
  uint8_t a[2][kTcRows * 128];            // 2 x 16 KiB, rebuilt weights
  uint8_t b[kTcBStages][kTcTokens * 128];  // 3 x 32 KiB, x tiles
  float cbr[kStages * kCodewords * 4 * kDim];  // 96 KiB: each codeword 4 times side by side (128-byte rows)
  uint64_t mma_done[2];
  uint32_t tmem_base;
};
constexpr size_t kTcSmemBytes = sizeof(TcSmem) + 1024;  // + alignment of the tiles to 1024 bytes

// Byte offset of 16-byte chunk c (0..7) of row r in a K-major tile with the
// 128-byte swizzle: 8-row groups 1024 bytes apart, rows 128 bytes apart,
// chunk c stored at position c ^ (r mod 8).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor of such a tile (start 1024-byte aligned):
// start address, leading byte offset 16 (unused by swizzled K-major
// layouts), stride byte offset 1024 between 8-row groups, descriptor
// version 1, swizzle mode 2 (128 bytes).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kTcInstrDesc =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcTokens >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kTcInstrDesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(mbar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive accumulator columns of the warp's 32 lanes (one row per lane).
__device__ __forceinline__ void tc_load32(uint32_t taddr, uint32_t v[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16-byte global -> shared asynchronous copy; src_bytes 0 writes zeros.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmParams P) {
  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  TcSmem& S = *reinterpret_cast<TcSmem*>(tc_smem_raw + ((1024u - (smem_u32(tc_smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // This CTA's matrix, 128-row block and 256-token tile (tiles fastest).
  const int64_t cta = blockIdx.x;
  int m = 0;
  while (m + 1 < P.n_mats && P.m[m + 1].cta_begin <= cta) m++;
  const GmMat& M = P.m[m];
  const int64_t local = cta - M.cta_begin;
  const int64_t rb = local / M.tok_tiles, tt = local - rb * M.tok_tiles;
  const int64_t row0 = rb * kTcRows, tok0 = tt * kTcTokens;
  const int64_t V = M.cols / kDim;
  const int n_steps = (int)((M.cols + kTcK - 1) / kTcK);

  // Rebuild role: row r of the block, vectors kTcVecs * part .. of each step.
  const int r = tid & (kTcRows - 1), part = tid >> 7;
  const int64_t row = row0 + r;
  const int64_t rr = row & (kTileRows - 1), tile = row / kTileRows;
  const uint32_t rowsel = (uint32_t)((rr >> 2) & 1);

  if (tid == 0) {
    mbar_init(&S.mma_done[0], 1);
    mbar_init(&S.mma_done[1], 1);
  }
  if (warp == 0) {  // the accumulator: 128 lanes x 256 fp32 columns of tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem_base)),
                 "r"(kTcTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  griddep_launch_dependents();
  griddep_wait();  // inputs may be written by the preceding kernel in the stream

  // Codeword (s, j) occupies the 128-byte row s * 256 + j, four copies of its
  // 32 bytes.  Lane l reads copy l & 3, first the half (l >> 2) & 1, so the 8
  // lanes of a quarter-warp touch 8 distinct 16-byte bank groups whatever
  // codewords they gather (one copy left random rows conflicting).
  for (int i = tid; i < kStages * kCodewords * 4 * 2; i += kTcThreads) {
    const int half = i & 1, row = i >> 3;  // i = (row * 4 + copy) * 2 + half
    reinterpret_cast<float4*>(S.cbr)[i] = __ldg(reinterpret_cast<const float4*>(M.codebooks) + 2 * row + half);
  }
  const float scale = row < M.rows ? f16_bits_to_f32(__ldg(M.scales + row)) : 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  // Index bytes of step k: the thread's kTcVecs vectors (2 bytes) of each stage.
  auto load_idx = [&](int k, uint32_t ib[kStages]) {
    const int slab = k >> 3, kc = k & 7;
    const int64_t off =
        tile * kTileBytes + rr * kSlabV + 16 * (kc >> 1) + 8 * ((uint32_t)(kc & 1) ^ rowsel) + kTcVecs * part;
#pragma unroll
    for (int s = 0; s < kStages; s++)
      ib[s] = __ldg(reinterpret_cast<const uint16_t*>(M.idx + ((int64_t)s * M.n_slabs + slab) * M.plane_stride + off));
  };
  // x tile of step k into b[stage]: 256 tokens x 8 chunks of 16 bytes, 4 chunks per thread.
  auto load_x = [&](int k, int stage) {
    const uint32_t base = smem_u32(S.b[stage]);
#pragma unroll
    for (int i = 0; i < kTcTokens * 8 / kTcThreads; i++) {
      const int q = tid + i * kTcThreads, n = q >> 3, c = q & 7;
      const int64_t tok = tok0 + n, col = (int64_t)k * kTcK + 8 * c;
      const bool ok = tok < M.tokens && col < M.cols;
      cp_async16_zfill(base + sw128_offset(n, c), ok ? (const void*)(M.x + tok * M.cols + col) : (const void*)M.x,
                       ok ? 16u : 0u);
    }
    cp_async_commit();
  };

  uint32_t ib[kStages];
  load_idx(0, ib);
  load_x(0, 0);
  bool ok = true;
  const float4* cbv = reinterpret_cast<const float4*>(S.cbr) + 2 * (lane & 3);  // this lane's copy
  const int h0 = (lane >> 2) & 1;                                                // its first half
  for (int k = 0; k < n_steps; k++) {
    const int ab = k & 1, bs = k % kTcBStages;
    if (k >= 2)  // the MMAs of step k - 2 are done with a[ab] and b[(k + 1) % 3]
      ok = mbar_wait_bounded(&S.mma_done[ab], (uint32_t)((k - 2) >> 1) & 1u) && ok;
    if (k + 1 < n_steps) load_x(k + 1, (k + 1) % kTcBStages);

    // Rebuild: w = scale * ((C1 + C2) + C3) in binary32, rounded to bf16.
    const uint32_t abase = smem_u32(S.a[ab]);
#pragma unroll
    for (int e = 0; e < kTcVecs; e++) {
      const int c = kTcVecs * part + e;  // the vector's 16-byte chunk in the row
      const int64_t v = (int64_t)k * 8 + c;
      const uint32_t j1 = (ib[0] >> (8 * e)) & 0xFFu, j2 = (ib[1] >> (8 * e)) & 0xFFu, j3 = (ib[2] >> (8 * e)) & 0xFFu;
      // p: the half this lane reads first (h0), q: the other one
      const float4 ap = cbv[(0 * kCodewords + j1) * 8 + h0], aq = cbv[(0 * kCodewords + j1) * 8 + (h0 ^ 1)];
      const float4 bp = cbv[(1 * kCodewords + j2) * 8 + h0], bq = cbv[(1 * kCodewords + j2) * 8 + (h0 ^ 1)];
      const float4 cp = cbv[(2 * kCodewords + j3) * 8 + h0], cq = cbv[(2 * kCodewords + j3) * 8 + (h0 ^ 1)];
      const float sv = v < V ? scale : 0.0f;
      const uint32_t p01 = pack_bf16x2_rn(__fmul_rn(sv, __fadd_rn(__fadd_rn(ap.x, bp.x), cp.x)),
                                          __fmul_rn(sv, __fadd_rn(__fadd_rn(ap.y, bp.y), cp.y)));
      const uint32_t p23 = pack_bf16x2_rn(__fmul_rn(sv, __fadd_rn(__fadd_rn(ap.z, bp.z), cp.z)),
                                          __fmul_rn(sv, __fadd_rn(__fadd_rn(ap.w, bp.w), cp.w)));
      const uint32_t q01 = pack_bf16x2_rn(__fmul_rn(sv, __fadd_rn(__fadd_rn(aq.x, bq.x), cq.x)),
                                          __fmul_rn(sv, __fadd_rn(__fadd_rn(aq.y, bq.y), cq.y)));
      const uint32_t q23 = pack_bf16x2_rn(__fmul_rn(sv, __fadd_rn(__fadd_rn(aq.z, bq.z), cq.z)),
                                          __fmul_rn(sv, __fadd_rn(__fadd_rn(aq.w, bq.w), cq.w)));
      // weights 0..3 are the half-0 values, 4..7 the half-1 values
      const uint4 pk = h0 ? make_uint4(q01, q23, p01, p23) : make_uint4(p01, p23, q01, q23);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(abase + sw128_offset(r, c)), "r"(pk.x),
                   "r"(pk.y), "r"(pk.z), "r"(pk.w)
                   : "memory");
    }
    if (k + 1 < n_steps) load_idx(k + 1, ib);
    if (k + 1 < n_steps) cp_async_wait<1>();  // this step's x tile has landed
    else cp_async_wait<0>();
    fence_proxy_async_smem();  // the tiles, written by the generic proxy, are read by the tensor core
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint64_t ad = sw128_desc(abase), bd = sw128_desc(smem_u32(S.b[bs]));
#pragma unroll
      for (int kk = 0; kk < kTcK / 16; kk++)  // K = 16 per instruction: 32 bytes further along the rows
        tc_mma(tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), (k | kk) != 0 ? 1u : 0u);
      tc_commit(&S.mma_done[ab]);
    }
  }
  // The last step's MMAs (and with them all earlier ones) are complete.
  ok = mbar_wait_bounded(&S.mma_done[(n_steps - 1) & 1], (uint32_t)((n_steps - 1) >> 1) & 1u) && ok;
  tc_fence_after();

  // Epilogue: warp w reads lanes 32 (w mod 4) .. (its rows) and columns
  // 64 (w / 4) .. (its tokens), 32 at a time.
  const int q = warp & 3, cgrp = warp >> 2;
  const int64_t orow = row0 + q * 32 + lane;
#pragma unroll 1
  for (int cc = 0; cc < kTcTokens / (kTcThreads / 128) / 32; cc++) {
    const int col = cgrp * (kTcTokens / (kTcThreads / 128)) + cc * 32;
    uint32_t v[32];
    tc_load32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)col, v);
    if (orow < M.rows) {
#pragma unroll
      for (int j = 0; j < 32; j++) {
        const int64_t tok = tok0 + col + j;
        if (tok < M.tokens) M.y[tok * M.rows + orow] = __uint_as_float(v[j]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols));
  }
  (void)ok;  // a timed-out wait has recorded kDevErrMbarTimeout in the device error word
}

}  // namespace vq3r
