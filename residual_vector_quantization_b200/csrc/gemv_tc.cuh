// VQ3R decode-GEMV for batches of 8..32 tokens on the fifth-generation tensor
// cores (tcgen05), with the rebuilt weights in tensor memory.
//
// Page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验", §1 (the MoE decode
// step) and §2 (W ~ scale x (C1[i1] + C2[i2] + C3[i3]) per 8-vector).  With B
// tokens the x-projected tables cost one shared-memory lookup per index byte
// and token, so beyond a few tokens it is cheaper to rebuild each weight once
// and contract it with all B tokens: y^T = W_hat x^T, a dense (rows x cols) .
// (cols x B) product.
//
// Rebuilding a weight gathers three 32-byte codewords per 8 weights from
// shared memory (12 bytes per weight); that gather is the kernel's bound.
// The rebuilt tile goes to tensor memory (tcgen05.st), which the tensor core
// reads as operand A, so it costs no further shared-memory traffic; x^T is
// operand B, staged in shared memory in the 128-byte-swizzled K-major layout.
//
// Work.  A CTA per SM, four warp-groups of four warps.  The work is the
// sequence of K-steps (128-row M-tile of a matrix, 16 columns), matrices in
// order, M-tiles in order, K-steps in order; warp-group w of the grid takes
// the w-th of 4 x grid equal contiguous pieces.  Within a piece the
// warp-group accumulates an M-tile's K-steps in tensor memory and, where the
// tile (or the piece) ends, adds scale x accumulator into y with atomic adds.
// y is zeroed first behind the same grid barrier as the lookup-table kernel
// (one CTA per SM, all resident).
//
// One K-step, per warp-group: thread t (warp q of the group, lane l) owns row
// 32q + l of the M-tile.  It rebuilds the row's 16 weights (two 8-vectors)
// in binary32 as decode does, ((C1 + C2) + C3), splits each into bf16 hi =
// rn(w) and lo = rn(w - hi) (hi + lo carries w to about 2^-16), and stores hi
// and lo into its tensor-memory lane (8 columns each).  Two K-steps make a
// super-step: after a group barrier one thread issues four tcgen05.mma
// (M = 128, N = 16 or 32, K = 16: hi.x and lo.x of each K-step, bf16 in, fp32
// accumulate) and commits them to the super-buffer's mbarrier.  Three
// super-buffers per group let the rebuild run ahead of the tensor core.  The
// K-steps of an 8-step x chunk are unrolled, so every index byte sits at a
// position known at compile time.  The row scale multiplies the fp32 sums at
// the end.
#pragma once

#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_mma.cuh"

namespace vq3r {

constexpr int kTgThreads = 512;
constexpr int kTgGroups = 4;                 // warp-groups per CTA
constexpr int kTgRows = 128;                 // M: rows of an M-tile
constexpr int kTgK = 16;                     // columns per K-step (two 8-vectors)
constexpr int kTgChunkK = 8;                 // K-steps per x chunk (128 columns)
constexpr int kTgABufs = 3;                  // A super-buffers per group (two K-steps each)
constexpr int kTgXBufs = 3;                  // x chunks per group
constexpr int kTgMaxN = 32;                  // tokens, padded to 16 or 32
constexpr int kTgMinB = 17;                  // smallest batch routed to this kernel (below it mma.sync is faster)
constexpr int kTgTmemCols = 512;             // whole tensor memory: 128 columns per group
constexpr int kTgGroupCols = kTgTmemCols / kTgGroups;
constexpr int kTgChunkBytes = kTgMaxN * kTgChunkK * kTgK * 2;  // 8 KiB: 32 tokens x 128 columns bf16

struct TgSmem {
  uint8_t xb[kTgGroups][kTgXBufs][kTgChunkBytes];    // 96 KiB, x^T chunks (operand B), 1024-byte aligned
  float cbr[kStages * kCodewords * 4 * kDim];        // 96 KiB: each codeword 4 times side by side (128-byte rows)
  uint64_t a_free[kTgGroups][kTgABufs];              // tensor core done with an A super-buffer
  uint64_t d_full[kTgGroups];                        // an M-tile's accumulator is complete
  unsigned long long arr_start, arr_seq;             // this CTA's grid-barrier arrival
  uint32_t tmem_base;
};
constexpr size_t kTgSmemBytes = sizeof(TgSmem) + 1024;  // + alignment of the x chunks to 1024 bytes

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N tokens, M = 128.
__host__ __device__ constexpr uint32_t tg_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTgRows >> 4) << 24);
}

// D (tensor memory) += A (tensor memory) x B (shared memory descriptor).
__device__ __forceinline__ void tg_mma(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The warp's 32 lanes store 8 consecutive 32-bit columns each.
__device__ __forceinline__ void tg_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ void tg_load16(uint32_t taddr, uint32_t v[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Named barrier of one warp-group (ids 1..4; 0 is __syncthreads).
__device__ __forceinline__ void tg_group_sync(int group) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + group), "r"(128) : "memory");
}

// Position in the K-step sequence: matrix, M-tile, K-step.
struct TgPos {
  int m;
  int64_t tile;  // 128-row M-tile within the matrix
  int64_t k;     // K-step within the tile
};

__device__ __forceinline__ int64_t tg_ksteps(const GvParams& P, int m) {
  return (P.g[P.m[m].group].cols / kDim + 1) / 2;  // ceil(cols / 16)
}
__device__ __forceinline__ int64_t tg_mtiles(const GvParams& P, int m) { return (P.m[m].rows + kTgRows - 1) / kTgRows; }

__device__ __forceinline__ TgPos tg_locate(const GvParams& P, int64_t q) {
  TgPos p;
  p.m = 0;
  for (;;) {
    const int64_t n = tg_mtiles(P, p.m) * tg_ksteps(P, p.m);
    if (q < n || p.m + 1 >= P.n_mats) break;
    q -= n;
    p.m++;
  }
  const int64_t nk = tg_ksteps(P, p.m);
  p.tile = q / nk;
  p.k = q - p.tile * nk;
  return p;
}

// x^T chunk of K-steps [k0, k0 + 8) of matrix group G into buffer dst:
// N token rows x 128 columns bf16 as two 64-column atoms (128-byte swizzle,
// 8-row groups 1024 bytes apart); tokens >= B and columns >= cols are zero.
template <int N>
__device__ __forceinline__ void tg_load_x(const GvGroup& G, int B, int64_t k0, uint32_t dst, int t) {
  const uint16_t* x = static_cast<const uint16_t*>(G.x);
#pragma unroll
  for (int i = 0; i < N * 16 / 128; i++) {
    const int q = t + i * 128;            // 16-byte chunk: token n, atom a, chunk c
    const int n = q >> 4, a = (q >> 3) & 1, c = q & 7;
    const int64_t col = k0 * kTgK + a * 64 + 8 * c;
    const bool ok = n < B && col < G.cols;
    cp_async16_zfill(dst + (uint32_t)(a * N * 128) + sw128_offset(n, c),
                     ok ? (const void*)(x + (int64_t)n * G.cols + col) : (const void*)x, ok ? 16u : 0u);
  }
  cp_async_commit();
}

// Index bytes of the thread's row for 8 K-steps (16 vectors) starting at K-step
// k0 (a multiple of 8): one 16-byte load per stage, halves put back in vector
// order.  Rows past the matrix read the tile's zero padding.
__device__ __forceinline__ void tg_load_idx(const GvMat& M, int n_slabs, int64_t row, int64_t k0, uint4 (&ib)[3]) {
  const int64_t tile = row / kTileRows, rr = row - tile * kTileRows;
  const int64_t slab = k0 / (kSlabV / 2), q = (k0 % (kSlabV / 2)) / kTgChunkK;
  const uint8_t* p = M.idx + slab * M.plane_stride + tile * kTileBytes + rr * kSlabV + 16 * q;
  const bool swap = ((rr >> 2) & 1) != 0;
#pragma unroll
  for (int s = 0; s < kStages; s++) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p + (int64_t)s * n_slabs * M.plane_stride));
    ib[s] = swap ? make_uint4(v.z, v.w, v.x, v.y) : v;
  }
}

template <int NT>
__global__ void __launch_bounds__(kTgThreads, 1) gemv_tc_kernel(const __grid_constant__ GvParams P) {
  constexpr int N = 16 * NT;  // tokens, padded
  extern __shared__ __align__(1024) unsigned char tg_smem_raw[];
  TgSmem& S = *reinterpret_cast<TgSmem*>(tg_smem_raw + ((1024u - (smem_u32(tg_smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp >> 2, q = warp & 3, t = tid & 127;  // warp-group, warp within it, thread within it
  const int B = P.B;

  // This warp-group's piece of the K-step sequence.
  const int64_t W = (int64_t)gridDim.x * kTgGroups, wg = (int64_t)blockIdx.x * kTgGroups + grp;
  const int64_t q0 = wg * P.total_units / W, q1 = (wg + 1) * P.total_units / W;

  if (tid == 0) {
    for (int g = 0; g < kTgGroups; g++) {
      for (int b = 0; b < kTgABufs; b++) mbar_init(&S.a_free[g][b], 1);
      mbar_init(&S.d_full[g], 1);
    }
  }
  if (warp == 0) {  // all 512 columns: 128 per warp-group (accumulator, then four A buffers of 16)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem_base)),
                 "r"(kTgTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  griddep_launch_dependents();
  griddep_wait();  // inputs may be written by the preceding kernel in the stream

  // Zero this CTA's share of y, arrive on the grid barrier (waited for before the first add).
  zero_run(zero_job(P, blockIdx.x), tid);
  zero_rest(P, tid);
  // Codeword (s, j) occupies the 128-byte row s * 256 + j, four copies of its
  // 32 bytes.  Lane l reads copy l & 3, first the half (l >> 2) & 1, so the 8
  // lanes of a quarter-warp touch 8 distinct 16-byte bank groups whatever
  // codewords they gather.  (All matrices of a call share the codebooks.)
  const float* cbg = P.g[0].codebooks;
  for (int i = tid; i < kStages * kCodewords * 4 * 2; i += kTgThreads) {
    const int half = i & 1, crow = i >> 3;  // i = (crow * 4 + copy) * 2 + half
    reinterpret_cast<float4*>(S.cbr)[i] = __ldg(reinterpret_cast<const float4*>(cbg) + 2 * crow + half);
  }
  tc_fence_before();
  __syncthreads();  // the CTA's zeros precede its count; codebooks, barriers and tensor memory are set up
  tc_fence_after();
  if (tid == 0) {
    const Arrival a = barrier_arrive(P.hdr);
    S.arr_start = a.start;
    S.arr_seq = a.seq;
  }
  __syncthreads();  // the arrival record is read by every group's first add
  const uint32_t tmem = S.tmem_base + (uint32_t)(grp * kTgGroupCols);
  const uint32_t tmem_d = tmem;                      // N accumulator columns
  const uint32_t tmem_a = tmem + kTgMaxN;            // A super-buffer b, K-step e: hi at + 32 b + 16 e, lo + 8
  const uint32_t lane_off = (uint32_t)(q * 32) << 16;
  const uint32_t xbase = smem_u32(S.xb[grp][0]);
  const float4* cbv = reinterpret_cast<const float4*>(S.cbr) + 2 * (lane & 3);  // this lane's copy
  const int h0 = (lane >> 2) & 1;                                                // its first half
  bool ok = true;
  bool waited = false;  // the grid barrier (first add of this group)

  // Pipeline state of the group (every thread holds the same values).  A
  // super-step is two K-steps: one group barrier, four MMAs, one commit.
  int ss = 0;          // super-steps issued so far
  int sb = 0;          // A super-buffer of the next one (ss % 3)
  int sround = 0;      // ss / 3: completions of that buffer's barrier to wait for, plus one
  int xslot = 0;       // x buffer of the next chunk load (rotates 0, 1, 2)
  int xl0 = -1, xl1 = -1, xl2 = -1;  // last super-step whose MMAs read each x buffer
  int64_t items = 0;   // accumulators read back by this group so far
  // Load the x chunk of K-steps [k0, k0 + 8) into the next buffer; returns it.
  // The buffer's previous contents must have been read: the MMAs of
  // super-step ss - 4 and earlier are known complete (the A-buffer wait of
  // the step before); a later reader is waited for on its own A buffer's
  // barrier (not reused since, so the phase is the latest one).
  auto load_chunk = [&](const GvGroup& G, int64_t k0) -> int {
    const int xb = xslot;
    xslot = xslot == kTgXBufs - 1 ? 0 : xslot + 1;
    const int last = xb == 0 ? xl0 : xb == 1 ? xl1 : xl2;
    if (last >= 0 && last > ss - 4)
      ok = mbar_wait_bounded(&S.a_free[grp][last % 3], (uint32_t)((last / 3) & 1)) && ok;
    tg_load_x<N>(G, B, k0, xbase + (uint32_t)(xb * kTgChunkBytes), t);
    return xb;
  };
  if (q0 < q1) {
    TgPos pos = tg_locate(P, q0);
    int64_t left = q1 - q0;
    while (left > 0) {
      const GvMat& M = P.m[pos.m];
      const GvGroup& G = P.g[M.group];
      const int64_t nk = tg_ksteps(P, pos.m);
      const int64_t kstart = pos.k;
      const int64_t kend = (nk - kstart < left) ? nk : kstart + left;  // this item: K-steps [kstart, kend)
      const int64_t row = pos.tile * kTgRows + q * 32 + lane;
      const float scale = row < M.rows ? f16_bits_to_f32(__ldg(M.scales + row)) : 0.0f;
      const int64_t V = G.cols / kDim;
      int64_t k0 = kstart - (kstart % kTgChunkK);  // x chunks and index words cover 8 K-steps from a multiple of 8
      uint4 ib[3], nb[3];
      tg_load_idx(M, G.n_slabs, row, k0, ib);
      int xcur = load_chunk(G, k0);
      for (; k0 < kend; k0 += kTgChunkK) {
        int xnext = -1;
        if (k0 + kTgChunkK < kend) {  // prefetch the next chunk's indices and x
          tg_load_idx(M, G.n_slabs, row, k0 + kTgChunkK, nb);
          xnext = load_chunk(G, k0 + kTgChunkK);
        } else {
          cp_async_commit();  // an empty group keeps the count of groups in flight the same
        }
        const uint32_t xaddr = xbase + (uint32_t)(xcur * kTgChunkBytes);
        bool xwait = true;
#pragma unroll
        for (int pp = 0; pp < kTgChunkK / 2; pp++) {
          const int64_t ka = k0 + 2 * pp;  // K-steps ka and ka + 1
          const bool in0 = ka >= kstart && ka < kend, in1 = ka + 1 >= kstart && ka + 1 < kend;
          if (!in0 && !in1) continue;
          if (sround > 0) ok = mbar_wait_bounded(&S.a_free[grp][sb], (uint32_t)((sround - 1) & 1)) && ok;
          const uint32_t abuf = tmem_a + lane_off + (uint32_t)(32 * sb);
#pragma unroll
          for (int e = 0; e < 2; e++) {
            if (!(e ? in1 : in0)) continue;
            // vectors at bytes c, c + 1 of the chunk's index words: the row's 16 weights of K-step ka + e
            const int c = 2 * (2 * pp + e);
            const bool full = 2 * (ka + e) + 1 < V;  // both vectors inside the row (else the second is zero)
            uint32_t hi[8], lo[8];
#pragma unroll
            for (int h = 0; h < 2; h++) {
              const int bb = c + h;
              const uint32_t sh = 8 * (bb & 3);
              const uint32_t j1 = (word_of(ib[0], bb >> 2) >> sh) & 0xFFu;
              const uint32_t j2 = (word_of(ib[1], bb >> 2) >> sh) & 0xFFu;
              const uint32_t j3 = (word_of(ib[2], bb >> 2) >> sh) & 0xFFu;
              const float4 ap = cbv[j1 * 8 + h0], aq = cbv[j1 * 8 + (h0 ^ 1)];
              const float4 bp = cbv[(kCodewords + j2) * 8 + h0], bq = cbv[(kCodewords + j2) * 8 + (h0 ^ 1)];
              const float4 cp = cbv[(2 * kCodewords + j3) * 8 + h0], cq = cbv[(2 * kCodewords + j3) * 8 + (h0 ^ 1)];
              float4 wp = make_float4(__fadd_rn(__fadd_rn(ap.x, bp.x), cp.x), __fadd_rn(__fadd_rn(ap.y, bp.y), cp.y),
                                      __fadd_rn(__fadd_rn(ap.z, bp.z), cp.z), __fadd_rn(__fadd_rn(ap.w, bp.w), cp.w));
              float4 wq = make_float4(__fadd_rn(__fadd_rn(aq.x, bq.x), cq.x), __fadd_rn(__fadd_rn(aq.y, bq.y), cq.y),
                                      __fadd_rn(__fadd_rn(aq.z, bq.z), cq.z), __fadd_rn(__fadd_rn(aq.w, bq.w), cq.w));
              if (h == 1 && !full) {  // a vector past the row end contributes nothing (x is zero there too)
                wp = make_float4(0.f, 0.f, 0.f, 0.f);
                wq = wp;
              }
              // weights 0..3 are half 0, 4..7 half 1 (p is half h0)
              const float4 w0 = h0 ? wq : wp, w1 = h0 ? wp : wq;
              lo[4 * h + 0] = split_bf16x2(make_float2(w0.x, w0.y), hi[4 * h + 0]);
              lo[4 * h + 1] = split_bf16x2(make_float2(w0.z, w0.w), hi[4 * h + 1]);
              lo[4 * h + 2] = split_bf16x2(make_float2(w1.x, w1.y), hi[4 * h + 2]);
              lo[4 * h + 3] = split_bf16x2(make_float2(w1.z, w1.w), hi[4 * h + 3]);
            }
            tg_st8(abuf + (uint32_t)(16 * e), hi);
            tg_st8(abuf + (uint32_t)(16 * e + 8), lo);
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          if (xwait) {  // this chunk's x has landed (the newer group may still be in flight)
            cp_async_wait<1>();
            fence_proxy_async_smem();  // x, written by the generic proxy, is read by the tensor core
            xwait = false;
          }
          tc_fence_before();
          tg_group_sync(grp);
          if (t == 0) {
            tc_fence_after();
#pragma unroll
            for (int e = 0; e < 2; e++) {
              if (!(e ? in1 : in0)) continue;
              const int kk = 2 * pp + e;  // K-step within the chunk
              const uint64_t bd = sw128_desc(xaddr + (uint32_t)((kk >> 2) * N * 128)) + (uint64_t)(2 * (kk & 3));
              const uint32_t at = tmem_a + (uint32_t)(32 * sb + 16 * e);
              tg_mma(tmem_d, at, bd, tg_idesc(N), ka + e != kstart ? 1u : 0u);
              tg_mma(tmem_d, at + 8u, bd, tg_idesc(N), 1u);
            }
            tc_commit(&S.a_free[grp][sb]);
            if (ka + 1 >= kend - 1) tc_commit(&S.d_full[grp]);  // the item's last K-step is in this pair
          }
          if (xcur == 0) xl0 = ss;
          else if (xcur == 1) xl1 = ss;
          else xl2 = ss;
          ss++;
          if (++sb == 3) {
            sb = 0;
            sround++;
          }
        }
        if (xnext >= 0) {
#pragma unroll
          for (int st = 0; st < kStages; st++) ib[st] = nb[st];
          xcur = xnext;
        }
      }
      // Read the accumulator back: this thread's row, N tokens; add scale x sum into y.
      ok = mbar_wait_bounded(&S.d_full[grp], (uint32_t)(items & 1)) && ok;
      items++;
      tc_fence_after();
      uint32_t v[32];
      tg_load16(tmem_d + lane_off, v);
      if (N > 16) tg_load16(tmem_d + lane_off + 16u, v + 16);
      tc_fence_before();
      if (!waited) {  // every y is zeroed before this group's first add
        if (t == 0) barrier_wait(P.hdr, Arrival{S.arr_start, S.arr_seq});
        tg_group_sync(grp);
        waited = true;
      }
      if (row < M.rows) {
#pragma unroll
        for (int bt = 0; bt < N; bt++)
          if (bt < B) red_add_f32(M.y + (int64_t)bt * M.rows + row, scale * __uint_as_float(v[bt]));
      }
      left -= kend - kstart;
      // next item: the next M-tile (or matrix) from its first K-step
      if (kend == nk) {
        pos.k = 0;
        if (++pos.tile == tg_mtiles(P, pos.m)) {
          pos.tile = 0;
          pos.m++;
        }
      } else {
        pos.k = kend;
      }
    }
  }
  if (!waited && tid == 0) barrier_close(P.hdr, Arrival{S.arr_start, S.arr_seq});  // added nothing
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(S.tmem_base), "r"(kTgTmemCols));
  }
  (void)ok;  // a timed-out wait has recorded kDevErrMbarTimeout in the device error word
}

}  // namespace vq3r
