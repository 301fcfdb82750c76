// VQ3R codebook training on the GPU: Lloyd k-means per stage, stage s on the
// residuals left by stage s - 1.
//
// Page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验", §2 and §4:
// each layer's codebooks are fitted by Lloyd iterations on vectors sampled
// from its experts, stage by stage on the residuals.  Readings (the page
// leaves them open): initial centroids = the first 256 training vectors;
// assignment by the encoder's distance (every binary32 operation rounded,
// k ascending) and tie rule (lowest index); centroid = binary64 sum of the
// members' components in training order, divided by the count, rounded to
// binary32; an empty cluster keeps its centroid; a fixed number of
// iterations; residual r - C[a] in binary32 after the last assignment.
//
// Kernels per iteration:
//   train_assign_kernel  nearest centroid of every vector (one thread per
//                        vector, centroids in shared memory) and its squared
//                        distance in binary64 for the distortion trace,
//                        summed per CTA;
//   train_update_kernel  one warp per centroid: it scans the assignments in
//                        training order 32 at a time (ballot), and lanes 0..7
//                        add the members' components k = lane in that order,
//                        so the binary64 sums are the sequential ones;
//   train_residual_kernel  r -= C[a] after the stage's last assignment.
#pragma once

#include "vq3r_common.cuh"

namespace vq3r {

constexpr int kTrainThreads = 256;
constexpr int kTrainUpdateWarps = 8;  // centroids per CTA of the update kernel

// a[i] = nearest of the K centroids to vector i; part[blockIdx.x] = binary64
// sum over the CTA's vectors of their squared distance to it (for the trace).
// K = 256 (VQ3R) or 64 (VQ4P).
template <int K>
__global__ void __launch_bounds__(kTrainThreads) train_assign_kernel(const float* __restrict__ R, int64_t n,
                                                                     const float* __restrict__ C,
                                                                     int32_t* __restrict__ a, double* __restrict__ part) {
  __shared__ float cs[K * kDim];
  __shared__ double red[kTrainThreads / 32];
  for (int i = threadIdx.x; i < K * kDim; i += kTrainThreads) cs[i] = C[i];
  __syncthreads();
  double acc = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * kTrainThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kTrainThreads) {
    float r[kDim];
    const float4 r0 = __ldg(reinterpret_cast<const float4*>(R + i * kDim));
    const float4 r1 = __ldg(reinterpret_cast<const float4*>(R + i * kDim) + 1);
    r[0] = r0.x; r[1] = r0.y; r[2] = r0.z; r[3] = r0.w;
    r[4] = r1.x; r[5] = r1.y; r[6] = r1.z; r[7] = r1.w;
    float best = __int_as_float(0x7F800000);
    int bi = 0;
#pragma unroll 4
    for (int j = 0; j < K; j++) {
      const float* c = cs + j * kDim;  // broadcast reads
      float e = __fsub_rn(r[0], c[0]);
      float d = __fmul_rn(e, e);
#pragma unroll
      for (int k = 1; k < kDim; k++) {
        e = __fsub_rn(r[k], c[k]);
        d = __fadd_rn(d, __fmul_rn(e, e));
      }
      if (d < best) {
        best = d;
        bi = j;
      }
    }
    a[i] = bi;
    double dist = 0.0;
#pragma unroll
    for (int k = 0; k < kDim; k++) {
      const double e = (double)r[k] - (double)cs[bi * kDim + k];
      dist = __dadd_rn(dist, __dmul_rn(e, e));
    }
    acc = __dadd_rn(acc, dist);
  }
  // fixed-order CTA sum (the trace is compared with a tolerance, not bit for bit)
  for (int o = 16; o > 0; o >>= 1) acc = __dadd_rn(acc, __shfl_down_sync(0xFFFFFFFFu, acc, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kTrainThreads / 32; w++) t = __dadd_rn(t, red[w]);
    part[blockIdx.x] = t;
  }
}

// Centroid j = blockIdx.x * kTrainUpdateWarps + warp: the binary64 mean of its
// members in training order, rounded to binary32 (unchanged when empty).
template <int K>
__global__ void __launch_bounds__(kTrainUpdateWarps * 32) train_update_kernel(const float* __restrict__ R, int64_t n,
                                                                              const int32_t* __restrict__ a,
                                                                              float* __restrict__ C) {
  const int lane = threadIdx.x & 31, j = blockIdx.x * kTrainUpdateWarps + (threadIdx.x >> 5);
  if (j >= K) return;
  double sum = 0.0;  // component k = lane (lanes 0..7)
  int64_t cnt = 0;
  constexpr int kChunks = 8;  // 256 assignments per round, their loads all in flight
  for (int64_t base = 0; base < n; base += 32 * kChunks) {
    int32_t av[kChunks];
#pragma unroll
    for (int q = 0; q < kChunks; q++) {
      const int64_t i = base + 32 * q + lane;
      av[q] = i < n ? __ldg(a + i) : -1;
    }
#pragma unroll
    for (int q = 0; q < kChunks; q++) {  // vectors base + 32 q + lane, in training order
      unsigned m = __ballot_sync(0xFFFFFFFFu, av[q] == j);
      cnt += __popc(m);
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1;
        if (lane < kDim) sum = __dadd_rn(sum, (double)__ldg(R + (base + 32 * q + b) * kDim + lane));
      }
    }
  }
  if (cnt > 0 && lane < kDim) C[j * kDim + lane] = __double2float_rn(__ddiv_rn(sum, (double)cnt));
}

// r -= C[a] in binary32 (the residual the next stage trains on).
__global__ void __launch_bounds__(kTrainThreads) train_residual_kernel(float* __restrict__ R, int64_t n,
                                                                       const float* __restrict__ C,
                                                                       const int32_t* __restrict__ a) {
  const int64_t total = n * kDim;
  for (int64_t t = (int64_t)blockIdx.x * kTrainThreads + threadIdx.x; t < total; t += (int64_t)gridDim.x * kTrainThreads) {
    const int64_t i = t / kDim;
    const int k = (int)(t - i * kDim);
    R[t] = __fsub_rn(R[t], __ldg(C + __ldg(a + i) * kDim + k));
  }
}

// trace = sum of the per-CTA partials, in CTA order.
__global__ void train_trace_kernel(const double* __restrict__ part, int nparts, double* __restrict__ out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    double t = 0.0;
    for (int p = 0; p < nparts; p++) t = __dadd_rn(t, part[p]);
    *out = t;
  }
}

}  // namespace vq3r
