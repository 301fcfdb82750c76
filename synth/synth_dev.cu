/* Device side of the seeded input generator (see synth_gen.h); bulk inputs
 * for large workloads.  Same header as the host side, compiled with
 * -fmad=false. */
#include <cuda_runtime.h>
#include "synth_gen.h"

__global__ void synth_fill_kernel(void* out, int out_dtype, int64_t cols, int64_t row0, int64_t nrows,
                                  uint64_t seed, uint32_t tag, synth_dist d) {
  int64_t total = nrows * cols;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = i / cols, c = i - r * cols;
    int64_t row = row0 + r;
    double rowf = synth_row_factor(seed, tag, (uint64_t)row, d.row_sigma);
    float f = synth_round_f32(synth_value(seed, tag, cols, row, c, &d, rowf));
    if (out_dtype == SYNTH_OUT_BF16) ((uint16_t*)out)[i] = synth_f32_to_bf16(f);
    else ((float*)out)[i] = f;
  }
}

extern "C" int synth_fill_rows_device(void* out, int out_dtype, int64_t cols, int64_t row0, int64_t nrows,
                                      uint64_t seed, uint32_t tag, const synth_dist* d, void* stream) {
  if (!out || cols <= 0 || nrows < 0 || !d) return 1;
  if (nrows == 0) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 2;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 2;
  synth_fill_kernel<<<sms * 8, 256, 0, (cudaStream_t)stream>>>(out, out_dtype, cols, row0, nrows, seed, tag, *d);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
