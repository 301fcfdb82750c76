// C ABI of the VQ3R library (declared in include/vq3r.h): argument checks,
// launch configuration and status codes.  All arithmetic runs in the
// kernels of encode.cuh, decode.cuh and gemv.cuh.
#include <atomic>
#include <mutex>

#include "decode.cuh"
#include "encode.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_mma.cuh"
#include "gemv_tc.cuh"
#include "train.cuh"
#include "outliers.cuh"
#include "vq3r_common.cuh"

using namespace vq3r;

namespace {

thread_local int t_last_cuda_error = 0;

vq3r_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = (int)e;
  return VQ3R_ERR_CUDA;
}

vq3r_status check_launch() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? VQ3R_OK : cuda_fail(e);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int d) { return d == VQ3R_F32 || d == VQ3R_BF16 || d == VQ3R_F16; }

vq3r_status check_shape(int64_t rows, int64_t cols, int64_t min_rows) {
  if (rows < min_rows || cols < kDim || cols % kDim) return VQ3R_ERR_SHAPE;
  if (rows > 0 && cols > INT64_MAX / 8 / rows) return VQ3R_ERR_SHAPE;
  return VQ3R_OK;
}

// Per-device launch setup: SM count and the dynamic shared-memory opt-ins.
constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
std::atomic<bool> g_dev_ready[kMaxDevices];  // set once a setup has succeeded; a failed one is retried
int g_dev_sms[kMaxDevices];
// The tiled GEMV waits on a grid barrier, so every one of its CTAs (at most
// one per SM) must be resident at once: a CTA must fit on an SM next to
// nothing else.  Checked once per device with the occupancy calculator.
bool g_dev_tiles_fit[kMaxDevices];
bool g_dev_tc_fit[kMaxDevices];  // the same for the tensor-core GEMV (one persistent CTA per SM, grid barrier)

constexpr int kNumTilesKernels = 18;  // instantiations of gemv_tiles_kernel (occupancy-checked together)

cudaError_t device_setup(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (g_dev_ready[dev].load(std::memory_order_acquire)) {
    *sms = g_dev_sms[dev];
    return cudaSuccess;
  }
  std::lock_guard<std::mutex> lock(g_dev_mu);
  {
    cudaError_t r = cudaDeviceGetAttribute(&g_dev_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    const int enc = (int)sizeof(EncSmem);
    const int gv = (int)kGvSmemBytes;
    const int gt = (int)kTilesSmemBytes;
    if (r == cudaSuccess) r = cudaFuncSetAttribute(encode_kernel<VQ3R_F32, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, enc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(encode_kernel<VQ3R_BF16, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, enc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(encode_kernel<VQ3R_F16, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, enc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(encode_kernel<VQ3R_F32, FMT_VQ4P>, cudaFuncAttributeMaxDynamicSharedMemorySize, enc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(encode_kernel<VQ3R_BF16, FMT_VQ4P>, cudaFuncAttributeMaxDynamicSharedMemorySize, enc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(encode_kernel<VQ3R_F16, FMT_VQ4P>, cudaFuncAttributeMaxDynamicSharedMemorySize, enc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_lut_kernel<VQ3R_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, gv);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_lut_kernel<VQ3R_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, gv);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_lut_kernel<VQ3R_F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, gv);
    const void* tiles_kernels[kNumTilesKernels] = {
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F32, kTileSlots, 1>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_BF16, kTileSlots, 1>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F16, kTileSlots, 1>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F32, kTileSlots, 2>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_BF16, kTileSlots, 2>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F16, kTileSlots, 2>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F32, 1, 1, FMT_VQ4P>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_BF16, 1, 1, FMT_VQ4P>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F16, 1, 1, FMT_VQ4P>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F32, 1, 2, FMT_VQ4P>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_BF16, 1, 2, FMT_VQ4P>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F16, 1, 2, FMT_VQ4P>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F32, kTileSlots, 1, FMT_VQ3R, true>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_BF16, kTileSlots, 1, FMT_VQ3R, true>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F16, kTileSlots, 1, FMT_VQ3R, true>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F32, kTileSlots, 2, FMT_VQ3R, true>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_BF16, kTileSlots, 2, FMT_VQ3R, true>),
        reinterpret_cast<const void*>(gemv_tiles_kernel<VQ3R_F16, kTileSlots, 2, FMT_VQ3R, true>)};
    for (int k = 0; k < kNumTilesKernels && r == cudaSuccess; k++)
      r = cudaFuncSetAttribute(tiles_kernels[k], cudaFuncAttributeMaxDynamicSharedMemorySize, gt);
    const int gm = (int)kMmaSmemBytes;
    const int gc = (int)(kCbrFloats * sizeof(float));
    if (r == cudaSuccess) r = cudaFuncSetAttribute(decode_bulk_kernel<VQ3R_F32, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)decode_bulk_smem<FMT_VQ3R>());
    if (r == cudaSuccess) r = cudaFuncSetAttribute(decode_bulk_kernel<VQ3R_F16, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)decode_bulk_smem<FMT_VQ3R>());
    if (r == cudaSuccess) r = cudaFuncSetAttribute(decode_bulk_kernel<VQ3R_F32, FMT_VQ4P>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)decode_bulk_smem<FMT_VQ4P>());
    if (r == cudaSuccess) r = cudaFuncSetAttribute(decode_bulk_kernel<VQ3R_F16, FMT_VQ4P>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)decode_bulk_smem<FMT_VQ4P>());
    if (r == cudaSuccess) r = cudaFuncSetAttribute(decode_kernel<VQ3R_F32, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, gc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(decode_kernel<VQ3R_F16, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, gc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(relfro_partial_kernel<VQ3R_F32, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, gc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(relfro_partial_kernel<VQ3R_BF16, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, gc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(relfro_partial_kernel<VQ3R_F16, FMT_VQ3R>, cudaFuncAttributeMaxDynamicSharedMemorySize, gc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(relfro_partial_kernel<VQ3R_F32, FMT_VQ3R, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, gc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(relfro_partial_kernel<VQ3R_BF16, FMT_VQ3R, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, gc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(relfro_partial_kernel<VQ3R_F16, FMT_VQ3R, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, gc);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, gm);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_mma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, gm);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_mma_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, gm);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_mma_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, gm);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmemBytes);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTgSmemBytes);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(gemv_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTgSmemBytes);
    const int go = (int)outlier_select_smem(kOutMaxCols);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(outlier_select_kernel<VQ3R_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, go);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(outlier_select_kernel<VQ3R_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, go);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(outlier_select_kernel<VQ3R_F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, go);
    if (r != cudaSuccess) return r;
    int fit = 1;
    for (int k = 0; k < kNumTilesKernels && r == cudaSuccess; k++) {
      int n = 0;
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, tiles_kernels[k], kGvThreads, gt);
      if (n < 1) fit = 0;
    }
    if (r != cudaSuccess) return r;
    g_dev_tiles_fit[dev] = fit != 0;
    int ntc1 = 0, ntc2 = 0;
    r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ntc1, gemv_tc_kernel<1>, kTgThreads, kTgSmemBytes);
    if (r == cudaSuccess) r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ntc2, gemv_tc_kernel<2>, kTgThreads, kTgSmemBytes);
    if (r != cudaSuccess) return r;
    g_dev_tc_fit[dev] = ntc1 >= 1 && ntc2 >= 1;
  }
  g_dev_ready[dev].store(true, std::memory_order_release);
  *sms = g_dev_sms[dev];
  return cudaSuccess;
}

constexpr size_t kWsAlign = 256;
constexpr size_t kWsHeaderBytes = 256;  // GEMV workspace header, see plan_gemv
size_t align_up(size_t x) { return (x + kWsAlign - 1) / kWsAlign * kWsAlign; }

constexpr int kErrMaxBlocks = 4096;

// ---- GEMV schedule (host) ----

struct GemvPlan {
  GvParams P;
  size_t ws_bytes;
};

// Groups matrices sharing (codebooks, x, cols), lays out the workspace and
// numbers the work units.  Matrices are stored grouped (each group's
// matrices contiguous in P.m); empty matrices are dropped.
// tokm: tokens per table token (2 for the tiled kernel's two-token tables, else 1).
// nst: table stages per slab, 3 for VQ3R, 1 for VQ4P (its four 64-codeword
// stages share one 256-entry table).  outl (tiled kernel only, may be null):
// the matrices' sparse outlier residuals, whose sums start y.
vq3r_status plan_gemv(const vq3r_gemv_desc* mats, int n_mats, int B, int tokm, char* ws_base, GemvPlan* plan,
                      int nst = kStages, const vq3r_outlier_tiles* outl = nullptr) {
  GvParams& P = plan->P;
  memset(&P, 0, sizeof(P));
  P.B = B;
  P.tokm = tokm;
  P.nb = (B + tokm - 1) / tokm;
  P.nst = nst;
  P.vec8 = 1;
  P.layout = mats[0].layout;
  if (P.layout != VQ3R_LAYOUT_PLANES && P.layout != VQ3R_LAYOUT_TILES) return VQ3R_ERR_SHAPE;
  const bool tiles = P.layout == VQ3R_LAYOUT_TILES;
  P.tile_rows = tiles ? kTileRows : kGvTileRows;
  int n_groups = 0;
  int group_of[VQ3R_GEMV_MAX_MATS];
  for (int i = 0; i < n_mats; i++) {
    const vq3r_gemv_desc& d = mats[i];
    vq3r_status st = check_shape(d.rows, d.cols, 0);
    if (st != VQ3R_OK) return st;
    if (d.cols / kDim > (int64_t)kSlabV * (1 << 20) || d.rows >= ((int64_t)1 << 31)) return VQ3R_ERR_SHAPE;
    if (d.layout != P.layout || d.reserved != 0) return VQ3R_ERR_SHAPE;
    const int64_t plane = tiles ? (d.rows + kTileRows - 1) / kTileRows * kTileBytes : d.rows * (d.cols / kDim);
    if (d.plane_stride != 0 && (d.plane_stride < plane || (tiles && d.plane_stride % kTileBytes))) return VQ3R_ERR_SHAPE;
    group_of[i] = -1;
    if (d.rows == 0) continue;  // an empty matrix may carry NULL pointers
    if (!d.idx || !d.scales || !d.codebooks || !d.x || !d.y) return VQ3R_ERR_NULL;
    if (!aligned16(d.idx) || !aligned16(d.scales) || !aligned16(d.codebooks) || !aligned16(d.x) || !aligned16(d.y))
      return VQ3R_ERR_ALIGN;
    const int64_t stride = d.plane_stride ? d.plane_stride : plane;
    // 64-bit index loads need 8-byte aligned rows and planes; otherwise bytes are loaded one by one
    if ((d.cols / kDim) % 8 || (stride & 7)) P.vec8 = 0;
    int g = 0;
    while (g < n_groups && !(P.g[g].codebooks == d.codebooks && P.g[g].x == d.x && P.g[g].cols == d.cols)) g++;
    if (g == n_groups) {
      P.g[g].codebooks = d.codebooks;
      P.g[g].x = d.x;
      P.g[g].cols = d.cols;
      P.g[g].n_slabs = (int32_t)((d.cols / kDim + kSlabV - 1) / kSlabV);
      n_groups++;
    }
    group_of[i] = g;
  }
  P.n_groups = n_groups;
  int nm = 0;
  for (int g = 0; g < n_groups; g++) {
    P.g[g].mat_begin = (int16_t)nm;
    P.g[g].tiles = 0;
    for (int i = 0; i < n_mats; i++) {
      if (group_of[i] != g) continue;
      const vq3r_gemv_desc& d = mats[i];
      GvMat& M = P.m[nm++];
      M.idx = d.idx;
      M.scales = d.scales;
      M.y = d.y;
      M.rows = d.rows;
      M.plane_stride = d.plane_stride ? d.plane_stride
                                      : (tiles ? (d.rows + kTileRows - 1) / kTileRows * kTileBytes
                                               : d.rows * (d.cols / kDim));
      M.group = g;
      M.otiles = outl ? outl[i].otiles : nullptr;
      M.n_out = outl ? (int32_t)outl[i].k : 0;
      M.n_tiles = (int32_t)((d.rows + P.tile_rows - 1) / P.tile_rows);
      M.tile_prefix = P.g[g].tiles;
      P.g[g].tiles += M.n_tiles;
    }
    P.g[g].mat_end = (int16_t)nm;
  }
  P.n_mats = nm;
  // The workspace opens with a header (the tiled kernel's grid-barrier
  // arrival counts), kept apart from the planes kernel's partial sums so
  // that calls of either layout may share a workspace.
  P.hdr = reinterpret_cast<unsigned long long*>(ws_base);
  size_t off = kWsHeaderBytes;
  int64_t units = 0;
  for (int g = 0; g < n_groups; g++) {
    GvGroup& G = P.g[g];
    G.unit_begin = units;
    units += (int64_t)G.n_slabs * P.nst * P.nb * G.tiles;
  }
  // Partial sums of the planes kernel: one float per (token, stage, slab,
  // row).  The tiled kernels add into y directly and need only the header.
  for (int i = 0; i < nm; i++) {
    GvMat& M = P.m[i];
    M.partial = tiles ? nullptr : ws_base + off;
    if (!tiles) off = align_up(off + (size_t)B * kStages * P.g[M.group].n_slabs * (size_t)M.rows * sizeof(float));
  }
  P.total_units = units;
  for (int i = 0; i < nm; i++) P.has_out |= P.m[i].n_out > 0;
  plan->ws_bytes = off;
  return VQ3R_OK;
}

// Split the tiled kernel's units into n contiguous CTA ranges that balance
// cost = units + kTableCost * tables built, a table being the (group, slab,
// stage, token) run of G.tiles consecutive units.  Binary search on the
// largest range cost; for a given budget, ranges are filled greedily table by
// table.  Writes P.cta_begin[0..n] and P.n_split = n (ranges past the last
// unit are empty).
constexpr int64_t kTableCost = 2;  // a table build at a switch, and its stall, cost about two units

int64_t split_ranges(const GvParams& P, int64_t budget, int n, int64_t* begin) {
  int used = 0;
  int64_t unit = 0, cost = budget;  // cost of the open range; budget forces a new range first
  for (int g = 0; g < P.n_groups; g++) {
    const GvGroup& G = P.g[g];
    const int64_t n_tables = (int64_t)G.n_slabs * P.nst * P.nb;
    for (int64_t t = 0; t < n_tables; t++) {
      int64_t left = G.tiles;
      bool fresh = true;  // this table not yet charged to the open range
      while (left > 0) {
        if (cost + (fresh ? kTableCost : 0) + 1 > budget) {  // open a new range here
          if (begin && used <= n) begin[used] = unit;
          used++;
          cost = 0;
          fresh = true;
        }
        if (fresh) {
          cost += kTableCost;
          fresh = false;
        }
        int64_t take = budget - cost;
        if (take > left) take = left;
        if (take < 1) take = 1;
        cost += take;
        unit += take;
        left -= take;
      }
    }
  }
  return used;
}

void balance_split(GvParams& P, int n) {
  P.n_split = 0;
  if (n < 1 || n > kMaxSplit) return;
  int64_t lo = (P.total_units + n - 1) / n + kTableCost;  // no range can cost less
  int64_t hi = P.total_units + kTableCost * P.total_units;  // one range holds everything
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if (split_ranges(P, mid, n, nullptr) <= n) hi = mid;
    else lo = mid + 1;
  }
  const int64_t used = split_ranges(P, lo, n, P.cta_begin);
  for (int64_t c = used; c <= n; c++) P.cta_begin[c] = P.total_units;
  for (int c = 0; c < n; c++) {
    P.cta_key0[c] = P.cta_key_last[c] = 0;
    P.cta_m0[c] = P.cta_tile0[c] = 0;
    if (P.cta_begin[c] >= P.cta_begin[c + 1]) continue;  // no units
    const GvCursor first = unit_cursor(P, P.cta_begin[c]);
    const GvCursor last = unit_cursor(P, P.cta_begin[c + 1] - 1);
    P.cta_key0[c] = table_key(first.g, first.slab, first.s, first.b);
    P.cta_m0[c] = first.m;
    P.cta_tile0[c] = first.tile;
    P.cta_key_last[c] = table_key(last.g, last.slab, last.s, last.b);
  }
  P.n_split = n;
}

// Launch of the tiled lookup-table GEMV, one CTA per SM.  The kernel's grid
// barrier needs all CTAs resident at once; the cooperative launch attribute
// would guarantee it but measured 3.8 us slower per call (it gives up most of
// the programmatic-launch overlap), so the grid is sized to one CTA per SM
// and the fit of one CTA per SM is checked instead.
template <int FMT, int NSLOT, bool OUTL = false>
vq3r_status launch_tiles(GemvPlan& plan, vq3r_dtype x_dtype, int sms, cudaLaunchConfig_t& cfg) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!g_dev_tiles_fit[dev]) return cuda_fail(cudaErrorCooperativeLaunchTooLarge);
  GvParams& P = plan.P;
  const int grid = (int)(P.total_units < (int64_t)sms ? P.total_units : (int64_t)sms);
  balance_split(P, grid);
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = kTilesSmemBytes;
  if (P.tokm == 2) {
    switch (x_dtype) {
      case VQ3R_F32: e = cudaLaunchKernelEx(&cfg, gemv_tiles_kernel<VQ3R_F32, NSLOT, 2, FMT, OUTL>, P); break;
      case VQ3R_BF16: e = cudaLaunchKernelEx(&cfg, gemv_tiles_kernel<VQ3R_BF16, NSLOT, 2, FMT, OUTL>, P); break;
      default: e = cudaLaunchKernelEx(&cfg, gemv_tiles_kernel<VQ3R_F16, NSLOT, 2, FMT, OUTL>, P); break;
    }
  } else {
    switch (x_dtype) {
      case VQ3R_F32: e = cudaLaunchKernelEx(&cfg, gemv_tiles_kernel<VQ3R_F32, NSLOT, 1, FMT, OUTL>, P); break;
      case VQ3R_BF16: e = cudaLaunchKernelEx(&cfg, gemv_tiles_kernel<VQ3R_BF16, NSLOT, 1, FMT, OUTL>, P); break;
      default: e = cudaLaunchKernelEx(&cfg, gemv_tiles_kernel<VQ3R_F16, NSLOT, 1, FMT, OUTL>, P); break;
    }
  }
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();  // the tiled kernel adds its sums into y itself
}

template <int DT, int FMT>
vq3r_status launch_encode(const void* W, int64_t rows, int64_t cols, const float* cb, uint8_t* idx,
                          uint16_t* scales, cudaStream_t s, int sms) {
  const int64_t nvec = rows * (cols / kDim);
  const int g1 = (int)(rows < (int64_t)sms * 16 ? rows : (int64_t)sms * 16);
  row_scale_kernel<DT><<<g1, kScaleThreads, 0, s>>>(W, rows, cols, scales);
  const int64_t ntiles = (nvec + enc_tile<FMT>() - 1) / enc_tile<FMT>();
  const int g2 = (int)(ntiles < (int64_t)sms * 2 ? ntiles : (int64_t)sms * 2);
  encode_kernel<DT, FMT><<<g2, kEncThreads, sizeof(EncSmem), s>>>(W, cols, nvec, cb, scales, idx, 0.0f);
  return check_launch();
}

// CTAs for the row-split decode and error kernels: two per SM (96 KiB of
// replicated codebooks each), more when a CTA's share of 4-vector groups
// would not fit 32 bits; never more than rows or cap.
int64_t rowsplit_blocks(int64_t rows, int64_t cols, int sms, int64_t cap) {
  int64_t blocks = 2 * (int64_t)sms;
  // the error kernel counts a CTA's 4-vector groups in 32 bits
  const int64_t need = rows * ((cols / kDim + kErrVecs - 1) / kErrVecs) / ((int64_t)1 << 30) + 1;
  if (blocks < need) blocks = need;
  if (blocks > cap) blocks = cap;
  if (blocks > rows) blocks = rows;
  return blocks;
}

template <int DT, int FMT>
vq3r_status launch_relfro(const void* W, const uint8_t* idx, const uint16_t* scales, const float* cb, int64_t rows,
                          int64_t cols, double* err_out, double* partial, cudaStream_t s, int sms) {
  const int64_t blocks = rowsplit_blocks(rows, cols, sms, kErrMaxBlocks);
  relfro_partial_kernel<DT, FMT><<<(int)blocks, kErrThreads, fmt_cbr_floats<FMT>() * sizeof(float), s>>>(
      W, idx, scales, cb, rows, cols, partial);
  relfro_final_kernel<<<1, 256, 0, s>>>(partial, (int)blocks, err_out);
  return check_launch();
}

template <int FMT>
vq3r_status encode_entry(const void* W, vq3r_dtype w_dtype, int64_t rows, int64_t cols, const float* codebooks,
                         uint8_t* idx, uint16_t* scales, vq3r_stream stream) {
  vq3r_status st = check_shape(rows, cols, 0);
  if (st != VQ3R_OK) return st;
  if (!valid_dtype(w_dtype)) return VQ3R_ERR_DTYPE;
  if (rows == 0) return VQ3R_OK;
  if (!W || !codebooks || !idx || !scales) return VQ3R_ERR_NULL;
  if (!aligned16(W) || !aligned16(codebooks) || !aligned16(idx) || !aligned16(scales)) return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (w_dtype) {
    case VQ3R_F32: return launch_encode<VQ3R_F32, FMT>(W, rows, cols, codebooks, idx, scales, s, sms);
    case VQ3R_BF16: return launch_encode<VQ3R_BF16, FMT>(W, rows, cols, codebooks, idx, scales, s, sms);
    default: return launch_encode<VQ3R_F16, FMT>(W, rows, cols, codebooks, idx, scales, s, sms);
  }
}

template <int FMT>
vq3r_status decode_entry(const uint8_t* idx, const uint16_t* scales, const float* codebooks, int64_t rows,
                         int64_t cols, void* out, vq3r_dtype out_dtype, vq3r_stream stream) {
  vq3r_status st = check_shape(rows, cols, 0);
  if (st != VQ3R_OK) return st;
  if (out_dtype != VQ3R_F32 && out_dtype != VQ3R_F16) return VQ3R_ERR_DTYPE;
  if (rows == 0) return VQ3R_OK;
  if (!idx || !scales || !codebooks || !out) return VQ3R_ERR_NULL;
  if (!aligned16(idx) || !aligned16(scales) || !aligned16(codebooks) || !aligned16(out)) return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nvec = rows * (cols / kDim);
  if (nvec % 16 == 0) {  // index tiles staged by bulk copies (16-byte aligned planes)
    const int64_t ntiles = (nvec + kDecTileV - 1) / kDecTileV;
    const int grid = (int)(ntiles < 2 * (int64_t)sms ? ntiles : 2 * (int64_t)sms);
    const size_t smem = decode_bulk_smem<FMT>();
    if (out_dtype == VQ3R_F32)
      decode_bulk_kernel<VQ3R_F32, FMT><<<grid, kDecThreads, smem, s>>>(idx, scales, codebooks, rows, cols, out);
    else
      decode_bulk_kernel<VQ3R_F16, FMT><<<grid, kDecThreads, smem, s>>>(idx, scales, codebooks, rows, cols, out);
    return check_launch();
  }
  const int64_t blocks = rowsplit_blocks(rows, cols, sms, (int64_t)1 << 30);
  const size_t smem = fmt_cbr_floats<FMT>() * sizeof(float);
  if (out_dtype == VQ3R_F32)
    decode_kernel<VQ3R_F32, FMT><<<(int)blocks, kDecThreads, smem, s>>>(idx, scales, codebooks, rows, cols, out);
  else
    decode_kernel<VQ3R_F16, FMT><<<(int)blocks, kDecThreads, smem, s>>>(idx, scales, codebooks, rows, cols, out);
  return check_launch();
}

template <int FMT>
vq3r_status relfro_entry(const void* W, vq3r_dtype w_dtype, const uint8_t* idx, const uint16_t* scales,
                         const float* codebooks, int64_t rows, int64_t cols, double* err_out, void* workspace,
                         size_t ws_bytes, vq3r_stream stream) {
  if (!W || !idx || !scales || !codebooks || !err_out) return VQ3R_ERR_NULL;
  vq3r_status st = check_shape(rows, cols, 1);
  if (st != VQ3R_OK) return st;
  if (!valid_dtype(w_dtype)) return VQ3R_ERR_DTYPE;
  if (!workspace || ws_bytes < vq3r_rel_frobenius_workspace_size(rows, cols)) return VQ3R_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(idx) || !aligned16(scales) || !aligned16(codebooks) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(err_out) & 7u))
    return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* partial = static_cast<double*>(workspace);
  switch (w_dtype) {
    case VQ3R_F32: return launch_relfro<VQ3R_F32, FMT>(W, idx, scales, codebooks, rows, cols, err_out, partial, s, sms);
    case VQ3R_BF16: return launch_relfro<VQ3R_BF16, FMT>(W, idx, scales, codebooks, rows, cols, err_out, partial, s, sms);
    default: return launch_relfro<VQ3R_F16, FMT>(W, idx, scales, codebooks, rows, cols, err_out, partial, s, sms);
  }
}

int train_grid(int64_t n, int sms) {
  const int64_t need = (n + kTrainThreads - 1) / kTrainThreads;
  return (int)(need < 2 * (int64_t)sms ? need : 2 * (int64_t)sms);
}

// residuals [n][8] float, assignments [n] int32, per-CTA trace partials (at most 2 per SM, 1024 SMs)
size_t train_ws_bytes(int64_t n) {
  return align_up((size_t)n * kDim * sizeof(float)) + align_up((size_t)n * sizeof(int32_t)) + 2048 * sizeof(double);
}

// Lloyd training of S stages of K codewords (VQ3R: 3 x 256, VQ4P: 4 x 64).
template <int S, int K>
vq3r_status train_entry(const float* vecs, int64_t n, int iters, int nstages, float* codebooks, double* trace,
                        void* workspace, size_t ws_bytes, vq3r_stream stream) {
  if (!vecs || !codebooks) return VQ3R_ERR_NULL;
  if (n < K || n > ((int64_t)1 << 40) || iters < 0 || nstages < 1 || nstages > S) return VQ3R_ERR_SHAPE;
  if (!workspace || ws_bytes < train_ws_bytes(n)) return VQ3R_ERR_WORKSPACE;
  if (!aligned16(vecs) || !aligned16(codebooks) || !aligned16(workspace) || (trace && !aligned16(trace)))
    return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  if (sms > 1024) return VQ3R_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(workspace);
  float* R = reinterpret_cast<float*>(w);
  int32_t* a = reinterpret_cast<int32_t*>(w + align_up((size_t)n * kDim * sizeof(float)));
  double* part = reinterpret_cast<double*>(w + align_up((size_t)n * kDim * sizeof(float)) + align_up((size_t)n * sizeof(int32_t)));
  const int grid = train_grid(n, sms);
  e = cudaMemcpyAsync(R, vecs, (size_t)n * kDim * sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e);
  for (int st = 0; st < nstages; st++) {
    float* C = codebooks + (size_t)st * K * kDim;
    e = cudaMemcpyAsync(C, R, (size_t)K * kDim * sizeof(float), cudaMemcpyDeviceToDevice, s);  // first K
    if (e != cudaSuccess) return cuda_fail(e);
    for (int it = 0; it <= iters; it++) {
      train_assign_kernel<K><<<grid, kTrainThreads, 0, s>>>(R, n, C, a, part);
      if (trace) train_trace_kernel<<<1, 32, 0, s>>>(part, grid, trace + (size_t)st * (iters + 1) + it);
      if (it == iters) break;
      train_update_kernel<K><<<K / kTrainUpdateWarps, kTrainUpdateWarps * 32, 0, s>>>(R, n, a, C);
    }
    if (st + 1 < nstages) train_residual_kernel<<<grid, kTrainThreads, 0, s>>>(R, n, C, a);
  }
  return check_launch();
}

}  // namespace

extern "C" {

vq3r_status vq3r_encode(const void* W, vq3r_dtype w_dtype, int64_t rows, int64_t cols, const float* codebooks,
                        uint8_t* idx, uint16_t* scales, vq3r_stream stream) {
  return encode_entry<FMT_VQ3R>(W, w_dtype, rows, cols, codebooks, idx, scales, stream);
}

vq3r_status vq3r_decode(const uint8_t* idx, const uint16_t* scales, const float* codebooks, int64_t rows,
                        int64_t cols, void* out, vq3r_dtype out_dtype, vq3r_stream stream) {
  return decode_entry<FMT_VQ3R>(idx, scales, codebooks, rows, cols, out, out_dtype, stream);
}

size_t vq3r_gemv_workspace_size(const vq3r_gemv_desc* mats, int n_mats, int B) {
  if (!mats || n_mats < 1 || n_mats > VQ3R_GEMV_MAX_MATS || B < 1 || B > VQ3R_GEMV_MAX_B) return 0;
  GemvPlan plan;
  if (plan_gemv(mats, n_mats, B, 1, nullptr, &plan) != VQ3R_OK) return 0;  // the table-token count changes no size
  return plan.ws_bytes;
}

vq3r_status vq3r_gemv(const vq3r_gemv_desc* mats, int n_mats, int B, vq3r_dtype x_dtype, void* workspace,
                      size_t ws_bytes, vq3r_stream stream) {
  if (!mats) return VQ3R_ERR_NULL;
  if (n_mats < 1 || n_mats > VQ3R_GEMV_MAX_MATS || B < 1 || B > VQ3R_GEMV_MAX_B) return VQ3R_ERR_BATCH;
  if (!valid_dtype(x_dtype)) return VQ3R_ERR_DTYPE;
  GemvPlan plan;
  // The tiled lookup-table kernel takes 2 or more tokens as pairs (both of a
  // pair's tables resident, the index stream read once per pair); bf16 x
  // with more tokens goes to the tensor cores instead.
  const bool tiles_tables = mats[0].layout == VQ3R_LAYOUT_TILES && (x_dtype != VQ3R_BF16 || B < kMmaMinB);
  const int tokm = tiles_tables && B >= 2 ? 2 : 1;
  vq3r_status st = plan_gemv(mats, n_mats, B, tokm, static_cast<char*>(workspace), &plan);
  if (st != VQ3R_OK) return st;
  if (plan.P.total_units == 0) return VQ3R_OK;
  if (!workspace || ws_bytes < plan.ws_bytes) return VQ3R_ERR_WORKSPACE;
  if (!aligned16(workspace)) return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const GvParams& P = plan.P;
  // Kernels are launched with programmatic stream serialization: their CTAs
  // may be scheduled while the preceding kernel drains and wait
  // (griddepcontrol.wait) before reading any input.  The tiled kernel reduces
  // its own partial sums; the planes kernel is followed by the reduction
  // kernel, whose CTAs wait the same way for the partial sums.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  bool one_codebook = true;
  for (int g = 1; g < P.n_groups; g++) one_codebook = one_codebook && P.g[g].codebooks == P.g[0].codebooks;
  if (P.layout == VQ3R_LAYOUT_TILES && x_dtype == VQ3R_BF16 && B >= kTgMinB && one_codebook) {
    // Several tokens: rebuild the weights into tensor memory and contract on
    // the tcgen05 tensor cores.  The work is the sequence of K-steps (128-row
    // tile, 16 columns) of all matrices, split evenly over four warp-groups
    // per SM; like the lookup-table kernel it zeroes y behind a grid barrier,
    // so one CTA must fit per SM.
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (!g_dev_tc_fit[dev]) return cuda_fail(cudaErrorCooperativeLaunchTooLarge);
    int64_t ksteps = 0;
    for (int i = 0; i < P.n_mats; i++)
      ksteps += (P.m[i].rows + kTgRows - 1) / kTgRows * ((P.g[P.m[i].group].cols / kDim + 1) / 2);
    plan.P.total_units = ksteps;
    cfg.gridDim = dim3((unsigned)sms);
    cfg.blockDim = dim3(kTgThreads);
    cfg.dynamicSmemBytes = kTgSmemBytes;
    e = B <= 16 ? cudaLaunchKernelEx(&cfg, gemv_tc_kernel<1>, plan.P) : cudaLaunchKernelEx(&cfg, gemv_tc_kernel<2>, plan.P);
    if (e != cudaSuccess) return cuda_fail(e);
    return check_launch();
  }
  if (P.layout == VQ3R_LAYOUT_TILES && x_dtype == VQ3R_BF16 && B >= kMmaMinB) {
    // 11..16 tokens (or matrices with different codebooks): rebuild the weights
    // in registers and contract with mma.sync; each CTA owns 256 rows of one
    // matrix and loads its codebooks.  Measured on the 8-expert decode step:
    // 231 us at B = 12 (two-token tables: 250 us), 213 us at B = 8 (tables:
    // 171 us, so B <= 10 stays on the tables); the tensor-memory kernel wins
    // from 17 tokens (237 against 279 us at B = 32).
    // One CTA per 128 rows of a matrix; blk_begin numbers those blocks.
    int64_t blocks = 0;
    for (int i = 0; i < P.n_mats; i++) {
      plan.P.m[i].blk_begin = (int32_t)blocks;
      blocks += (P.m[i].rows + kMmaRows - 1) / kMmaRows;
    }
    if (blocks >= ((int64_t)1 << 31)) return VQ3R_ERR_SHAPE;
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kMmaThreads);
    cfg.dynamicSmemBytes = kMmaSmemBytes;
    switch ((B + 7) / 8) {
      case 1: e = cudaLaunchKernelEx(&cfg, gemv_mma_kernel<1>, P); break;
      case 2: e = cudaLaunchKernelEx(&cfg, gemv_mma_kernel<2>, P); break;
      case 3: e = cudaLaunchKernelEx(&cfg, gemv_mma_kernel<3>, P); break;
      default: e = cudaLaunchKernelEx(&cfg, gemv_mma_kernel<4>, P); break;
    }
    if (e != cudaSuccess) return cuda_fail(e);
    return check_launch();
  }
  if (P.layout == VQ3R_LAYOUT_TILES) return launch_tiles<FMT_VQ3R, kTileSlots>(plan, x_dtype, sms, cfg);
  {  // two CTAs per SM
    const int grid = (int)(P.total_units < 2 * (int64_t)sms ? P.total_units : 2 * (int64_t)sms);
    switch (x_dtype) {
      case VQ3R_F32: gemv_lut_kernel<VQ3R_F32><<<grid, kGvThreads, kGvSmemBytes, s>>>(P); break;
      case VQ3R_BF16: gemv_lut_kernel<VQ3R_BF16><<<grid, kGvThreads, kGvSmemBytes, s>>>(P); break;
      default: gemv_lut_kernel<VQ3R_F16><<<grid, kGvThreads, kGvSmemBytes, s>>>(P); break;
    }
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  int64_t maxrows = 1;
  for (int i = 0; i < P.n_mats; i++) maxrows = P.m[i].rows > maxrows ? P.m[i].rows : maxrows;
  cfg.gridDim = dim3((unsigned)((maxrows + kPlanesRedRows - 1) / kPlanesRedRows), (unsigned)P.n_mats);
  cfg.blockDim = dim3(2 * kPlanesRedRows);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, gemv_reduce_kernel, P);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

vq3r_status vq4p_gemv(const vq3r_gemv_desc* mats, int n_mats, int B, vq3r_dtype x_dtype, void* workspace,
                      size_t ws_bytes, vq3r_stream stream) {
  if (!mats) return VQ3R_ERR_NULL;
  if (n_mats < 1 || n_mats > VQ3R_GEMV_MAX_MATS || B < 1 || B > VQ3R_GEMV_MAX_B) return VQ3R_ERR_BATCH;
  if (!valid_dtype(x_dtype)) return VQ3R_ERR_DTYPE;
  if (mats[0].layout != VQ3R_LAYOUT_TILES) return VQ3R_ERR_SHAPE;  // plan_gemv checks that all layouts agree
  GemvPlan plan;
  vq3r_status st = plan_gemv(mats, n_mats, B, B >= 2 ? 2 : 1, static_cast<char*>(workspace), &plan, 1);
  if (st != VQ3R_OK) return st;
  if (plan.P.total_units == 0) return VQ3R_OK;
  if (!workspace || ws_bytes < plan.ws_bytes) return VQ3R_ERR_WORKSPACE;
  if (!aligned16(workspace)) return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return launch_tiles<FMT_VQ4P, 1>(plan, x_dtype, sms, cfg);
}

vq3r_status vq3r_gemm(const vq3r_gemm_desc* mats, int n_mats, vq3r_dtype x_dtype, vq3r_stream stream) {
  if (!mats) return VQ3R_ERR_NULL;
  if (n_mats < 1 || n_mats > VQ3R_GEMV_MAX_MATS) return VQ3R_ERR_BATCH;
  if (x_dtype != VQ3R_BF16) return VQ3R_ERR_DTYPE;  // the tensor-core product takes bf16 x
  GemmParams P;
  memset(&P, 0, sizeof(P));
  int64_t ctas = 0;
  int nm = 0;
  for (int i = 0; i < n_mats; i++) {
    const vq3r_gemm_desc& d = mats[i];
    vq3r_status st = check_shape(d.rows, d.cols, 0);
    if (st != VQ3R_OK) return st;
    if (d.tokens < 0 || d.tokens >= ((int64_t)1 << 31) || d.rows >= ((int64_t)1 << 31) ||
        d.cols / kDim > (int64_t)kSlabV * (1 << 20) || d.reserved != 0)
      return VQ3R_ERR_SHAPE;
    const int64_t plane = (d.rows + kTileRows - 1) / kTileRows * kTileBytes;
    if (d.plane_stride != 0 && (d.plane_stride < plane || d.plane_stride % kTileBytes)) return VQ3R_ERR_SHAPE;
    if (d.rows == 0 || d.tokens == 0) continue;  // nothing to compute; pointers may be NULL
    if (!d.idx || !d.scales || !d.codebooks || !d.x || !d.y) return VQ3R_ERR_NULL;
    if (!aligned16(d.idx) || !aligned16(d.scales) || !aligned16(d.codebooks) || !aligned16(d.x) || !aligned16(d.y))
      return VQ3R_ERR_ALIGN;
    GmMat& M = P.m[nm++];
    M.idx = d.idx;
    M.scales = d.scales;
    M.codebooks = d.codebooks;
    M.x = static_cast<const uint16_t*>(d.x);
    M.y = d.y;
    M.rows = d.rows;
    M.cols = d.cols;
    M.tokens = d.tokens;
    M.plane_stride = d.plane_stride ? d.plane_stride : plane;
    M.n_slabs = (int32_t)((d.cols / kDim + kSlabV - 1) / kSlabV);
    M.tok_tiles = (int32_t)((d.tokens + kTcTokens - 1) / kTcTokens);
    M.cta_begin = ctas;
    ctas += (d.rows + kTcRows - 1) / kTcRows * M.tok_tiles;
  }
  if (nm == 0) return VQ3R_OK;
  if (ctas >= ((int64_t)1 << 31)) return VQ3R_ERR_SHAPE;
  P.n_mats = nm;
  P.total_ctas = ctas;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = kTcSmemBytes;
  e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel, P);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

size_t vq3r_train_workspace_size(int64_t n) {
  if (n < kCodewords || n > ((int64_t)1 << 40)) return 0;
  return train_ws_bytes(n);
}

size_t vq4p_train_workspace_size(int64_t n) {
  if (n < 64 || n > ((int64_t)1 << 40)) return 0;
  return train_ws_bytes(n);
}

vq3r_status vq3r_train(const float* vecs, int64_t n, int iters, int nstages, float* codebooks, double* trace,
                       void* workspace, size_t ws_bytes, vq3r_stream stream) {
  return train_entry<kStages, kCodewords>(vecs, n, iters, nstages, codebooks, trace, workspace, ws_bytes, stream);
}

vq3r_status vq4p_train(const float* vecs, int64_t n, int iters, int nstages, float* codebooks, double* trace,
                       void* workspace, size_t ws_bytes, vq3r_stream stream) {
  return train_entry<4, 64>(vecs, n, iters, nstages, codebooks, trace, workspace, ws_bytes, stream);
}

size_t vq3r_tiles_size(int64_t rows, int64_t cols) {
  if (check_shape(rows, cols, 0) != VQ3R_OK) return 0;
  const int64_t n_slabs = (cols / kDim + kSlabV - 1) / kSlabV;
  const int64_t n_tiles = (rows + kTileRows - 1) / kTileRows;
  return (size_t)kStages * n_slabs * n_tiles * kTileBytes;
}

vq3r_status vq3r_pack_tiles(const uint8_t* idx, int64_t rows, int64_t cols, int64_t plane_stride, uint8_t* packed,
                            vq3r_stream stream) {
  vq3r_status st = check_shape(rows, cols, 0);
  if (st != VQ3R_OK) return st;
  if (cols / kDim > (int64_t)kSlabV * (1 << 20)) return VQ3R_ERR_SHAPE;
  const int64_t plane = rows * (cols / kDim);
  if (plane_stride != 0 && plane_stride < plane) return VQ3R_ERR_SHAPE;
  if (rows == 0) return VQ3R_OK;
  if (!idx || !packed) return VQ3R_ERR_NULL;
  if (!aligned16(packed)) return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  const int32_t n_slabs = (int32_t)((cols / kDim + kSlabV - 1) / kSlabV);
  const int64_t n_tiles = (rows + kTileRows - 1) / kTileRows;
  if ((int64_t)kStages * n_slabs * n_tiles >= ((int64_t)1 << 32)) return VQ3R_ERR_SHAPE;  // block numbers are 32-bit
  const int64_t chunks = (int64_t)kStages * n_slabs * n_tiles * (kTileBytes / 16);
  int64_t blocks = (chunks + 255) / 256;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  pack_tiles_kernel<<<(int)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      idx, rows, cols / kDim, plane_stride ? plane_stride : plane, n_slabs, n_tiles, packed);
  return check_launch();
}

size_t vq3r_rel_frobenius_workspace_size(int64_t rows, int64_t cols) {
  (void)rows;
  (void)cols;
  return (size_t)kErrMaxBlocks * 2 * sizeof(double);
}

vq3r_status vq3r_rel_frobenius_error(const void* W, vq3r_dtype w_dtype, const uint8_t* idx, const uint16_t* scales,
                                     const float* codebooks, int64_t rows, int64_t cols, double* err_out,
                                     void* workspace, size_t ws_bytes, vq3r_stream stream) {
  return relfro_entry<FMT_VQ3R>(W, w_dtype, idx, scales, codebooks, rows, cols, err_out, workspace, ws_bytes, stream);
}

vq3r_status vq4p_encode(const void* W, vq3r_dtype w_dtype, int64_t rows, int64_t cols, const float* codebooks,
                        uint8_t* planes, uint16_t* scales, vq3r_stream stream) {
  return encode_entry<FMT_VQ4P>(W, w_dtype, rows, cols, codebooks, planes, scales, stream);
}

vq3r_status vq4p_decode(const uint8_t* planes, const uint16_t* scales, const float* codebooks, int64_t rows,
                        int64_t cols, void* out, vq3r_dtype out_dtype, vq3r_stream stream) {
  return decode_entry<FMT_VQ4P>(planes, scales, codebooks, rows, cols, out, out_dtype, stream);
}

vq3r_status vq4p_rel_frobenius_error(const void* W, vq3r_dtype w_dtype, const uint8_t* planes, const uint16_t* scales,
                                     const float* codebooks, int64_t rows, int64_t cols, double* err_out,
                                     void* workspace, size_t ws_bytes, vq3r_stream stream) {
  return relfro_entry<FMT_VQ4P>(W, w_dtype, planes, scales, codebooks, rows, cols, err_out, workspace, ws_bytes,
                                stream);
}

// ---- outlier-aware variant ----

static vq3r_status check_outliers(int64_t rows, int64_t cols, int64_t k) {
  vq3r_status st = check_shape(rows, cols, 0);
  if (st != VQ3R_OK) return st;
  if (cols > kOutMaxCols || k < 0 || k > cols) return VQ3R_ERR_SHAPE;
  return VQ3R_OK;
}

vq3r_status vq3r_outliers(const void* W, vq3r_dtype w_dtype, const uint8_t* idx, const uint16_t* scales,
                          const float* codebooks, int64_t rows, int64_t cols, int64_t k, uint16_t* ocols,
                          uint16_t* ovals, vq3r_stream stream) {
  vq3r_status st = check_outliers(rows, cols, k);
  if (st != VQ3R_OK) return st;
  if (!valid_dtype(w_dtype)) return VQ3R_ERR_DTYPE;
  if (rows == 0 || k == 0) return VQ3R_OK;
  if (!W || !idx || !scales || !codebooks || !ocols || !ovals) return VQ3R_ERR_NULL;
  if (!aligned16(W) || !aligned16(idx) || !aligned16(scales) || !aligned16(codebooks) || !aligned16(ocols) ||
      !aligned16(ovals))
    return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t smem = outlier_select_smem(cols);
  const int per_sm = smem <= 100 * 1024 ? 2 : 1;
  const int grid = (int)(rows < (int64_t)sms * per_sm ? rows : (int64_t)sms * per_sm);
  switch (w_dtype) {
    case VQ3R_F32:
      outlier_select_kernel<VQ3R_F32><<<grid, kOutThreads, smem, s>>>(W, idx, scales, codebooks, rows, cols, (int)k, ocols, ovals);
      break;
    case VQ3R_BF16:
      outlier_select_kernel<VQ3R_BF16><<<grid, kOutThreads, smem, s>>>(W, idx, scales, codebooks, rows, cols, (int)k, ocols, ovals);
      break;
    default:
      outlier_select_kernel<VQ3R_F16><<<grid, kOutThreads, smem, s>>>(W, idx, scales, codebooks, rows, cols, (int)k, ocols, ovals);
  }
  return check_launch();
}

vq3r_status vq3r_decode_outliers(const uint8_t* idx, const uint16_t* scales, const float* codebooks,
                                 const uint16_t* ocols, const uint16_t* ovals, int64_t rows, int64_t cols, int64_t k,
                                 float* out, vq3r_stream stream) {
  vq3r_status st = check_outliers(rows, cols, k);
  if (st != VQ3R_OK) return st;
  if (rows > 0 && k > 0 && (!ocols || !ovals)) return VQ3R_ERR_NULL;
  st = decode_entry<FMT_VQ3R>(idx, scales, codebooks, rows, cols, out, VQ3R_F32, stream);
  if (st != VQ3R_OK || rows == 0 || k == 0) return st;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  const int64_t n = rows * k, need = (n + 255) / 256;
  const int grid = (int)(need < ((int64_t)1 << 30) ? need : ((int64_t)1 << 30));
  outlier_apply_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(out, rows, cols, k, ocols, ovals);
  return check_launch();
}

size_t vq3r_rel_frobenius_outliers_workspace_size(int64_t rows, int64_t cols, int64_t k) {
  (void)k;
  return vq3r_rel_frobenius_workspace_size(rows, cols);
}

vq3r_status vq3r_rel_frobenius_error_outliers(const void* W, vq3r_dtype w_dtype, const uint8_t* idx,
                                              const uint16_t* scales, const float* codebooks, const uint16_t* ocols,
                                              const uint16_t* ovals, int64_t rows, int64_t cols, int64_t k,
                                              double* err_out, void* workspace, size_t ws_bytes,
                                              vq3r_stream stream) {
  if (!W || !idx || !scales || !codebooks || !err_out) return VQ3R_ERR_NULL;
  vq3r_status st = check_outliers(rows, cols, k);
  if (st != VQ3R_OK) return st;
  if (rows < 1) return VQ3R_ERR_SHAPE;
  if (k > 0 && (!ocols || !ovals)) return VQ3R_ERR_NULL;
  if (!valid_dtype(w_dtype)) return VQ3R_ERR_DTYPE;
  if (!workspace || ws_bytes < vq3r_rel_frobenius_outliers_workspace_size(rows, cols, k)) return VQ3R_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(idx) || !aligned16(scales) || !aligned16(codebooks) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(err_out) & 7u) || (k > 0 && (!aligned16(ocols) || !aligned16(ovals))))
    return VQ3R_ERR_ALIGN;
  if (k == 0) return relfro_entry<FMT_VQ3R>(W, w_dtype, idx, scales, codebooks, rows, cols, err_out, workspace,
                                            ws_bytes, stream);
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* partial = static_cast<double*>(workspace);
  const int64_t blocks = rowsplit_blocks(rows, cols, sms, kErrMaxBlocks);
  const size_t smem = kCbrFloats * sizeof(float);
  const int kk = (int)k;
  switch (w_dtype) {
    case VQ3R_F32:
      relfro_partial_kernel<VQ3R_F32, FMT_VQ3R, true><<<(int)blocks, kErrThreads, smem, s>>>(W, idx, scales, codebooks, rows, cols, partial, ocols, ovals, kk);
      break;
    case VQ3R_BF16:
      relfro_partial_kernel<VQ3R_BF16, FMT_VQ3R, true><<<(int)blocks, kErrThreads, smem, s>>>(W, idx, scales, codebooks, rows, cols, partial, ocols, ovals, kk);
      break;
    default:
      relfro_partial_kernel<VQ3R_F16, FMT_VQ3R, true><<<(int)blocks, kErrThreads, smem, s>>>(W, idx, scales, codebooks, rows, cols, partial, ocols, ovals, kk);
  }
  relfro_final_kernel<<<1, 256, 0, s>>>(partial, (int)blocks, err_out);
  return check_launch();
}

vq3r_status vq3r_gemv_outliers(const vq3r_outlier_desc* mats, int n_mats, int B, vq3r_dtype x_dtype,
                               vq3r_stream stream) {
  if (!mats) return VQ3R_ERR_NULL;
  if (n_mats < 1 || n_mats > kOutGemvMaxMats || B < 1 || B > VQ3R_GEMV_MAX_B) return VQ3R_ERR_BATCH;
  if (!valid_dtype(x_dtype)) return VQ3R_ERR_DTYPE;
  OutGemvParams P;
  memset(&P, 0, sizeof(P));
  int m = 0;
  int64_t total = 0;
  for (int i = 0; i < n_mats; i++) {
    const vq3r_outlier_desc& d = mats[i];
    vq3r_status st = check_outliers(d.rows, d.cols, d.k);
    if (st != VQ3R_OK) return st;
    if (d.reserved != 0) return VQ3R_ERR_SHAPE;
    if (d.rows == 0 || d.k == 0) continue;
    if (!d.ocols || !d.ovals || !d.x || !d.y) return VQ3R_ERR_NULL;
    if (!aligned16(d.ocols) || !aligned16(d.ovals) || !aligned16(d.x) || !aligned16(d.y)) return VQ3R_ERR_ALIGN;
    P.ocols[m] = d.ocols;
    P.ovals[m] = d.ovals;
    P.x[m] = d.x;
    P.y[m] = d.y;
    P.rows[m] = d.rows;
    P.k[m] = d.k;
    P.cols[m] = d.cols;
    P.row_begin[m] = total;
    total += d.rows;
    m++;
  }
  if (m == 0) return VQ3R_OK;
  P.row_begin[m] = total;
  P.n_mats = m;
  P.B = B;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  const int64_t grid = (total + 255) / 256;
  if (grid > INT32_MAX) return VQ3R_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (x_dtype) {
    case VQ3R_F32: outlier_gemv_kernel<VQ3R_F32><<<(int)grid, 256, 0, s>>>(P); break;
    case VQ3R_BF16: outlier_gemv_kernel<VQ3R_BF16><<<(int)grid, 256, 0, s>>>(P); break;
    default: outlier_gemv_kernel<VQ3R_F16><<<(int)grid, 256, 0, s>>>(P);
  }
  return check_launch();
}

size_t vq3r_outliers_tiles_size(int64_t rows, int64_t k) {
  if (rows < 0 || k < 0 || k > kOutMaxCols) return 0;
  return (size_t)((rows + kOutTileRows - 1) / kOutTileRows) * (size_t)k * kOutTileRows * 4;
}

vq3r_status vq3r_pack_outliers(const uint16_t* ocols, const uint16_t* ovals, int64_t rows, int64_t k, uint32_t* otiles,
                               vq3r_stream stream) {
  if (rows < 0 || k < 0 || k > kOutMaxCols) return VQ3R_ERR_SHAPE;
  if (rows == 0 || k == 0) return VQ3R_OK;
  if (!ocols || !ovals || !otiles) return VQ3R_ERR_NULL;
  if (!aligned16(otiles)) return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  const int64_t n_tiles = (rows + kOutTileRows - 1) / kOutTileRows;
  const int64_t n = n_tiles * k * kOutTileRows;
  int64_t blocks = (n + 255) / 256;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  pack_outliers_kernel<<<(int)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(ocols, ovals, rows, k, n_tiles,
                                                                                     otiles);
  return check_launch();
}

vq3r_status vq3r_gemv_with_outliers(const vq3r_gemv_desc* mats, const vq3r_outlier_tiles* outl, int n_mats, int B,
                                    vq3r_dtype x_dtype, void* workspace, size_t ws_bytes, vq3r_stream stream) {
  if (!mats || !outl) return VQ3R_ERR_NULL;
  if (n_mats < 1 || n_mats > VQ3R_GEMV_MAX_MATS || B < 1 || B > VQ3R_GEMV_MAX_B) return VQ3R_ERR_BATCH;
  if (!valid_dtype(x_dtype)) return VQ3R_ERR_DTYPE;
  bool any = false;
  for (int i = 0; i < n_mats; i++) {
    const vq3r_outlier_tiles& o = outl[i];
    const vq3r_gemv_desc& d = mats[i];
    if (o.k < 0 || o.k > d.cols || (o.k > 0 && d.cols > kOutMaxCols)) return VQ3R_ERR_SHAPE;
    if (d.rows <= 0 || o.k == 0) continue;
    if (!o.otiles) return VQ3R_ERR_NULL;
    if (!aligned16(o.otiles)) return VQ3R_ERR_ALIGN;
    any = true;
  }
  // The lookup-table kernel starts y at the outliers' sums instead of zero
  // (before its grid barrier); the other kernels are followed by a separate
  // sparse add over the outlier tiles.
  const bool fused = mats[0].layout == VQ3R_LAYOUT_TILES && (x_dtype != VQ3R_BF16 || B < kMmaMinB);
  if (!fused || !any) {
    vq3r_status st = vq3r_gemv(mats, n_mats, B, x_dtype, workspace, ws_bytes, stream);
    if (st != VQ3R_OK || !any) return st;
    OutTilesParams Q;
    memset(&Q, 0, sizeof(Q));
    int m = 0;
    int64_t total = 0;
    for (int i = 0; i < n_mats; i++) {
      if (mats[i].rows <= 0 || outl[i].k == 0) continue;
      Q.ot[m] = outl[i].otiles;
      Q.x[m] = mats[i].x;
      Q.y[m] = mats[i].y;
      Q.rows[m] = mats[i].rows;
      Q.k[m] = outl[i].k;
      Q.cols[m] = mats[i].cols;
      Q.row_begin[m] = total;
      total += mats[i].rows;
      m++;
    }
    Q.row_begin[m] = total;
    Q.n_mats = m;
    Q.B = B;
    const int64_t grid = (total + 255) / 256;
    if (grid > INT32_MAX) return VQ3R_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (x_dtype) {
      case VQ3R_F32: outlier_tiles_add_kernel<VQ3R_F32><<<(int)grid, 256, 0, s>>>(Q); break;
      case VQ3R_BF16: outlier_tiles_add_kernel<VQ3R_BF16><<<(int)grid, 256, 0, s>>>(Q); break;
      default: outlier_tiles_add_kernel<VQ3R_F16><<<(int)grid, 256, 0, s>>>(Q);
    }
    return check_launch();
  }
  GemvPlan plan;
  vq3r_status st = plan_gemv(mats, n_mats, B, B >= 2 ? 2 : 1, static_cast<char*>(workspace), &plan, kStages, outl);
  if (st != VQ3R_OK) return st;
  if (plan.P.total_units == 0) return VQ3R_OK;
  if (!workspace || ws_bytes < plan.ws_bytes) return VQ3R_ERR_WORKSPACE;
  if (!aligned16(workspace)) return VQ3R_ERR_ALIGN;
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return launch_tiles<FMT_VQ3R, kTileSlots, true>(plan, x_dtype, sms, cfg);
}

}  // extern "C"

namespace {

// Scratch of vq3r_gemv_noalloc: file-scope device array, one per GPU that
// loads the library.  Host code must not pass the symbol itself to a kernel
// (in host code it names a host-side stand-in); the device address comes
// from cudaGetSymbolAddress, looked up once per device with that device
// current.
static __device__ __align__(256) unsigned char g_gemv_noalloc_scratch[VQ3R_GEMV_NOALLOC_BYTES];

// Looked-up addresses, per device; null until a lookup has succeeded.  A
// failed lookup is not remembered, so the next call tries again.
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];

cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gemv_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

vq3r_status vq3r_gemv_noalloc(const vq3r_gemv_desc* mats, int n_mats, int B, vq3r_dtype x_dtype,
                              vq3r_stream stream) {
  if (!mats) return VQ3R_ERR_NULL;
  if (n_mats < 1 || n_mats > VQ3R_GEMV_MAX_MATS || B < 1 || B > VQ3R_GEMV_MAX_B) return VQ3R_ERR_BATCH;
  const size_t need = vq3r_gemv_workspace_size(mats, n_mats, B);
  if (need > (size_t)VQ3R_GEMV_NOALLOC_BYTES) return VQ3R_ERR_WORKSPACE;
  void* scratch = nullptr;
  const cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  return vq3r_gemv(mats, n_mats, B, x_dtype, scratch, VQ3R_GEMV_NOALLOC_BYTES, stream);
}

const char* vq3r_status_string(vq3r_status s) {
  switch (s) {
    case VQ3R_OK: return "VQ3R_OK";
    case VQ3R_ERR_NULL: return "VQ3R_ERR_NULL: a required pointer is NULL";
    case VQ3R_ERR_SHAPE: return "VQ3R_ERR_SHAPE: rows/cols invalid (cols must be a positive multiple of 8)";
    case VQ3R_ERR_ALIGN: return "VQ3R_ERR_ALIGN: device pointers must be 16-byte aligned";
    case VQ3R_ERR_DTYPE: return "VQ3R_ERR_DTYPE: unsupported dtype";
    case VQ3R_ERR_BATCH: return "VQ3R_ERR_BATCH: B must be in [1, 32] and n_mats in [1, 32]";
    case VQ3R_ERR_CUDA: return "VQ3R_ERR_CUDA: CUDA launch or call failed";
    case VQ3R_ERR_WORKSPACE: return "VQ3R_ERR_WORKSPACE: workspace missing or too small";
    default: return "VQ3R: unknown status";
  }
}

int vq3r_last_cuda_error(void) { return t_last_cuda_error; }

vq3r_status vq3r_selftest_wait_timeout(vq3r_stream stream) {
  int sms = 0;
  cudaError_t e = device_setup(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return check_launch();
}

vq3r_status vq3r_device_error(int* code) {
  if (!code) return VQ3R_ERR_NULL;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(code, g_device_error, sizeof(int));
  const int zero = 0;
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  return e == cudaSuccess ? VQ3R_OK : cuda_fail(e);
}

}  // extern "C"
