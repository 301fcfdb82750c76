/*
 * vq3r.h -- C ABI of the VQ3R codec library for NVIDIA B200 (sm_100a).
 *
 * VQ3R (page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验",
 * xdnf.cn/news/289497, §2) stores a weight matrix W (rows x cols, a row being
 * one output channel) as
 *   - one FP16 scale per row, and
 *   - for each 8-wide vector W[i, 8v : 8v+8], three uint8 indices i1, i2, i3
 *     into three 256-entry codebooks C1, C2, C3 of 8-dim fp32 vectors,
 * so that W[i, 8v+k] ~ scale_i * (C1[i1][k] + C2[i2][k] + C3[i3][k]):
 * 3 index bytes per 8 weights = exactly 3.00 bits/weight.
 *
 * Layouts (all row-major, no padding):
 *   W          [rows][cols]             f32, bf16 or f16
 *   codebooks  [3][256][8] float        stage-major (C1, then C2, then C3), 24 KiB
 *   idx        [3][rows][cols/8] uint8  three index planes, plane s = stage s+1
 *   scales     [rows] uint16            IEEE binary16 bit patterns
 *   x          [B][cols]                activations, f32, bf16 or f16
 *   y          [B][rows] float
 *
 * Conventions shared by every call:
 *   - Every data pointer is DEVICE memory owned by the caller, 16-byte
 *     aligned (VQ3R_ERR_ALIGN otherwise).  The library never allocates or
 *     frees device memory; temporary storage is the caller's `workspace`.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and return after enqueuing the work.
 *   - Argument errors are detected before anything is launched and nothing
 *     is written.  A failed launch returns VQ3R_ERR_CUDA.
 *   - cols must be a positive multiple of 8 (VQ3R_ERR_SHAPE).
 *   - Calls that overlap on the GPU must not share output or workspace
 *     buffers.
 */
#ifndef VQ3R_H
#define VQ3R_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VQ3R_OK = 0,
  VQ3R_ERR_NULL = 1,      /* a required pointer is NULL */
  VQ3R_ERR_SHAPE = 2,     /* rows < 0 (or < 1 where stated), cols < 8, cols % 8 != 0, size overflow */
  VQ3R_ERR_ALIGN = 3,     /* a device pointer is not 16-byte aligned */
  VQ3R_ERR_DTYPE = 4,     /* unsupported dtype for this argument */
  VQ3R_ERR_BATCH = 5,     /* B outside [1, 32], or n_mats outside [1, VQ3R_GEMV_MAX_MATS] */
  VQ3R_ERR_CUDA = 6,      /* a CUDA call or kernel launch failed (see vq3r_last_cuda_error) */
  VQ3R_ERR_WORKSPACE = 7  /* workspace NULL or smaller than the *_workspace_size result */
} vq3r_status;

typedef enum { VQ3R_F32 = 0, VQ3R_BF16 = 1, VQ3R_F16 = 2 } vq3r_dtype;

typedef void* vq3r_stream; /* cudaStream_t */

#define VQ3R_STAGES 3
#define VQ3R_CODEWORDS 256
#define VQ3R_DIM 8
#define VQ3R_GEMV_MAX_B 32
#define VQ3R_GEMV_MAX_MATS 32

/*
 * vq3r_encode -- per-row FP16 scale and greedy 3-stage residual assignment.
 *
 * Page §2 (per-row FP16 scale, 3 stages of 256 x 8-dim codebooks, stage s
 * quantises the residual left by stage s-1) and §4 (one pass over the three
 * stages writing only the winning indices).  For row i:
 *   scale_i = binary16(sqrt(ss_i / cols)), RNE, saturating at 65504, where
 *     ss_i is the binary64 sum of w^2 taken in a fixed order: per 8-vector
 *     q_v = ((w0^2 + w1^2) + ...) + w7^2, partials t_p = sum over v = p mod 128
 *     (v ascending), then t_p += t_{p+h} for h = 64, 32, ..., 1.
 *   r = (float)w / (float)scale_i (IEEE division; r = 0 if scale_i = 0).
 * For each stage s = 1..3: d_j = sum_{k=0..7} (r_k - C_s[j][k])^2 in binary32,
 * k ascending, every operation rounded (no fused multiply-add); i_s = the
 * j with the smallest d_j, the lowest j on ties; r -= C_s[i_s].
 * Results are bit-identical to that definition.
 *
 *   W         [rows][cols], w_dtype in {F32, BF16, F16}
 *   codebooks [3][256][8] float
 *   idx       out, [3][rows][cols/8] uint8
 *   scales    out, [rows] binary16 bits
 * rows == 0 is a no-op (pointers may then be NULL).  Non-finite weights give
 * unspecified (but in-bounds) indices.
 */
vq3r_status vq3r_encode(const void* W, vq3r_dtype w_dtype, int64_t rows, int64_t cols, const float* codebooks,
                        uint8_t* idx, uint16_t* scales, vq3r_stream stream);

/*
 * vq3r_decode -- reconstruct the weights (page §2 reconstruction rule).
 *   w_hat[i][8v+k] = (float)scale_i * ((C1[i1][k] + C2[i2][k]) + C3[i3][k])
 * in binary32, every operation rounded; an F16 output is the RNE conversion
 * of that binary32 value (overflow to +-inf).
 *
 *   idx, scales, codebooks as written by vq3r_encode
 *   out       [rows][cols], out_dtype in {F32, F16}
 * rows == 0 is a no-op (pointers may then be NULL).
 */
vq3r_status vq3r_decode(const uint8_t* idx, const uint16_t* scales, const float* codebooks, int64_t rows,
                        int64_t cols, void* out, vq3r_dtype out_dtype, vq3r_stream stream);

/*
 * vq3r_gemv -- y = W_hat . x for a group of VQ3R matrices, B = 1..32 tokens
 * (the MoE decode step, page §1: a few experts' matrices per token).
 *   y[b][i] = sum_c w_hat[i][c] * x[b][c], fp32 accumulation, w_hat as in
 *   vq3r_decode.  Summation order is the library's own: results agree with
 *   an exact (binary64) product to about 1e-4 relative to rms(y), not bit
 *   for bit.  TILES calls below 11 tokens (and all TILES calls with F32 or
 *   F16 x), and TILES calls of 17 or more bf16 tokens whose matrices share
 *   one codebooks pointer (the tensor-memory kernel, which splits the
 *   columns of a row block between warp groups), add partial sums into y
 *   with atomic adds, in the order the GPU schedules them, so two identical
 *   calls may differ in the last bits of y; PLANES calls and the other TILES
 *   calls of 11 or more bf16 tokens give the same bits every time.
 *
 * One descriptor per matrix; matrices may differ in shape, codebooks and x.
 * Matrices that share (codebooks, x, cols) share the x-projected tables the
 * kernel builds in shared memory, so one call over the gate and up matrices
 * of all active experts builds each table once per SM that needs it.  y must
 * not overlap any input.
 *
 * Workspace: a 256-byte header, then, for PLANES, one float partial sum per
 * (token, stage, 64-column slab, row), added in a second kernel.  TILES
 * calls need the header only: the kernel zeroes y, and its CTAs meet on a
 * grid barrier kept in the header (arrival counts) before the first add.
 * Fill a workspace with zeros once before its first call (e.g.
 * cudaMemsetAsync after allocating it); nothing needs clearing between
 * calls, replays of a captured CUDA graph included.  The TILES kernel runs
 * one CTA per SM and needs all of them resident together.  The library
 * checks once per device that one CTA fits on an SM (else VQ3R_ERR_CUDA,
 * vq3r_last_cuda_error() = cudaErrorCooperativeLaunchTooLarge); it does not
 * launch cooperatively (that measured about 4 us slower per call), so if
 * another workload holds SMs for more than about a second, the call
 * finishes with vq3r_device_error() = 2 and y undefined.
 *   mats      HOST array of n_mats descriptors (copied before return)
 *   B         tokens, 1..32
 *   x_dtype   dtype of every x, {F32, BF16, F16}
 *   workspace device scratch of at least vq3r_gemv_workspace_size() bytes
 * A matrix with rows == 0 contributes nothing (its pointers may be NULL);
 * rows must be below 2^31 and cols / 8 at most 2^26 (VQ3R_ERR_SHAPE).
 * TILES descriptors need plane_stride a multiple of 32768 and at least
 * ceil(rows / 512) * 32768; mixing layouts in one call is VQ3R_ERR_SHAPE.
 */
/* Index layouts accepted by vq3r_gemv (the encoder writes VQ3R_LAYOUT_PLANES). */
typedef enum {
  VQ3R_LAYOUT_PLANES = 0, /* [3][rows][cols/8], as written by vq3r_encode */
  VQ3R_LAYOUT_TILES = 1   /* blocks of 512 rows x 64 columns, see vq3r_pack_tiles */
} vq3r_layout;

typedef struct {
  const uint8_t* idx;       /* PLANES: plane 0 of [3][rows][cols/8]; TILES: first block, see below */
  const uint16_t* scales;   /* [rows] binary16 */
  const float* codebooks;   /* [3][256][8] */
  int64_t rows, cols;
  const void* x;            /* [B][cols] */
  float* y;                 /* [B][rows] */
  int64_t plane_stride;     /* PLANES: bytes from one index plane to the next; 0 = rows * cols / 8.
                               A row range [r0, r0 + rows) of a larger encoded matrix
                               (e.g. one expert of a stacked layer) is described by
                               idx + r0 * cols / 8, scales + r0 and that matrix's
                               plane size (VQ3R_ERR_SHAPE if below rows * cols / 8).
                               TILES: bytes from one (stage, slab) column of blocks to
                               the next, i.e. n_tiles * 32768 of the packed matrix; 0 =
                               ceil(rows / 512) * 32768.  A row range starting at a
                               multiple of 512 is idx + (r0 / 512) * 32768, scales + r0. */
  int32_t layout;           /* vq3r_layout; all descriptors of one call use the same one */
  int32_t reserved;         /* must be 0 */
} vq3r_gemv_desc;

size_t vq3r_gemv_workspace_size(const vq3r_gemv_desc* mats, int n_mats, int B);

/*
 * vq3r_pack_tiles -- repack encoded index planes into the tiled layout that
 * lets vq3r_gemv stream each work unit as one contiguous block (a one-time
 * conversion of static weights; results of vq3r_gemv are the same for both
 * layouts).  Layout: for stage s (0..2), slab (64 index columns, n_slabs =
 * ceil(cols / 512)) and tile (512 rows, n_tiles = ceil(rows / 512)), a block
 * of 512 x 64 bytes at ((s * n_slabs + slab) * n_tiles + tile) * 32768; row r
 * of a block at r * 64, index column c at
 *   16 * (c >> 4) + 8 * (((c >> 3) & 1) ^ ((r >> 2) & 1)) + (c & 7).
 * Rows and columns past the matrix are zero.
 *   idx          [3][rows][cols/8] planes, plane_stride bytes apart (0 = rows * cols / 8)
 *   packed       out, vq3r_tiles_size(rows, cols) bytes, 16-byte aligned
 */
size_t vq3r_tiles_size(int64_t rows, int64_t cols);
vq3r_status vq3r_pack_tiles(const uint8_t* idx, int64_t rows, int64_t cols, int64_t plane_stride, uint8_t* packed,
                            vq3r_stream stream);
vq3r_status vq3r_gemv(const vq3r_gemv_desc* mats, int n_mats, int B, vq3r_dtype x_dtype, void* workspace,
                      size_t ws_bytes, vq3r_stream stream);

/*
 * vq3r_rel_frobenius_error -- the Gate 3 metric of page §3.1:
 *   err = sqrt( sum (w - w_hat)^2 / sum w^2 ),
 * w the original weight widened to binary64, w_hat the binary32 decode of
 * vq3r_decode, both sums accumulated in binary64 (library order; agrees with
 * a sequential binary64 sum to ~1e-12 relative).
 *
 *   W, w_dtype   original weights [rows][cols]
 *   err_out      DEVICE pointer to one double (written asynchronously)
 *   workspace    at least vq3r_rel_frobenius_workspace_size() bytes
 * rows must be >= 1.  An all-zero W gives NaN (0/0).
 */
size_t vq3r_rel_frobenius_workspace_size(int64_t rows, int64_t cols);
vq3r_status vq3r_rel_frobenius_error(const void* W, vq3r_dtype w_dtype, const uint8_t* idx, const uint16_t* scales,
                                     const float* codebooks, int64_t rows, int64_t cols, double* err_out,
                                     void* workspace, size_t ws_bytes, vq3r_stream stream);

/*
 * vq3r_gemv_noalloc -- vq3r_gemv for callers that cannot allocate device
 * memory: a decode loop running under a memory pool that forbids new
 * allocations after warm-up, code that must not trigger the implicit device
 * synchronisation of cudaMalloc/cudaFree, or a host that simply has no
 * allocator to offer.  The paper has no counterpart; this is a library
 * convenience.
 *
 * Same arguments and results as vq3r_gemv, minus the workspace: the scratch
 * is one array of VQ3R_GEMV_NOALLOC_BYTES (16 MiB) in the library's device
 * image, which every GPU that loads the library holds until the process
 * exits.  The call allocates nothing (no cudaMalloc, cudaFree or allocating
 * library routine).
 *   - A call whose vq3r_gemv_workspace_size() exceeds 16 MiB returns
 *     VQ3R_ERR_WORKSPACE before launching anything.  TILES calls need 256
 *     bytes whatever their size; in the PLANES layout the 8-expert MoE
 *     decode step of 2048 x 7168 / 7168 x 2048 matrices needs 7.9 MiB at
 *     B = 1 as one call.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before capturing a stream into a graph.  If that lookup fails the call
 *     returns VQ3R_ERR_CUDA and the next call looks it up again.
 *   - All calls share the one array: calls that overlap on the GPU (different
 *     streams, or different host threads on the same device) race and must be
 *     serialised by the caller.  The array is zeroed when the library is
 *     loaded, as vq3r_gemv requires of a new workspace.
 */
#define VQ3R_GEMV_NOALLOC_BYTES (16u << 20)
vq3r_status vq3r_gemv_noalloc(const vq3r_gemv_desc* mats, int n_mats, int B, vq3r_dtype x_dtype, vq3r_stream stream);

/*
 * vq3r_train -- fit the three codebooks (page §2: per-layer codebooks by
 * Lloyd k-means on sampled vectors; stage s is trained on the residuals left
 * by stage s - 1).  Readings where the page is silent: the initial
 * centroids are the first 256 training vectors (of the stage's residuals);
 * assignment uses vq3r_encode's distance and tie rule; a centroid is the
 * binary64 sum of its members' components in training order, divided by
 * their count and rounded to binary32; an empty cluster keeps its centroid;
 * `iters` updates, then a final assignment from which the residuals
 * r - C[a] (binary32) of the next stage are taken.  Results are bit-identical
 * to that definition.
 *   vecs       [n][8] float, DEVICE, the training vectors (already divided by
 *              their rows' scales), n >= 256 (VQ3R_ERR_SHAPE)
 *   iters      Lloyd updates per stage, >= 0
 *   nstages    1..3
 *   codebooks  out, [nstages][256][8] float, DEVICE
 *   trace      out, DEVICE or NULL: [nstages][iters + 1] binary64 total
 *              squared distance after each assignment (summed in the
 *              library's order: equal to the sequential sum to ~1e-12)
 *   workspace  at least vq3r_train_workspace_size(n) bytes, DEVICE
 * Launches about nstages * (2 * iters + 3) small kernels.
 */
size_t vq3r_train_workspace_size(int64_t n);
vq3r_status vq3r_train(const float* vecs, int64_t n, int iters, int nstages, float* codebooks, double* trace,
                       void* workspace, size_t ws_bytes, vq3r_stream stream);

/*
 * vq3r_gemm -- the many-token product for prompts (prefill), on the tensor
 * cores:  Y[t][i] = sum_c bf16(w_hat[i][c]) * x[t][c],  fp32 accumulation.
 * w_hat is the binary32 value vq3r_decode writes (page §2 reconstruction
 * rule); bf16() rounds it to nearest even, the operand type of the bf16
 * tensor-core product.  The pages define no batched product (their
 * measurements are per token, page §1); this call is the prefill counterpart
 * of vq3r_gemv and reuses its TILES layout.  Summation order is the
 * library's: results agree with a binary64 product of the same bf16 weights
 * to about 1e-5 relative to rms(Y), not bit for bit.  The bf16 rounding of
 * w_hat (relative error up to 2^-9 per weight) makes this product differ
 * from vq3r_gemv's for the same token by about 1e-3 relative to rms(Y):
 * vq3r_gemv carries each weight as a bf16 pair hi + lo (about 2^-17) on its
 * tensor-core paths and in binary32 on its lookup paths.  A caller that needs
 * the decode step's accuracy for a few prompt tokens can call vq3r_gemv with
 * up to 32 tokens.
 *
 * One descriptor per matrix (up to VQ3R_GEMV_MAX_MATS), each with its own
 * tokens, e.g. the experts of an MoE layer and the tokens routed to each.
 *   idx       first TILES block (see vq3r_pack_tiles); plane_stride as in
 *             vq3r_gemv_desc (0 = ceil(rows / 512) * 32768, else a multiple
 *             of 32768 and at least that)
 *   scales, codebooks as written by / given to vq3r_encode
 *   x         [tokens][cols] bf16, row-major, DEVICE
 *   y         [tokens][rows] fp32, row-major, DEVICE, written (not added to);
 *             must not overlap any input
 *   tokens    number of rows of x and y; 0 (or rows == 0) is a no-op for the
 *             matrix (its pointers may then be NULL)
 * x_dtype must be VQ3R_BF16 (VQ3R_ERR_DTYPE otherwise).  rows and tokens
 * below 2^31, cols a multiple of 8 and cols / 8 at most 2^26
 * (VQ3R_ERR_SHAPE); all pointers 16-byte aligned (VQ3R_ERR_ALIGN).  Needs no
 * workspace.  One CTA per 128 rows x 256 tokens of a matrix; each uses 256
 * columns of tensor memory and about 225 KiB of shared memory, so one runs
 * per SM.  A bounded wait that gives up (about one second) sets
 * vq3r_device_error() = 1 and leaves y undefined.
 */
typedef struct {
  const uint8_t* idx;
  const uint16_t* scales;
  const float* codebooks;
  int64_t rows, cols;
  const void* x;
  float* y;
  int64_t plane_stride;
  int64_t tokens;
  int64_t reserved;         /* must be 0 */
} vq3r_gemm_desc;

vq3r_status vq3r_gemm(const vq3r_gemm_desc* mats, int n_mats, vq3r_dtype x_dtype, vq3r_stream stream);

/*
 * VQ4P -- the sibling format of page §5 at the same 3.00 bits/weight: four
 * stages of 64-entry codebooks (6-bit indices) instead of three of 256.
 * Readings where the page names the format but gives no layout: the
 * encoder, scale, distance, tie rule and stage order are vq3r_encode's with
 * S = 4 stages and K = 64 codewords; the four indices of a vector form the
 * 24-bit word  w = i1 | i2 << 6 | i3 << 12 | i4 << 18  whose byte p (p = 0,
 * 1, 2) is stored in byte plane p, so the index storage is byte for byte
 * that of VQ3R.
 *   codebooks  [4][64][8] float, stage-major, 8 KiB
 *   planes     [3][rows][cols/8] uint8, plane p = byte p of w
 *   w_hat[i][8v+k] = (float)scale_i * (((C1[i1][k] + C2[i2][k]) + C3[i3][k]) + C4[i4][k])
 * in binary32, every operation rounded.  Arguments, conventions, errors and
 * bit-exactness are those of the VQ3R call of the same name.
 */
vq3r_status vq4p_encode(const void* W, vq3r_dtype w_dtype, int64_t rows, int64_t cols, const float* codebooks,
                        uint8_t* planes, uint16_t* scales, vq3r_stream stream);
vq3r_status vq4p_decode(const uint8_t* planes, const uint16_t* scales, const float* codebooks, int64_t rows,
                        int64_t cols, void* out, vq3r_dtype out_dtype, vq3r_stream stream);
/* workspace: at least vq3r_rel_frobenius_workspace_size(rows, cols) bytes */
vq3r_status vq4p_rel_frobenius_error(const void* W, vq3r_dtype w_dtype, const uint8_t* planes, const uint16_t* scales,
                                     const float* codebooks, int64_t rows, int64_t cols, double* err_out,
                                     void* workspace, size_t ws_bytes, vq3r_stream stream);
/*
 * vq4p_gemv -- vq3r_gemv for VQ4P weights: y[b][i] = sum_c w_hat[i][c] * x[b][c],
 * w_hat as vq4p_decode writes it, B = 1..32 tokens.  Descriptors, workspace,
 * errors and the grid-barrier conditions are those of vq3r_gemv with TILES
 * descriptors, except:
 *   - every descriptor must be VQ3R_LAYOUT_TILES (VQ3R_ERR_SHAPE otherwise):
 *     the three byte planes repacked by vq3r_pack_tiles, which moves bytes
 *     and so serves either format;
 *   - codebooks are [4][64][8] float;
 *   - every token count runs on the lookup-table kernel: one 256-row table per
 *     64-column slab holds the four stages' codewords, and from B = 2 two
 *     tokens share each pass over the indices.
 * Partial sums are added into y with atomic adds (last bits of y depend on
 * scheduling); results agree with a binary64 product of the decoded weights
 * to about 1e-4 relative to rms(y).
 *   workspace  at least vq3r_gemv_workspace_size() of the same descriptors
 *              (256 bytes), zero-filled before its first use
 */
vq3r_status vq4p_gemv(const vq3r_gemv_desc* mats, int n_mats, int B, vq3r_dtype x_dtype, void* workspace,
                      size_t ws_bytes, vq3r_stream stream);
/* vq3r_train's Lloyd reading with 64 centroids per stage (initial centroids:
 * the first 64 vectors); n >= 64, nstages 1..4, codebooks [nstages][64][8]. */
size_t vq4p_train_workspace_size(int64_t n);
vq3r_status vq4p_train(const float* vecs, int64_t n, int iters, int nstages, float* codebooks, double* trace,
                       void* workspace, size_t ws_bytes, vq3r_stream stream);

/*
 * Outlier-aware variant -- a sparse FP16 residual on top of the VQ3R
 * encoding (page "XFP：质量目标驱动的自适应码本量化",
 * zingnex.cn/forum/thread/xfp-llm, 技术实现 / 权重分解: a weight matrix is a
 * dense index tensor into learned codebooks plus a sparse FP16 outlier
 * residual kept at full precision, with an outlier budget).  The page gives
 * no selection rule or layout; readings:
 *   e = (double)w - (double)w_hat, w_hat the binary32 decode of vq3r_decode;
 *   per row, the k positions with the largest |e| (ordered by the binary64
 *   bit pattern of |e|; a NaN ranks first), ties to the lower column;
 *   each stores its column and o = fp16(e) (nearest even, saturating at
 *   +-65504); the decode adds (float)o to w_hat in binary32.
 * Layout: ocols [rows][k] uint16 (ascending within a row), ovals [rows][k]
 * uint16 binary16 bits: 4 bytes per outlier, 32 k / cols bits per weight.
 * cols <= 16384 (VQ3R_ERR_SHAPE otherwise), 0 <= k <= cols.
 *
 * vq3r_outliers: the outliers of W given its VQ3R encoding (idx, scales,
 *   codebooks as written by vq3r_encode).  Bit-identical to the reading.
 *   k == 0 or rows == 0 is a no-op.
 * vq3r_decode_outliers: vq3r_decode to binary32 followed by the outlier
 *   additions (out [rows][cols] float).  A row's columns must be distinct
 *   (as vq3r_outliers writes them); a repeated column is a data race.
 * vq3r_rel_frobenius_error_outliers: vq3r_rel_frobenius_error of the decode
 *   with outliers; workspace of vq3r_rel_frobenius_outliers_workspace_size.
 * vq3r_gemv_outliers: y[b][i] += sum_q (float)o_iq * x[b][c_iq] (binary32,
 *   q ascending) for each descriptor, in one launch: enqueue it after the
 *   vq3r_gemv call that wrote y to get the product with the outliers.
 *   1 <= n_mats <= 32, 1 <= B <= 32.  No two descriptors may write the same
 *   elements of y (each y element is updated by one thread, without atomics).
 * The error call and the sparse add read a row's columns as sorted
 * ascending, as vq3r_outliers writes them.
 */
typedef struct {
  const uint16_t* ocols;
  const uint16_t* ovals;
  int64_t rows, cols, k;
  const void* x;            /* [B][cols], x_dtype */
  float* y;                 /* [B][rows] */
  int64_t reserved;         /* must be 0 */
} vq3r_outlier_desc;

vq3r_status vq3r_outliers(const void* W, vq3r_dtype w_dtype, const uint8_t* idx, const uint16_t* scales,
                          const float* codebooks, int64_t rows, int64_t cols, int64_t k, uint16_t* ocols,
                          uint16_t* ovals, vq3r_stream stream);
vq3r_status vq3r_decode_outliers(const uint8_t* idx, const uint16_t* scales, const float* codebooks,
                                 const uint16_t* ocols, const uint16_t* ovals, int64_t rows, int64_t cols, int64_t k,
                                 float* out, vq3r_stream stream);
size_t vq3r_rel_frobenius_outliers_workspace_size(int64_t rows, int64_t cols, int64_t k);
vq3r_status vq3r_rel_frobenius_error_outliers(const void* W, vq3r_dtype w_dtype, const uint8_t* idx,
                                              const uint16_t* scales, const float* codebooks, const uint16_t* ocols,
                                              const uint16_t* ovals, int64_t rows, int64_t cols, int64_t k,
                                              double* err_out, void* workspace, size_t ws_bytes,
                                              vq3r_stream stream);
vq3r_status vq3r_gemv_outliers(const vq3r_outlier_desc* mats, int n_mats, int B, vq3r_dtype x_dtype,
                               vq3r_stream stream);

/*
 * Outlier tiles -- the layout vq3r_gemv_with_outliers streams: per 512-row
 * tile t of a matrix and outlier number q (0 <= q < k), 512 uint32 words
 *   otiles[(t * k + q) * 512 + r] = ocols[512 t + r][q] | ovals[512 t + r][q] << 16
 * for rows 512 t + r < rows, and 0xFFFFFFFF past the last row, so the q-th
 * outliers of a tile's rows are one contiguous 2 KiB block (4 bytes per
 * outlier, like ocols + ovals).
 * vq3r_outliers_tiles_size: bytes of that layout, ceil(rows / 512) * k * 2048
 *   (0 for a negative size or k > 16384).
 * vq3r_pack_outliers: ocols / ovals [rows][k] (as vq3r_outliers writes them)
 *   -> otiles (DEVICE, 16-byte aligned).  rows == 0 or k == 0 is a no-op.
 *
 * vq3r_gemv_with_outliers -- y = (W_hat + O) . x in one call: vq3r_gemv of
 * mats and the sparse outlier product of outl[i] for each matrix i.
 * outl[i].otiles points at the outlier tile block of mats[i]'s first row
 * (a row range of a larger matrix starts at a multiple of 512 rows, as for
 * TILES indices); outl[i].k = 0 marks a matrix without outliers (otiles may
 * then be NULL), otherwise 0 < k <= cols <= 16384.  Workspace, B, x_dtype and
 * the other conditions are vq3r_gemv's.  Per row i and token b the
 * outliers' part is sum_q (float)o_iq * x[b][c_iq] in binary32 (fused
 * multiply-adds, q ascending).  TILES calls that run on the lookup-table
 * kernel (F32 and F16 x, and bf16 x below 11 tokens) compute it inside that
 * kernel's single launch, as the value y starts from instead of zero, before
 * the lookups add into it.  Other calls launch vq3r_gemv and then a sparse
 * add over the outlier tiles, which adds it to y.
 */
typedef struct {
  const uint32_t* otiles;   /* outlier tiles of the matrix's first row, DEVICE */
  int64_t k;                /* outliers per row; 0: none */
} vq3r_outlier_tiles;

size_t vq3r_outliers_tiles_size(int64_t rows, int64_t k);
vq3r_status vq3r_pack_outliers(const uint16_t* ocols, const uint16_t* ovals, int64_t rows, int64_t k, uint32_t* otiles,
                               vq3r_stream stream);
vq3r_status vq3r_gemv_with_outliers(const vq3r_gemv_desc* mats, const vq3r_outlier_tiles* outl, int n_mats, int B,
                                    vq3r_dtype x_dtype, void* workspace, size_t ws_bytes, vq3r_stream stream);

/* Human-readable name of a status code (static string). */
const char* vq3r_status_string(vq3r_status s);

/* cudaError_t value of the most recent VQ3R_ERR_CUDA on the calling thread (0 if none). */
int vq3r_last_cuda_error(void);

/* Device-side error word, set by a kernel whose bounded wait gave up
 * (0 = none; 1 = a shared-memory bulk copy did not complete; 2 = not all
 * CTAs of a vq3r_gemv TILES call reached its grid barrier).  Synchronises the current device;
 * reading it clears it. */
vq3r_status vq3r_device_error(int* code);

/* Failure-path self-test: launches one warp that waits on a shared-memory
 * barrier nothing completes.  After about one second the bounded wait gives
 * up and records device error 1 (read it with vq3r_device_error); the kernel
 * returns and the context stays usable.  Takes about one second. */
vq3r_status vq3r_selftest_wait_timeout(vq3r_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* VQ3R_H */
