"""VQ3R codec for NVIDIA B200: thin Python binding of libvq3r.so.

The names mirror the C ABI in include/vq3r.h (vq3r_encode, vq3r_decode,
vq3r_gemv, vq3r_rel_frobenius_error).  This module only marshals arguments:
torch supplies device memory and the current stream; every step of the
codec runs in the library's CUDA kernels.  There is no CPU fallback: if
the library is missing, importing a function raises.
"""
import ctypes
import os

import torch

_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_DIR, "csrc", "libvq3r.so")

VQ3R_F32, VQ3R_BF16, VQ3R_F16 = 0, 1, 2
_DT = {torch.float32: VQ3R_F32, torch.bfloat16: VQ3R_BF16, torch.float16: VQ3R_F16}
STAGES, CODEWORDS, DIM = 3, 256, 8
VQ4P_STAGES, VQ4P_CODEWORDS = 4, 64  # VQ4P: 4 stages x 64 codewords, indices packed in 3 byte planes
GEMV_MAX_B = 32
GEMV_MAX_MATS = 32
LAYOUT_PLANES, LAYOUT_TILES = 0, 1
TILE_ROWS, TILE_BYTES, SLAB_COLS = 512, 32768, 512

EXPORTED = ["vq3r_encode", "vq3r_decode", "vq3r_gemv", "vq3r_gemv_workspace_size", "vq3r_rel_frobenius_error",
            "vq3r_rel_frobenius_workspace_size", "vq3r_status_string", "vq3r_last_cuda_error",
            "vq3r_device_error", "vq3r_gemv_noalloc", "vq3r_tiles_size", "vq3r_pack_tiles", "vq3r_gemm",
            "vq3r_train", "vq3r_train_workspace_size", "vq4p_encode", "vq4p_decode", "vq4p_rel_frobenius_error",
            "vq4p_train", "vq4p_train_workspace_size", "vq3r_outliers", "vq3r_decode_outliers",
            "vq3r_rel_frobenius_error_outliers", "vq3r_rel_frobenius_outliers_workspace_size", "vq3r_gemv_outliers",
            "vq3r_selftest_wait_timeout", "vq4p_gemv", "vq3r_outliers_tiles_size", "vq3r_pack_outliers",
            "vq3r_gemv_with_outliers"]


class VQ3RError(RuntimeError):
    def __init__(self, status, where):
        msg = _lib().vq3r_status_string(status).decode()
        if status == 6:
            msg += " (cudaError %d)" % _lib().vq3r_last_cuda_error()
        super().__init__("%s: %s" % (where, msg))
        self.status = status


class GemvDesc(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("codebooks", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("plane_stride", ctypes.c_int64), ("layout", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class GemmDesc(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("codebooks", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("plane_stride", ctypes.c_int64), ("tokens", ctypes.c_int64), ("reserved", ctypes.c_int64)]


class OutlierDesc(ctypes.Structure):
    _fields_ = [("ocols", ctypes.c_void_p), ("ovals", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("k", ctypes.c_int64), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("reserved", ctypes.c_int64)]


_L = None


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libvq3r.so is not built (run residual_vector_quantization_b200.build.build())")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.vq3r_encode.argtypes = [P, I32, I64, I64, P, P, P, P]
        L.vq3r_decode.argtypes = [P, P, P, I64, I64, P, I32, P]
        L.vq3r_gemv.argtypes = [P, I32, I32, I32, P, SZ, P]
        L.vq3r_gemv_workspace_size.argtypes = [P, I32, I32]
        L.vq3r_gemv_noalloc.argtypes = [P, I32, I32, I32, P]
        L.vq4p_gemv.argtypes = L.vq3r_gemv.argtypes
        L.vq3r_tiles_size.argtypes = [I64, I64]
        L.vq3r_tiles_size.restype = SZ
        L.vq3r_pack_tiles.argtypes = [P, I64, I64, I64, P, P]
        L.vq3r_gemv_workspace_size.restype = SZ
        L.vq3r_rel_frobenius_error.argtypes = [P, I32, P, P, P, I64, I64, P, P, SZ, P]
        L.vq3r_rel_frobenius_workspace_size.argtypes = [I64, I64]
        L.vq3r_rel_frobenius_workspace_size.restype = SZ
        L.vq3r_status_string.argtypes = [I32]
        L.vq3r_status_string.restype = ctypes.c_char_p
        L.vq3r_last_cuda_error.restype = I32
        L.vq3r_device_error.argtypes = [P]
        L.vq3r_gemm.argtypes = [P, I32, I32, P]
        L.vq3r_train.argtypes = [P, I64, I32, I32, P, P, P, SZ, P]
        L.vq3r_train_workspace_size.argtypes = [I64]
        L.vq3r_train_workspace_size.restype = SZ
        L.vq4p_encode.argtypes = L.vq3r_encode.argtypes
        L.vq4p_decode.argtypes = L.vq3r_decode.argtypes
        L.vq4p_rel_frobenius_error.argtypes = L.vq3r_rel_frobenius_error.argtypes
        L.vq4p_train.argtypes = L.vq3r_train.argtypes
        L.vq4p_train_workspace_size.argtypes = [I64]
        L.vq4p_train_workspace_size.restype = SZ
        L.vq3r_outliers.argtypes = [P, I32, P, P, P, I64, I64, I64, P, P, P]
        L.vq3r_decode_outliers.argtypes = [P, P, P, P, P, I64, I64, I64, P, P]
        L.vq3r_rel_frobenius_outliers_workspace_size.argtypes = [I64, I64, I64]
        L.vq3r_rel_frobenius_outliers_workspace_size.restype = SZ
        L.vq3r_rel_frobenius_error_outliers.argtypes = [P, I32, P, P, P, P, P, I64, I64, I64, P, P, SZ, P]
        L.vq3r_gemv_outliers.argtypes = [P, I32, I32, I32, P]
        L.vq3r_gemv_with_outliers.argtypes = [P, P, I32, I32, I32, P, SZ, P]
        L.vq3r_outliers_tiles_size.argtypes = [I64, I64]
        L.vq3r_outliers_tiles_size.restype = SZ
        L.vq3r_pack_outliers.argtypes = [P, P, I64, I64, P, P]
        L.vq3r_selftest_wait_timeout.argtypes = [P]
        L.vq3r_selftest_wait_timeout.restype = I32
        for f in ("vq3r_encode", "vq3r_decode", "vq3r_gemv", "vq3r_rel_frobenius_error", "vq3r_device_error",
                  "vq3r_gemv_noalloc", "vq3r_pack_tiles", "vq3r_gemm", "vq3r_train", "vq4p_encode", "vq4p_decode",
                  "vq4p_rel_frobenius_error", "vq4p_train", "vq4p_gemv", "vq3r_outliers", "vq3r_decode_outliers",
                  "vq3r_rel_frobenius_error_outliers", "vq3r_gemv_outliers", "vq3r_gemv_with_outliers", "vq3r_pack_outliers"):
            getattr(L, f).restype = I32
        _L = L
    return _L


def lib():
    """The loaded ctypes handle of libvq3r.so."""
    return _lib()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(st, where):
    if st != 0:
        raise VQ3RError(st, where)


def _dev(t, name):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous()):
        raise ValueError("%s must be a contiguous CUDA tensor" % name)
    return t.data_ptr()


def _encode(fn, W, codebooks, idx, scales, stream):
    rows, cols = W.shape
    if idx is None:
        idx = torch.empty((STAGES, rows, cols // DIM), dtype=torch.uint8, device=W.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.int16, device=W.device)
    if W.dtype not in _DT:
        raise ValueError("W dtype must be float32, bfloat16 or float16")
    _check(getattr(_lib(), fn)(_dev(W, "W"), _DT[W.dtype], rows, cols, _dev(codebooks, "codebooks"),
                               _dev(idx, "idx"), _dev(scales, "scales"), _stream(stream)), fn)
    return idx, scales


def _decode(fn, idx, scales, codebooks, out_dtype, out, stream):
    _, rows, V = idx.shape
    if out is None:
        out = torch.empty((rows, V * DIM), dtype=out_dtype, device=idx.device)
    _check(getattr(_lib(), fn)(_dev(idx, "idx"), _dev(scales, "scales"), _dev(codebooks, "codebooks"), rows,
                               V * DIM, _dev(out, "out"), _DT[out.dtype], _stream(stream)), fn)
    return out


def vq3r_encode(W, codebooks, idx=None, scales=None, stream=None):
    """Encode W [rows][cols] (f32/bf16/f16) -> (idx uint8 [3][rows][cols/8], scales int16 [rows] fp16 bits)."""
    return _encode("vq3r_encode", W, codebooks, idx, scales, stream)


def vq3r_decode(idx, scales, codebooks, out_dtype=torch.float32, out=None, stream=None):
    """Reconstruct W_hat [rows][cols] as float32 or float16."""
    return _decode("vq3r_decode", idx, scales, codebooks, out_dtype, out, stream)


def vq4p_encode(W, codebooks, planes=None, scales=None, stream=None):
    """VQ4P encode with codebooks [4][64][8] -> (planes uint8 [3][rows][cols/8] holding the packed 24-bit
    index words, scales int16 [rows] fp16 bits)."""
    return _encode("vq4p_encode", W, codebooks, planes, scales, stream)


def vq4p_decode(planes, scales, codebooks, out_dtype=torch.float32, out=None, stream=None):
    """Reconstruct W_hat [rows][cols] from VQ4P planes as float32 or float16."""
    return _decode("vq4p_decode", planes, scales, codebooks, out_dtype, out, stream)


def _descs(mats):
    """ctypes descriptor array for vq3r_gemv.  Each entry is a dict with
    idx, scales, codebooks, x [B][cols], y [B][rows] and optionally:
      layout "tiles": idx is a tiled tensor from vq3r_pack_tiles (1-D uint8)
                      and "cols" gives the matrix width;
      row0, rows:     a row range of a larger encoded (or packed) matrix; for
                      tiles row0 must be a multiple of 512."""
    arr = (GemvDesc * len(mats))()
    for i, m in enumerate(mats):
        idx, scales, cb, x, y = m["idx"], m["scales"], m["codebooks"], m["x"], m["y"]
        if not (idx.is_cuda and idx.is_contiguous() and scales.is_cuda and scales.is_contiguous()):
            raise ValueError("idx and scales must be contiguous CUDA tensors")
        if m.get("layout", "planes") == "tiles":
            cols = m["cols"]
            total_rows = scales.shape[0]
            r0, rows = m.get("row0", 0), m.get("rows", total_rows)
            if r0 % TILE_ROWS:
                raise ValueError("row0 of a tiled matrix must be a multiple of 512")
            n_tiles = (total_rows + TILE_ROWS - 1) // TILE_ROWS
            arr[i] = GemvDesc(idx.data_ptr() + (r0 // TILE_ROWS) * TILE_BYTES, scales.data_ptr() + 2 * r0,
                              _dev(cb, "codebooks"), rows, cols, _dev(x, "x"), _dev(y, "y"), n_tiles * TILE_BYTES,
                              LAYOUT_TILES, 0)
        elif "rows" in m:
            # a row range of a larger encoded matrix: idx is the full [3][R][V] tensor
            r0, rows = m.get("row0", 0), m["rows"]
            V = idx.shape[2]
            arr[i] = GemvDesc(idx.data_ptr() + r0 * V, scales.data_ptr() + 2 * r0, _dev(cb, "codebooks"), rows,
                              V * DIM, _dev(x, "x"), _dev(y, "y"), idx.shape[1] * V, LAYOUT_PLANES, 0)
        else:
            arr[i] = GemvDesc(_dev(idx, "idx"), _dev(scales, "scales"), _dev(cb, "codebooks"), idx.shape[1],
                              idx.shape[2] * DIM, _dev(x, "x"), _dev(y, "y"), 0, LAYOUT_PLANES, 0)
    return arr


def _gemm_descs(mats):
    """ctypes descriptor array for vq3r_gemm.  Each entry is a dict with idx (a tiled tensor from
    vq3r_pack_tiles), scales, codebooks, cols, x [T][cols] bf16, y [T][rows] float32 and optionally row0, rows
    (a row range of a larger packed matrix, row0 a multiple of 512)."""
    arr = (GemmDesc * len(mats))()
    for i, m in enumerate(mats):
        idx, scales, cb, x, y = m["idx"], m["scales"], m["codebooks"], m["x"], m["y"]
        if not (idx.is_cuda and idx.is_contiguous() and scales.is_cuda and scales.is_contiguous()):
            raise ValueError("idx and scales must be contiguous CUDA tensors")
        if x.dtype != torch.bfloat16:
            raise ValueError("x must be bfloat16")
        total_rows = scales.shape[0]
        r0, rows = m.get("row0", 0), m.get("rows", total_rows)
        if r0 % TILE_ROWS:
            raise ValueError("row0 of a tiled matrix must be a multiple of 512")
        n_tiles = (total_rows + TILE_ROWS - 1) // TILE_ROWS
        arr[i] = GemmDesc(idx.data_ptr() + (r0 // TILE_ROWS) * TILE_BYTES, scales.data_ptr() + 2 * r0,
                          _dev(cb, "codebooks"), rows, m["cols"], _dev(x, "x"), _dev(y, "y"), n_tiles * TILE_BYTES,
                          x.shape[0], 0)
    return arr


def vq3r_gemm(mats, stream=None):
    """Prefill product on the tensor cores: y[t][i] = sum_c bf16(w_hat[i][c]) x[t][c] for each descriptor
    dict {idx (tiled), scales, codebooks, cols, x [T][cols] bf16, y [T][rows] float32} (see _gemm_descs)."""
    arr = _gemm_descs(mats)
    _check(_lib().vq3r_gemm(arr, len(mats), _DT[torch.bfloat16], _stream(stream)), "vq3r_gemm")
    return [m["y"] for m in mats]


def vq3r_train_workspace_size(n):
    return _lib().vq3r_train_workspace_size(n)


def vq4p_train_workspace_size(n):
    return _lib().vq4p_train_workspace_size(n)


def _train(fn, K, vecs, iters, nstages, codebooks, trace, workspace, stream):
    n = vecs.shape[0]
    if vecs.dtype != torch.float32 or vecs.dim() != 2 or vecs.shape[1] != DIM:
        raise ValueError("vecs must be a float32 [n][8] tensor")
    if codebooks is None:
        codebooks = torch.empty((nstages, K, DIM), dtype=torch.float32, device=vecs.device)
    if trace is None:
        trace = torch.empty((nstages, iters + 1), dtype=torch.float64, device=vecs.device)
    if workspace is None:
        ws = getattr(_lib(), fn + "_workspace_size")(n)
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=vecs.device)
    _check(getattr(_lib(), fn)(_dev(vecs, "vecs"), n, iters, nstages, _dev(codebooks, "codebooks"),
                               _dev(trace, "trace"), _dev(workspace, "workspace"), workspace.numel(),
                               _stream(stream)), fn)
    return codebooks, trace


def vq3r_train(vecs, iters, nstages=STAGES, codebooks=None, trace=None, workspace=None, stream=None):
    """Lloyd codebooks from training vectors [n][8] float32 -> (codebooks [nstages][256][8] float32,
    trace [nstages][iters + 1] float64: the total squared distance after each assignment)."""
    return _train("vq3r_train", CODEWORDS, vecs, iters, nstages, codebooks, trace, workspace, stream)


def vq4p_train(vecs, iters, nstages=VQ4P_STAGES, codebooks=None, trace=None, workspace=None, stream=None):
    """VQ4P Lloyd codebooks [nstages][64][8] float32 and the distortion trace, as vq3r_train."""
    return _train("vq4p_train", VQ4P_CODEWORDS, vecs, iters, nstages, codebooks, trace, workspace, stream)


def vq3r_tiles_size(rows, cols):
    return _lib().vq3r_tiles_size(rows, cols)


def vq3r_pack_tiles(idx, out=None, stream=None):
    """Repack index planes [3][rows][cols/8] into the tiled layout (1-D uint8 tensor)."""
    _, rows, V = idx.shape
    n = vq3r_tiles_size(rows, V * DIM)
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=idx.device)
    _check(_lib().vq3r_pack_tiles(_dev(idx, "idx"), rows, V * DIM, 0, _dev(out, "out"), _stream(stream)),
           "vq3r_pack_tiles")
    return out


def vq3r_gemv_workspace_size(mats, B):
    arr = _descs(mats)
    return _lib().vq3r_gemv_workspace_size(arr, len(mats), B)


def vq3r_gemv(mats, B, workspace=None, stream=None):
    """y = W_hat . x for each descriptor dict {idx, scales, codebooks, x [B][cols], y [B][rows] float32}.

    With keys "row0" and "rows" the descriptor covers rows [row0, row0 + rows) of the
    encoded matrix (idx [3][R][V], scales [R]), e.g. one expert of a stacked layer."""
    arr = _descs(mats)
    ws = _lib().vq3r_gemv_workspace_size(arr, len(mats), B)
    if workspace is None:
        workspace = torch.zeros(max(ws, 16), dtype=torch.uint8, device=mats[0]["idx"].device)
    xdt = _DT[mats[0]["x"].dtype]
    _check(_lib().vq3r_gemv(arr, len(mats), B, xdt, _dev(workspace, "workspace"), workspace.numel(),
                            _stream(stream)), "vq3r_gemv")
    return [m["y"] for m in mats]


def vq4p_gemv(mats, B, workspace=None, stream=None):
    """y = W_hat . x for VQ4P matrices: descriptor dicts as for vq3r_gemv with layout "tiles" (planes
    repacked by vq3r_pack_tiles) and codebooks [4][64][8]."""
    arr = _descs(mats)
    ws = _lib().vq3r_gemv_workspace_size(arr, len(mats), B)
    if workspace is None:
        workspace = torch.zeros(max(ws, 16), dtype=torch.uint8, device=mats[0]["idx"].device)
    xdt = _DT[mats[0]["x"].dtype]
    _check(_lib().vq4p_gemv(arr, len(mats), B, xdt, _dev(workspace, "workspace"), workspace.numel(),
                            _stream(stream)), "vq4p_gemv")
    return [m["y"] for m in mats]


def vq3r_gemv_noalloc(mats, B, stream=None):
    """vq3r_gemv without a workspace argument: the library's own static device
    scratch (16 MiB, shared by all calls; overlapping calls race) is used and
    nothing is allocated, here or in the library."""
    arr = _descs(mats)
    xdt = _DT[mats[0]["x"].dtype]
    _check(_lib().vq3r_gemv_noalloc(arr, len(mats), B, xdt, _stream(stream)), "vq3r_gemv_noalloc")
    return [m["y"] for m in mats]


def vq3r_rel_frobenius_workspace_size(rows, cols):
    return _lib().vq3r_rel_frobenius_workspace_size(rows, cols)


def _relfro(fn, W, idx, scales, codebooks, out, workspace, stream):
    rows, cols = W.shape
    if out is None:
        out = torch.empty(1, dtype=torch.float64, device=W.device)
    if workspace is None:
        workspace = torch.empty(vq3r_rel_frobenius_workspace_size(rows, cols), dtype=torch.uint8, device=W.device)
    _check(getattr(_lib(), fn)(_dev(W, "W"), _DT[W.dtype], _dev(idx, "idx"), _dev(scales, "scales"),
                               _dev(codebooks, "codebooks"), rows, cols, _dev(out, "out"),
                               _dev(workspace, "workspace"), workspace.numel(), _stream(stream)), fn)
    return out


def vq3r_rel_frobenius_error(W, idx, scales, codebooks, out=None, workspace=None, stream=None):
    """Device float64 tensor [1] holding sqrt(sum (w - w_hat)^2 / sum w^2)."""
    return _relfro("vq3r_rel_frobenius_error", W, idx, scales, codebooks, out, workspace, stream)


def vq4p_rel_frobenius_error(W, planes, scales, codebooks, out=None, workspace=None, stream=None):
    """vq3r_rel_frobenius_error for VQ4P planes and codebooks [4][64][8]."""
    return _relfro("vq4p_rel_frobenius_error", W, planes, scales, codebooks, out, workspace, stream)


def vq3r_outliers(W, idx, scales, codebooks, k, ocols=None, ovals=None, stream=None):
    """Sparse FP16 outlier residual of W over its VQ3R encoding: the k largest |w - w_hat| per row ->
    (ocols uint16-as-int16 [rows][k], ovals int16 [rows][k] binary16 bits)."""
    rows, cols = W.shape
    if W.dtype not in _DT:
        raise ValueError("W dtype must be float32, bfloat16 or float16")
    if ocols is None:
        ocols = torch.empty((rows, k), dtype=torch.int16, device=W.device)
    if ovals is None:
        ovals = torch.empty((rows, k), dtype=torch.int16, device=W.device)
    _check(_lib().vq3r_outliers(_dev(W, "W"), _DT[W.dtype], _dev(idx, "idx"), _dev(scales, "scales"),
                                _dev(codebooks, "codebooks"), rows, cols, k, _dev(ocols, "ocols"),
                                _dev(ovals, "ovals"), _stream(stream)), "vq3r_outliers")
    return ocols, ovals


def vq3r_decode_outliers(idx, scales, codebooks, ocols, ovals, out=None, stream=None):
    """W_hat [rows][cols] float32 with the outliers added."""
    _, rows, V = idx.shape
    k = ocols.shape[1]
    if out is None:
        out = torch.empty((rows, V * DIM), dtype=torch.float32, device=idx.device)
    _check(_lib().vq3r_decode_outliers(_dev(idx, "idx"), _dev(scales, "scales"), _dev(codebooks, "codebooks"),
                                       _dev(ocols, "ocols"), _dev(ovals, "ovals"), rows, V * DIM, k,
                                       _dev(out, "out"), _stream(stream)), "vq3r_decode_outliers")
    return out


def vq3r_rel_frobenius_outliers_workspace_size(rows, cols, k):
    return _lib().vq3r_rel_frobenius_outliers_workspace_size(rows, cols, k)


def vq3r_rel_frobenius_error_outliers(W, idx, scales, codebooks, ocols, ovals, out=None, workspace=None,
                                      stream=None):
    """Device float64 tensor [1]: the relative Frobenius error of the decode with outliers."""
    rows, cols = W.shape
    k = ocols.shape[1]
    if out is None:
        out = torch.empty(1, dtype=torch.float64, device=W.device)
    if workspace is None:
        workspace = torch.empty(vq3r_rel_frobenius_outliers_workspace_size(rows, cols, k), dtype=torch.uint8,
                                device=W.device)
    _check(_lib().vq3r_rel_frobenius_error_outliers(
        _dev(W, "W"), _DT[W.dtype], _dev(idx, "idx"), _dev(scales, "scales"), _dev(codebooks, "codebooks"),
        _dev(ocols, "ocols"), _dev(ovals, "ovals"), rows, cols, k, _dev(out, "out"), _dev(workspace, "workspace"),
        workspace.numel(), _stream(stream)), "vq3r_rel_frobenius_error_outliers")
    return out


def _outlier_descs(mats):
    arr = (OutlierDesc * len(mats))()
    for i, m in enumerate(mats):
        oc, ov, x, y = m["ocols"], m["ovals"], m["x"], m["y"]
        r0 = m.get("row0", 0)
        rows = m.get("rows", oc.shape[0])
        k = oc.shape[1]
        if not (oc.is_cuda and oc.is_contiguous() and ov.is_cuda and ov.is_contiguous()):
            raise ValueError("ocols and ovals must be contiguous CUDA tensors")
        arr[i] = OutlierDesc(oc.data_ptr() + 2 * r0 * k, ov.data_ptr() + 2 * r0 * k, rows, m["cols"], k,
                             _dev(x, "x"), _dev(y, "y"), 0)
    return arr


def vq3r_gemv_outliers(mats, B, stream=None):
    """y += the outliers' product for each dict {ocols, ovals, cols, x [B][cols], y [B][rows]} (optionally
    row0, rows: a row range of a larger matrix's outliers), in one launch; enqueue after vq3r_gemv."""
    arr = _outlier_descs(mats)
    xdt = _DT[mats[0]["x"].dtype]
    _check(_lib().vq3r_gemv_outliers(arr, len(mats), B, xdt, _stream(stream)), "vq3r_gemv_outliers")
    return [m["y"] for m in mats]


class OutlierTiles(ctypes.Structure):
    _fields_ = [("otiles", ctypes.c_void_p), ("k", ctypes.c_int64)]


def vq3r_pack_outliers(ocols, ovals, out=None, stream=None):
    """Outliers [rows][k] (from vq3r_outliers) -> the outlier-tile layout, an int32 tensor [ceil(rows/512)][k][512]
    of column | value << 16 words."""
    rows, k = ocols.shape
    n_tiles = (rows + TILE_ROWS - 1) // TILE_ROWS
    if out is None:
        out = torch.empty((n_tiles, k, TILE_ROWS), dtype=torch.int32, device=ocols.device)
    _check(_lib().vq3r_pack_outliers(_dev(ocols, "ocols"), _dev(ovals, "ovals"), rows, k, _dev(out, "out"),
                                     _stream(stream)), "vq3r_pack_outliers")
    return out


def _outlier_tiles(mats):
    """vq3r_outlier_tiles array: a dict's "otiles" (from vq3r_pack_outliers; its row0, a multiple of 512, picks the
    first tile) or k = 0 where it has none."""
    arr = (OutlierTiles * len(mats))()
    for i, m in enumerate(mats):
        ot = m.get("otiles")
        if ot is None:
            arr[i] = OutlierTiles(None, 0)
            continue
        if not (ot.is_cuda and ot.is_contiguous() and ot.dim() == 3):
            raise ValueError("otiles must be a contiguous CUDA tensor from vq3r_pack_outliers")
        r0 = m.get("row0", 0)
        if r0 % TILE_ROWS:
            raise ValueError("row0 of a matrix with outlier tiles must be a multiple of 512")
        k = ot.shape[1]
        arr[i] = OutlierTiles(ot.data_ptr() + (r0 // TILE_ROWS) * k * TILE_ROWS * 4, k)
    return arr


def vq3r_gemv_with_outliers(mats, B, workspace=None, stream=None):
    """y = (W_hat + O) . x: vq3r_gemv's descriptor dicts, each optionally with "otiles" (the matrix's outliers
    packed by vq3r_pack_outliers; with row0 / rows, rows of that larger matrix as for idx)."""
    garr = _descs(mats)
    oarr = _outlier_tiles(mats)
    ws = _lib().vq3r_gemv_workspace_size(garr, len(mats), B)
    if workspace is None:
        workspace = torch.zeros(max(ws, 16), dtype=torch.uint8, device=mats[0]["idx"].device)
    xdt = _DT[mats[0]["x"].dtype]
    _check(_lib().vq3r_gemv_with_outliers(garr, oarr, len(mats), B, xdt, _dev(workspace, "workspace"),
                                          workspace.numel(), _stream(stream)), "vq3r_gemv_with_outliers")
    return [m["y"] for m in mats]


def vq3r_selftest_wait_timeout(stream=None):
    """Launch the failure-path self-test (a bounded wait that runs out after about one second)."""
    _check(_lib().vq3r_selftest_wait_timeout(_stream(stream)), "vq3r_selftest_wait_timeout")


def vq3r_device_error():
    code = ctypes.c_int(0)
    _check(_lib().vq3r_device_error(ctypes.byref(code)), "vq3r_device_error")
    return code.value
