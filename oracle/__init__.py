"""VQ3R oracle (Python side): ctypes marshalling around the plain C oracle in
vq3r_oracle.c.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg use it; the product path never imports it.

Every function here is marshalling; the arithmetic is in vq3r_oracle.c,
which cites the passages of "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验"
(xdnf.cn/news/289497) that each step follows.
"""
import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_DIR, "libvq3r_oracle.so")
_SRC = os.path.join(_DIR, "vq3r_oracle.c")

DTYPES = {"f32": 0, "bf16": 1, "f16": 2}
K, D = 256, 8


def build():
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                           "-fPIC", "-shared", "-o", _SO, _SRC, "-lm"])


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
            build()
        L = ctypes.CDLL(_SO)
        P, I64, I32, D_ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.orc_set_threads.argtypes = [I32]
        L.orc_max_threads.restype = I32
        L.orc_fp16_from_double_sat.argtypes = [D_]
        L.orc_fp16_from_double_sat.restype = ctypes.c_uint16
        L.orc_fp16_from_float.argtypes = [ctypes.c_float]
        L.orc_fp16_from_float.restype = ctypes.c_uint16
        L.orc_fp16_to_double.argtypes = [ctypes.c_uint16]
        L.orc_fp16_to_double.restype = D_
        L.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_float.restype = ctypes.c_float
        L.orc_bf16_from_float.argtypes = [ctypes.c_float]
        L.orc_bf16_from_float.restype = ctypes.c_uint16
        L.orc_row_sumsq.argtypes = [P, I32, I64, I64]
        L.orc_row_sumsq.restype = D_
        L.orc_row_scales.argtypes = [P, I32, I64, I64, P]
        L.orc_normalize_rows.argtypes = [P, I32, I64, I64, P, P]
        L.orc_encode_vectors.argtypes = [P, I64, P, I32, P, P]
        L.orc_encode.argtypes = [P, I32, I64, I64, P, I32, P, P]
        L.orc_encode.restype = I32
        L.orc_decode.argtypes = [P, P, P, I64, I64, I32, P, I32]
        L.orc_decode.restype = I32
        L.orc_rel_frobenius.argtypes = [P, I32, P, I64]
        L.orc_rel_frobenius.restype = D_
        L.orc_gemv.argtypes = [P, I64, I64, P, I32, I32, P]
        L.orc_gemv.restype = I32
        L.orc_lloyd_train.argtypes = [P, I64, I32, I32, P, P]
        L.orc_lloyd_train.restype = I32
        L.orc_rtn4_row.argtypes = [P, I32, I64, I64, P, P]
        L.orc_rtn4_row.restype = I32
        L.orc_bruteforce_joint.argtypes = [P, I64, P, P, P]
        L.orc_vq4p_pack.argtypes = [P, I64, P]
        L.orc_vq4p_unpack.argtypes = [P, I64, P]
        L.orc_vq4p_encode_vectors.argtypes = [P, I64, P, P, P]
        L.orc_vq4p_encode.argtypes = [P, I32, I64, I64, P, P, P]
        L.orc_vq4p_encode.restype = I32
        L.orc_vq4p_decode.argtypes = [P, P, P, I64, I64, P, I32]
        L.orc_vq4p_decode.restype = I32
        L.orc_vq4p_train.argtypes = [P, I64, I32, P, P]
        L.orc_vq4p_train.restype = I32
        L.orc_vq4p_bruteforce.argtypes = [P, I64, P, P, P]
        L.orc_outliers_select.argtypes = [P, I32, P, I64, I64, I64, P, P]
        L.orc_outliers_select.restype = I32
        L.orc_outliers_apply.argtypes = [P, I64, I64, I64, P, P]
        L.orc_outliers_apply.restype = I32
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _w(W, dtype):
    return _c(W, np.float32 if dtype == "f32" else np.uint16)


def set_threads(n):
    lib().orc_set_threads(int(n))


def max_threads():
    return lib().orc_max_threads()


def fp16_from_double_sat(x):
    return lib().orc_fp16_from_double_sat(float(x))


def fp16_from_float(x):
    return lib().orc_fp16_from_float(float(np.float32(x)))


def fp16_to_double(h):
    return lib().orc_fp16_to_double(int(h))


def bf16_to_float(b):
    return lib().orc_bf16_to_float(int(b))


def row_sumsq(W, dtype, row):
    W = _w(W, dtype)
    return lib().orc_row_sumsq(W.ctypes.data, DTYPES[dtype], row, W.shape[1])


def row_scales(W, dtype):
    W = _w(W, dtype)
    out = np.empty(W.shape[0], dtype=np.uint16)
    lib().orc_row_scales(W.ctypes.data, DTYPES[dtype], W.shape[0], W.shape[1], out.ctypes.data)
    return out


def normalize_rows(W, dtype, scales):
    W = _w(W, dtype)
    scales = _c(scales, np.uint16)
    out = np.empty((W.shape[0] * (W.shape[1] // D), D), dtype=np.float32)
    lib().orc_normalize_rows(W.ctypes.data, DTYPES[dtype], W.shape[0], W.shape[1], scales.ctypes.data,
                             out.ctypes.data)
    return out


def encode_vectors(r, codebooks, nstages=3):
    r = _c(r, np.float32).reshape(-1, D)
    cb = _c(codebooks, np.float32)
    idx = np.empty((r.shape[0], nstages), dtype=np.uint8)
    res = np.empty_like(r)
    lib().orc_encode_vectors(r.ctypes.data, r.shape[0], cb.ctypes.data, nstages, idx.ctypes.data,
                             res.ctypes.data)
    return idx, res


def encode(W, dtype, codebooks, nstages=3):
    """-> (idx uint8 [nstages][rows][cols/8], scales uint16 [rows] binary16 bits)."""
    W = _w(W, dtype)
    rows, cols = W.shape
    cb = _c(codebooks, np.float32)
    idx = np.empty((nstages, rows, cols // D), dtype=np.uint8)
    sc = np.empty(rows, dtype=np.uint16)
    rc = lib().orc_encode(W.ctypes.data, DTYPES[dtype], rows, cols, cb.ctypes.data, nstages, idx.ctypes.data,
                          sc.ctypes.data)
    if rc:
        raise ValueError("orc_encode: bad shape")
    return idx, sc


def decode(idx, scales, codebooks, out="f32"):
    idx = _c(idx, np.uint8)
    nstages, rows, V = idx.shape
    scales = _c(scales, np.uint16)
    cb = _c(codebooks, np.float32)
    o = np.empty((rows, V * D), dtype=np.float32 if out == "f32" else np.uint16)
    rc = lib().orc_decode(idx.ctypes.data, scales.ctypes.data, cb.ctypes.data, rows, V * D, nstages,
                          o.ctypes.data, DTYPES[out])
    if rc:
        raise ValueError("orc_decode: bad shape")
    return o


def gemm(idx, scales, codebooks, x):
    """Prefill product Y[t][i] = sum_c bf16(w_hat[i][c]) * x[t][c] in binary64 for bf16 x [T][cols]: the
    weights as decode writes them, rounded to bfloat16 (RNE), the operand type of a bf16 tensor-core product.
    The pages define no batched product; this reading keeps decode's arithmetic and adds one rounding."""
    Wb = decode(idx, scales, codebooks, out="bf16")
    W = (Wb.astype(np.uint32) << 16).view(np.float32)
    return gemv(W, x, "bf16")


def rel_frobenius(W, dtype, What):
    W = _w(W, dtype)
    What = _c(What, np.float32)
    assert W.size == What.size
    return lib().orc_rel_frobenius(W.ctypes.data, DTYPES[dtype], What.ctypes.data, W.size)


def gemv(What, x, x_dtype):
    """y[b][i] = sum_c What[i][c] x[b][c] in binary64; x is [B][cols]."""
    What = _c(What, np.float32)
    x = _w(np.atleast_2d(x), x_dtype)
    rows, cols = What.shape
    B = x.shape[0]
    y = np.empty((B, rows), dtype=np.float64)
    rc = lib().orc_gemv(What.ctypes.data, rows, cols, x.ctypes.data, DTYPES[x_dtype], B, y.ctypes.data)
    if rc:
        raise ValueError("orc_gemv: bad shape")
    return y


def lloyd_train(vecs, iters, nstages=3):
    """-> (codebooks float32 [nstages][256][8], trace float64 [nstages][iters+1])."""
    v = _c(vecs, np.float32).reshape(-1, D)
    cb = np.empty((nstages, K, D), dtype=np.float32)
    tr = np.empty((nstages, iters + 1), dtype=np.float64)
    rc = lib().orc_lloyd_train(v.ctypes.data, v.shape[0], iters, nstages, cb.ctypes.data, tr.ctypes.data)
    if rc:
        raise ValueError("orc_lloyd_train failed (%d)" % rc)
    return cb, tr


def rtn4_row(W, dtype):
    W = _w(W, dtype)
    rows, cols = W.shape
    What = np.empty((rows, cols), dtype=np.float32)
    sc = np.empty(rows, dtype=np.uint16)
    lib().orc_rtn4_row(W.ctypes.data, DTYPES[dtype], rows, cols, What.ctypes.data, sc.ctypes.data)
    return What, sc


def bruteforce_joint(r, codebooks):
    r = _c(r, np.float32).reshape(-1, D)
    cb = _c(codebooks, np.float32)
    idx = np.empty((r.shape[0], 3), dtype=np.int32)
    err = np.empty(r.shape[0], dtype=np.float64)
    lib().orc_bruteforce_joint(r.ctypes.data, r.shape[0], cb.ctypes.data, idx.ctypes.data, err.ctypes.data)
    return idx, err


# ---------------------------------------------------------------- VQ3R's sibling VQ4P (page §5)
# 4 stages x 64-entry codebooks [4][64][8]; the 4 six-bit indices of a vector packed into the 24-bit word
# i1 | i2 << 6 | i3 << 12 | i4 << 18, stored as three byte planes [3][rows][cols/8].

K4, S4 = 64, 4


def vq4p_pack(idx4):
    """[4][...] indices (< 64) -> [3][...] byte planes."""
    idx4 = _c(idx4, np.uint8)
    shape = idx4.shape[1:]
    n = int(np.prod(shape))
    planes = np.empty((3,) + shape, dtype=np.uint8)
    lib().orc_vq4p_pack(idx4.ctypes.data, n, planes.ctypes.data)
    return planes


def vq4p_unpack(planes):
    planes = _c(planes, np.uint8)
    shape = planes.shape[1:]
    n = int(np.prod(shape))
    idx4 = np.empty((4,) + shape, dtype=np.uint8)
    lib().orc_vq4p_unpack(planes.ctypes.data, n, idx4.ctypes.data)
    return idx4


def vq4p_encode_vectors(r, codebooks):
    """Greedy 4-stage assignment of normalised vectors -> (idx [n][4], final residuals [n][8])."""
    r = _c(r, np.float32).reshape(-1, D)
    cb = _c(codebooks, np.float32)
    idx = np.empty((r.shape[0], S4), dtype=np.uint8)
    res = np.empty_like(r)
    lib().orc_vq4p_encode_vectors(r.ctypes.data, r.shape[0], cb.ctypes.data, idx.ctypes.data, res.ctypes.data)
    return idx, res


def vq4p_encode(W, dtype, codebooks):
    """-> (planes uint8 [3][rows][cols/8], scales uint16 [rows] binary16 bits)."""
    W = _w(W, dtype)
    rows, cols = W.shape
    cb = _c(codebooks, np.float32)
    planes = np.empty((3, rows, cols // D), dtype=np.uint8)
    sc = np.empty(rows, dtype=np.uint16)
    rc = lib().orc_vq4p_encode(W.ctypes.data, DTYPES[dtype], rows, cols, cb.ctypes.data, planes.ctypes.data,
                               sc.ctypes.data)
    if rc:
        raise ValueError("orc_vq4p_encode: bad shape")
    return planes, sc


def vq4p_decode(planes, scales, codebooks, out="f32"):
    planes = _c(planes, np.uint8)
    _, rows, V = planes.shape
    scales = _c(scales, np.uint16)
    cb = _c(codebooks, np.float32)
    o = np.empty((rows, V * D), dtype=np.float32 if out == "f32" else np.uint16)
    rc = lib().orc_vq4p_decode(planes.ctypes.data, scales.ctypes.data, cb.ctypes.data, rows, V * D, o.ctypes.data,
                               DTYPES[out])
    if rc:
        raise ValueError("orc_vq4p_decode: bad shape")
    return o


def vq4p_train(vecs, iters):
    """-> (codebooks float32 [4][64][8], trace float64 [4][iters+1])."""
    v = _c(vecs, np.float32).reshape(-1, D)
    cb = np.empty((S4, K4, D), dtype=np.float32)
    tr = np.empty((S4, iters + 1), dtype=np.float64)
    rc = lib().orc_vq4p_train(v.ctypes.data, v.shape[0], iters, cb.ctypes.data, tr.ctypes.data)
    if rc:
        raise ValueError("orc_vq4p_train failed (%d)" % rc)
    return cb, tr


def vq4p_bruteforce(r, codebooks):
    r = _c(r, np.float32).reshape(-1, D)
    cb = _c(codebooks, np.float32)
    idx = np.empty((r.shape[0], 4), dtype=np.int32)
    err = np.empty(r.shape[0], dtype=np.float64)
    lib().orc_vq4p_bruteforce(r.ctypes.data, r.shape[0], cb.ctypes.data, idx.ctypes.data, err.ctypes.data)
    return idx, err


def vq4p_gemv(planes, scales, codebooks, x, x_dtype):
    """y[b][i] = sum_c w_hat[i][c] x[b][c] in binary64 with the VQ4P decoded weights."""
    return gemv(vq4p_decode(planes, scales, codebooks), x, x_dtype)


def outliers_select(W, dtype, What, k):
    """Sparse FP16 outlier residual of W over its decode What: the k largest |(double)w - (double)w_hat| per
    row (ties to the lower column) -> (columns uint16 [rows][k] ascending, fp16 bits uint16 [rows][k])."""
    W = _w(W, dtype)
    What = _c(What, np.float32)
    rows, cols = W.shape
    oc = np.zeros((rows, k), dtype=np.uint16)
    ov = np.zeros((rows, k), dtype=np.uint16)
    rc = lib().orc_outliers_select(W.ctypes.data, DTYPES[dtype], What.ctypes.data, rows, cols, k, oc.ctypes.data,
                                   ov.ctypes.data)
    if rc:
        raise ValueError("orc_outliers_select: bad shape")
    return oc, ov


def outliers_apply(What, ocols, ovals):
    """What with (float)o added at each stored outlier (binary32); returns a new array."""
    out = np.array(What, dtype=np.float32, copy=True, order="C")
    ocols = _c(ocols, np.uint16)
    ovals = _c(ovals, np.uint16)
    rows, cols = out.shape
    k = ocols.shape[1] if ocols.ndim == 2 else 0
    rc = lib().orc_outliers_apply(out.ctypes.data, rows, cols, k, ocols.ctypes.data, ovals.ctypes.data)
    if rc:
        raise ValueError("orc_outliers_apply: bad arguments")
    return out
