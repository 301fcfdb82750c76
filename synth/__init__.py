"""Seeded synthetic inputs for the VQ3R codec (shared by the tests and the
benchmark; holds none of the codec's arithmetic).

Every element is a pure function of (seed, tag, element index) through
Philox4x32-10, so the host library (used for oracle inputs) and the device
library (used for bulk inputs) produce the same values for any row, and
sampled rows can be regenerated on the host at any size.
"""
import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_DIR, "libsynth_host.so")
_DEV_SO = os.path.join(_DIR, "libsynth_dev.so")

DIST_NORMAL = 0
DIST_STUDENT_T = 1
OUT_F32 = 0
OUT_BF16 = 1


class Dist(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("df", ctypes.c_int32), ("row_sigma", ctypes.c_double),
                ("outlier_p", ctypes.c_double), ("outlier_mag", ctypes.c_double)]


def normal():
    return Dist(DIST_NORMAL, 0, 0.0, 0.0, 0.0)


def student_t(df, row_sigma=0.0, outlier_p=0.0, outlier_mag=0.0):
    return Dist(DIST_STUDENT_T, df, row_sigma, outlier_p, outlier_mag)


def build(device=True):
    """Compile the host generator (gcc) and, if requested, the device one (nvcc, sm_100a)."""
    src = os.path.join(_DIR, "synth_host.c")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                           "-o", _HOST_SO, src, "-lm"])
    if device:
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-fmad=false",
                               "-Xcompiler", "-fPIC", "-shared", "-o", _DEV_SO,
                               os.path.join(_DIR, "synth_dev.cu")])


_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(_HOST_SO):
            build(device=False)
        lib = ctypes.CDLL(_HOST_SO)
        lib.synth_fill_rows.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32, ctypes.POINTER(Dist)]
        lib.synth_fill_row_list.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p,
                                            ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32, ctypes.POINTER(Dist)]
        lib.synth_sample.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_void_p]
        lib.synth_philox.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_normal_at.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64,
                                        ctypes.c_uint32]
        lib.synth_normal_at.restype = ctypes.c_double
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(_DEV_SO):
            raise RuntimeError("device generator library missing: run synth.build()")
        lib = ctypes.CDLL(_DEV_SO)
        lib.synth_fill_rows_device.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                               ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                               ctypes.POINTER(Dist), ctypes.c_void_p]
        _dev = lib
    return _dev


def philox(ctr, key):
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    _host_lib().synth_philox(c, k, o)
    return list(o)


def normal_at(seed, purpose, tag, e, j):
    return _host_lib().synth_normal_at(seed, purpose, tag, e, j)


def fill_rows(cols, row0, nrows, seed, tag, dist, dtype="bf16"):
    """Rows [row0, row0+nrows) of a (.. x cols) tensor; bf16 as uint16 bits, or float32."""
    out_dtype = OUT_BF16 if dtype == "bf16" else OUT_F32
    out = np.empty((nrows, cols), dtype=np.uint16 if out_dtype == OUT_BF16 else np.float32)
    rc = _host_lib().synth_fill_rows(out.ctypes.data, out_dtype, cols, row0, nrows, seed, tag,
                                     ctypes.byref(dist))
    if rc:
        raise ValueError("synth_fill_rows failed (%d)" % rc)
    return out


def fill_row_list(cols, rows, seed, tag, dist, dtype="bf16"):
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out_dtype = OUT_BF16 if dtype == "bf16" else OUT_F32
    out = np.empty((len(rows), cols), dtype=np.uint16 if out_dtype == OUT_BF16 else np.float32)
    rc = _host_lib().synth_fill_row_list(out.ctypes.data, out_dtype, cols, rows.ctypes.data, len(rows), seed,
                                         tag, ctypes.byref(dist))
    if rc:
        raise ValueError("synth_fill_row_list failed (%d)" % rc)
    return out


def sample(seed, tag, n, k):
    """k distinct items of [0, n), uniform without replacement, in draw (key) order."""
    out = np.empty(k, dtype=np.int64)
    rc = _host_lib().synth_sample(seed, tag, n, k, out.ctypes.data)
    if rc:
        raise ValueError("synth_sample failed (%d)" % rc)
    return out


def fill_rows_device(ptr, cols, row0, nrows, seed, tag, dist, dtype="bf16", stream=0):
    """Same values as fill_rows, written by a CUDA kernel into device memory at ptr."""
    out_dtype = OUT_BF16 if dtype == "bf16" else OUT_F32
    rc = _dev_lib().synth_fill_rows_device(ctypes.c_void_p(ptr), out_dtype, cols, row0, nrows, seed, tag,
                                           ctypes.byref(dist), ctypes.c_void_p(stream))
    if rc:
        raise RuntimeError("synth_fill_rows_device failed (%d)" % rc)


def bf16_bits_to_f32(a):
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
