"""The C-ABI library loads and exports every entry point include/vq3r.h
declares; host-side argument checks and workspace sizing (no GPU needed)."""
import ctypes
import os
import re

import pytest

import residual_vector_quantization_b200 as vq
from residual_vector_quantization_b200.build import SO

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "vq3r.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b((?:vq3r|vq4p)_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(SO):
        from residual_vector_quantization_b200.build import build
        build()
    return vq.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("vq3r_encode", "vq3r_decode", "vq3r_gemv", "vq3r_rel_frobenius_error", "vq4p_encode", "vq4p_decode",
              "vq4p_rel_frobenius_error", "vq4p_train"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(vq.EXPORTED) == set(declared_functions())  # the binding lists every call the header declares


def test_status_strings(lib):
    for s in range(8):
        assert lib.vq3r_status_string(s).decode().startswith("VQ3R")
    assert lib.vq3r_last_cuda_error() == 0


def test_null_and_shape_errors_return_before_any_launch(lib):
    fake = 0x100000  # never dereferenced: the checks fail first
    assert lib.vq3r_encode(None, 1, 4, 16, fake, fake, fake, None) == 1
    assert lib.vq3r_encode(fake, 1, 4, 12, fake, fake, fake, None) == 2
    assert lib.vq3r_encode(fake, 1, -1, 16, fake, fake, fake, None) == 2
    assert lib.vq3r_encode(fake, 1, 4, 0, fake, fake, fake, None) == 2
    assert lib.vq3r_encode(fake, 7, 4, 16, fake, fake, fake, None) == 4
    assert lib.vq3r_encode(fake + 2, 1, 4, 16, fake, fake, fake, None) == 3
    assert lib.vq3r_encode(fake, 1, 0, 16, fake, fake, fake, None) == 0  # empty: no-op
    assert lib.vq3r_decode(fake, fake, fake, 4, 16, fake, 1, None) == 4   # bf16 output unsupported
    assert lib.vq3r_decode(fake, fake, fake, 4, 16, None, 0, None) == 1
    assert lib.vq3r_rel_frobenius_error(fake, 1, fake, fake, fake, 0, 16, fake, fake, 1 << 20, None) == 2
    assert lib.vq3r_rel_frobenius_error(fake, 1, fake, fake, fake, 4, 16, fake, fake, 16, None) == 7


def _descs(specs):
    arr = (vq.GemvDesc * len(specs))()
    for i, (rows, cols, cb, x) in enumerate(specs):
        arr[i] = vq.GemvDesc(0x200000 + 0x1000 * i, 0x300000 + 0x1000 * i, cb, rows, cols, x, 0x400000 + 0x1000 * i, 0, 0, 0)
    return arr


def test_gemv_batch_and_workspace_checks(lib):
    arr = _descs([(2048, 7168, 0x10000, 0x20000)])
    assert lib.vq3r_gemv(arr, 1, 0, 1, 0x500000, 1 << 30, None) == 5
    assert lib.vq3r_gemv(arr, 1, 33, 1, 0x500000, 1 << 30, None) == 5
    assert lib.vq3r_gemv(arr, 0, 1, 1, 0x500000, 1 << 30, None) == 5
    assert lib.vq3r_gemv(arr, 1, 1, 9, 0x500000, 1 << 30, None) == 4
    assert lib.vq3r_gemv(arr, 1, 1, 1, 0x500000, 16, None) == 7
    assert lib.vq3r_gemv(arr, 1, 1, 1, None, 0, None) == 7
    assert lib.vq3r_gemv_workspace_size(arr, 1, 0) == 0


def test_vq4p_gemv_argument_checks(lib):
    arr = _descs([(2048, 7168, 0x10000, 0x20000)])
    assert lib.vq4p_gemv(None, 1, 1, 1, 0x500000, 1 << 30, None) == 1
    assert lib.vq4p_gemv(arr, 1, 1, 1, 0x500000, 1 << 30, None) == 2  # the planes layout is not accepted
    arr[0].layout = 1
    assert lib.vq4p_gemv(arr, 1, 0, 1, 0x500000, 1 << 30, None) == 5
    assert lib.vq4p_gemv(arr, 1, 33, 1, 0x500000, 1 << 30, None) == 5
    assert lib.vq4p_gemv(arr, 1, 1, 9, 0x500000, 1 << 30, None) == 4
    assert lib.vq4p_gemv(arr, 1, 1, 1, None, 0, None) == 7
    assert lib.vq4p_gemv(arr, 1, 1, 1, 0x500000, 255, None) == 7  # the 256-byte header is needed
    arr[0].plane_stride = 4 * 32768 + 16
    assert lib.vq4p_gemv(arr, 1, 1, 1, 0x500000, 1 << 30, None) == 2


def test_gemv_workspace_holds_the_partial_sums(lib):
    # a 256-byte header, then per matrix: B tokens x 3 stages x ceil(cols / 512) slabs x rows fp32 partial sums
    # (256-byte aligned)
    specs = [(2048, 7168, 0x10000, 0x20000)] * 16
    for B in (1, 4, 32):
        ws = lib.vq3r_gemv_workspace_size(_descs(specs), 16, B)
        assert ws == 256 + 16 * B * 3 * 14 * 2048 * 4
    specs = [(7168, 2048, 0x10000, 0x20000 + 0x10000 * i) for i in range(8)]
    ws = lib.vq3r_gemv_workspace_size(_descs(specs), 8, 1)
    assert ws == 256 + 8 * 3 * 4 * 7168 * 4


def test_gemv_plane_stride_checks(lib):
    arr = _descs([(2048, 7168, 0x10000, 0x20000)])
    arr[0].plane_stride = 2048 * 896 - 16  # smaller than one plane
    assert lib.vq3r_gemv(arr, 1, 1, 1, 0x500000, 1 << 30, None) == 2
    arr[0].plane_stride = 64 * 2048 * 896 + 8
    assert lib.vq3r_gemv_workspace_size(arr, 1, 1) > 0  # any stride >= one plane is accepted


def test_tiles_size_and_layout_checks(lib):
    assert lib.vq3r_tiles_size(2048, 7168) == 3 * 14 * 4 * 32768
    assert lib.vq3r_tiles_size(7168, 2048) == 3 * 4 * 14 * 32768
    assert lib.vq3r_tiles_size(5, 40) == 3 * 1 * 1 * 32768
    arr = _descs([(2048, 7168, 0x10000, 0x20000), (2048, 7168, 0x10000, 0x20000)])
    arr[1].layout = 1  # mixed layouts in one call
    assert lib.vq3r_gemv_workspace_size(arr, 2, 1) == 0
    assert lib.vq3r_gemv(arr, 2, 1, 1, 0x500000, 1 << 30, None) == 2
    arr[0].layout = 1
    arr[0].plane_stride = arr[1].plane_stride = 4 * 32768 + 16  # not a whole number of blocks
    assert lib.vq3r_gemv(arr, 2, 1, 1, 0x500000, 1 << 30, None) == 2
    arr[0].plane_stride = arr[1].plane_stride = 0
    # the tiled layout adds into y directly: the workspace is only the 256-byte header
    assert lib.vq3r_gemv_workspace_size(arr, 2, 1) == 256
    assert lib.vq3r_gemv_workspace_size(arr, 2, 32) == 256
    assert lib.vq3r_pack_tiles(None, 4, 16, 0, 0x100000, None) == 1
    assert lib.vq3r_pack_tiles(0x100000, 4, 12, 0, 0x100000, None) == 2


def _gemm_descs(specs):
    arr = (vq.GemmDesc * len(specs))()
    for i, (rows, cols, tokens) in enumerate(specs):
        arr[i] = vq.GemmDesc(0x200000 + 0x1000 * i, 0x300000 + 0x1000 * i, 0x10000, rows, cols, 0x20000,
                             0x400000 + 0x1000 * i, 0, tokens, 0)
    return arr


def test_gemm_argument_checks(lib):
    """vq3r_gemm's host checks, all before any launch (the pointers are never dereferenced)."""
    arr = _gemm_descs([(2048, 7168, 512)])
    assert lib.vq3r_gemm(None, 1, 1, None) == 1
    assert lib.vq3r_gemm(arr, 0, 1, None) == 5
    assert lib.vq3r_gemm(arr, 33, 1, None) == 5
    assert lib.vq3r_gemm(arr, 1, 0, None) == 4   # f32 x: the tensor-core product takes bf16
    assert lib.vq3r_gemm(arr, 1, 2, None) == 4
    bad = _gemm_descs([(2048, 7164, 512)])        # cols not a multiple of 8
    assert lib.vq3r_gemm(bad, 1, 1, None) == 2
    bad = _gemm_descs([(2048, 7168, -1)])
    assert lib.vq3r_gemm(bad, 1, 1, None) == 2
    bad = _gemm_descs([(2048, 7168, 512)])
    bad[0].plane_stride = 4 * 32768 + 16          # not a whole number of blocks
    assert lib.vq3r_gemm(bad, 1, 1, None) == 2
    bad[0].plane_stride = 2 * 32768               # below ceil(2048 / 512) blocks
    assert lib.vq3r_gemm(bad, 1, 1, None) == 2
    bad = _gemm_descs([(2048, 7168, 512)])
    bad[0].reserved = 1
    assert lib.vq3r_gemm(bad, 1, 1, None) == 2
    bad = _gemm_descs([(2048, 7168, 512)])
    bad[0].x = 0x20008                            # not 16-byte aligned
    assert lib.vq3r_gemm(bad, 1, 1, None) == 3
    bad = _gemm_descs([(2048, 7168, 512)])
    bad[0].y = None
    assert lib.vq3r_gemm(bad, 1, 1, None) == 1
    empty = _gemm_descs([(2048, 7168, 0), (0, 7168, 64)])  # nothing to compute: no launch, pointers unused
    empty[1].idx = None
    assert lib.vq3r_gemm(empty, 2, 1, None) == 0


def test_train_argument_checks(lib):
    fake = 0x100000
    need = lib.vq3r_train_workspace_size(1000)
    assert need >= 1000 * 32 + 1000 * 4
    assert lib.vq3r_train_workspace_size(255) == 0
    assert lib.vq3r_train(None, 1000, 5, 3, fake, None, fake, need, None) == 1
    assert lib.vq3r_train(fake, 1000, 5, 3, None, None, fake, need, None) == 1
    assert lib.vq3r_train(fake, 255, 5, 3, fake, None, fake, need, None) == 2   # fewer vectors than centroids
    assert lib.vq3r_train(fake, 1000, -1, 3, fake, None, fake, need, None) == 2
    assert lib.vq3r_train(fake, 1000, 5, 0, fake, None, fake, need, None) == 2
    assert lib.vq3r_train(fake, 1000, 5, 4, fake, None, fake, need, None) == 2
    assert lib.vq3r_train(fake, 1000, 5, 3, fake, None, fake, need - 1, None) == 7
    assert lib.vq3r_train(fake, 1000, 5, 3, fake, None, None, need, None) == 7
    assert lib.vq3r_train(fake + 4, 1000, 5, 3, fake, None, fake, need, None) == 3
    assert lib.vq3r_train(fake, 1000, 5, 3, fake, fake + 8, fake, need, None) == 3


def test_vq4p_argument_checks(lib):
    fake = 0x100000
    assert lib.vq4p_encode(None, 1, 4, 16, fake, fake, fake, None) == 1
    assert lib.vq4p_encode(fake, 1, 4, 12, fake, fake, fake, None) == 2
    assert lib.vq4p_encode(fake, 7, 4, 16, fake, fake, fake, None) == 4
    assert lib.vq4p_encode(fake, 1, 4, 16, fake + 8, fake, fake, None) == 3
    assert lib.vq4p_encode(fake, 1, 0, 16, fake, fake, fake, None) == 0
    assert lib.vq4p_decode(fake, fake, fake, 4, 16, fake, 1, None) == 4
    assert lib.vq4p_decode(fake, fake, None, 4, 16, fake, 0, None) == 1
    assert lib.vq4p_rel_frobenius_error(fake, 1, fake, fake, fake, 0, 16, fake, fake, 1 << 20, None) == 2
    assert lib.vq4p_rel_frobenius_error(fake, 1, fake, fake, fake, 4, 16, fake, fake, 16, None) == 7
    need = lib.vq4p_train_workspace_size(100)
    assert need >= 100 * 36 and lib.vq4p_train_workspace_size(63) == 0
    assert lib.vq4p_train_workspace_size(1000) == lib.vq3r_train_workspace_size(1000)
    assert lib.vq4p_train(fake, 63, 5, 4, fake, None, fake, need, None) == 2    # fewer vectors than centroids
    assert lib.vq4p_train(fake, 100, 5, 5, fake, None, fake, need, None) == 2   # at most 4 stages
    assert lib.vq4p_train(fake, 100, 5, 0, fake, None, fake, need, None) == 2
    assert lib.vq4p_train(fake, 100, 5, 4, fake, None, fake, need - 1, None) == 7
    assert lib.vq4p_train(None, 100, 5, 4, fake, None, fake, need, None) == 1


def test_outlier_argument_checks(lib):
    fake = 0x100000
    assert lib.vq3r_outliers(fake, 1, fake, fake, fake, 4, 16392, 3, fake, fake, None) == 2   # cols > 16384
    assert lib.vq3r_outliers(fake, 1, fake, fake, fake, 4, 64, 65, fake, fake, None) == 2     # k > cols
    assert lib.vq3r_outliers(fake, 1, fake, fake, fake, 4, 64, -1, fake, fake, None) == 2
    assert lib.vq3r_outliers(fake, 1, fake, fake, fake, 4, 64, 0, None, None, None) == 0      # no budget: no-op
    assert lib.vq3r_outliers(fake, 9, fake, fake, fake, 4, 64, 3, fake, fake, None) == 4
    assert lib.vq3r_outliers(fake, 1, fake, fake, fake, 4, 64, 3, None, fake, None) == 1
    assert lib.vq3r_outliers(fake, 1, fake, fake, fake, 4, 64, 3, fake + 2, fake, None) == 3
    assert lib.vq3r_decode_outliers(fake, fake, fake, None, fake, 4, 64, 3, fake, None) == 1
    need = lib.vq3r_rel_frobenius_outliers_workspace_size(4, 64, 3)
    assert need >= lib.vq3r_rel_frobenius_workspace_size(4, 64)
    assert lib.vq3r_rel_frobenius_error_outliers(fake, 1, fake, fake, fake, fake, fake, 4, 64, 3, fake, fake,
                                                 need - 8, None) == 7
    d = (vq.OutlierDesc * 1)(vq.OutlierDesc(fake, fake, 4, 64, 3, fake, fake, 1))
    assert lib.vq3r_gemv_outliers(d, 1, 1, 1, None) == 2   # reserved must be 0
    assert lib.vq3r_gemv_outliers(d, 0, 1, 1, None) == 5
    assert lib.vq3r_gemv_outliers(d, 1, 33, 1, None) == 5


def test_outlier_descriptor_and_budget_checks(lib):
    fake = 0x100000
    ok_desc = vq.OutlierDesc(fake, fake, 4, 64, 3, fake, fake, 0)
    null_y = vq.OutlierDesc(fake, fake, 4, 64, 3, fake, None, 0)
    bad_align = vq.OutlierDesc(fake + 2, fake, 4, 64, 3, fake, fake, 0)
    too_many = vq.OutlierDesc(fake, fake, 4, 64, 65, fake, fake, 0)
    empty = vq.OutlierDesc(None, None, 4, 64, 0, None, None, 0)   # k = 0: skipped, no pointers needed
    for d, want in ((null_y, 1), (bad_align, 3), (too_many, 2)):
        arr = (vq.OutlierDesc * 2)(ok_desc, d)
        assert lib.vq3r_gemv_outliers(arr, 2, 1, 1, None) == want
    assert lib.vq3r_gemv_outliers((vq.OutlierDesc * 1)(empty), 1, 1, 1, None) == 0
    assert lib.vq3r_gemv_outliers((vq.OutlierDesc * 1)(ok_desc), 1, 1, 9, None) == 4   # bad x dtype
    assert lib.vq3r_decode_outliers(fake, fake, fake, fake, fake, 4, 64, 65, fake, None) == 2
    assert lib.vq3r_decode_outliers(fake, fake, fake, fake, fake, 4, 16392, 3, fake, None) == 2
    assert lib.vq3r_rel_frobenius_error_outliers(fake, 1, fake, fake, fake, None, fake, 4, 64, 3, fake, fake,
                                                 1 << 20, None) == 1
    assert lib.vq3r_rel_frobenius_error_outliers(fake, 1, fake, fake, fake, fake, fake, 0, 64, 3, fake, fake,
                                                 1 << 20, None) == 2   # rows >= 1


def test_selftest_symbol_is_exported(lib):
    assert hasattr(lib, "vq3r_selftest_wait_timeout")
    assert "vq3r_selftest_wait_timeout" in vq.EXPORTED


def test_gemv_with_outliers_argument_checks(lib):
    arr = _descs([(2048, 7168, 0x10000, 0x20000)])
    ot = (vq.OutlierTiles * 1)()
    ot[0] = vq.OutlierTiles(0x30000, 14)
    assert lib.vq3r_gemv_with_outliers(arr, None, 1, 1, 1, 0x500000, 1 << 30, None) == 1
    assert lib.vq3r_gemv_with_outliers(arr, ot, 1, 0, 1, 0x500000, 1 << 30, None) == 5
    assert lib.vq3r_gemv_with_outliers(arr, ot, 1, 1, 9, 0x500000, 1 << 30, None) == 4
    ot[0].k = 7169  # more outliers than columns
    assert lib.vq3r_gemv_with_outliers(arr, ot, 1, 1, 1, 0x500000, 1 << 30, None) == 2
    ot[0].k = -1
    assert lib.vq3r_gemv_with_outliers(arr, ot, 1, 1, 1, 0x500000, 1 << 30, None) == 2
    ot[0].k = 14
    ot[0].otiles = 0x30004
    assert lib.vq3r_gemv_with_outliers(arr, ot, 1, 1, 1, 0x500000, 1 << 30, None) == 3
    ot[0].otiles = None
    assert lib.vq3r_gemv_with_outliers(arr, ot, 1, 1, 1, 0x500000, 1 << 30, None) == 1
    ot[0].otiles = 0x30000
    arr[0].layout = 1
    assert lib.vq3r_gemv_with_outliers(arr, ot, 1, 1, 1, None, 0, None) == 7
    assert lib.vq3r_outliers_tiles_size(2048, 14) == 4 * 14 * 2048
    assert lib.vq3r_outliers_tiles_size(513, 3) == 2 * 3 * 2048
    assert lib.vq3r_outliers_tiles_size(5, 16385) == 0
    assert lib.vq3r_pack_outliers(None, 0x100000, 4, 2, 0x200000, None) == 1
    assert lib.vq3r_pack_outliers(0x100000, 0x100000, 4, 2, 0x200008, None) == 3
    assert lib.vq3r_pack_outliers(0x100000, 0x100000, 4, -1, 0x200000, None) == 2
    assert lib.vq3r_pack_outliers(None, None, 0, 2, None, None) == 0
