"""Outlier-aware variant (sparse FP16 residual over VQ3R, page "XFP", 权重分解) on the CUDA path vs the oracle,
through the C ABI.

Bars: outlier columns and values bit-exact (integer selection work), the decode with outliers bit-exact, the
relative Frobenius error within 1e-9 relative, the GEMV with outliers within 2e-3 (rms floor).  Oracle inputs
come from the host generator or the oracle itself.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as wl
from vq3r_cases import GEMV_TOL, RELFRO_TOL, f32_to_bf16_bits, gemv_rel_err, random_codebooks

pytestmark = pytest.mark.gpu

vq = pytest.importorskip("residual_vector_quantization_b200")
DEV = "cuda"


def to_dev(a, dtype):
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(DEV)
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def u16(t):
    return t.cpu().numpy().view(np.uint16)


def check(W, dtype, cb, ks, B=2, seed=0):
    """Encode on the GPU (bit-exact with the oracle, checked elsewhere), then for each budget k: outliers, decode
    with outliers, error with outliers and the GEMV with outliers against the oracle."""
    W_t = to_dev(W, dtype)
    cb_t = torch.from_numpy(np.ascontiguousarray(cb)).to(DEV)
    idx_t, sc_t = vq.vq3r_encode(W_t, cb_t)
    idx_o, sc_o = oracle.encode(W, dtype, cb)
    np.testing.assert_array_equal(idx_t.cpu().numpy(), idx_o)
    What = oracle.decode(idx_o, sc_o, cb)
    rows, cols = What.shape
    rng = np.random.default_rng(seed)
    xb = f32_to_bf16_bits(rng.standard_normal((B, cols)).astype(np.float32))
    results = {}
    for k in ks:
        oc_t, ov_t = vq.vq3r_outliers(W_t, idx_t, sc_t, cb_t, k)
        oc_o, ov_o = oracle.outliers_select(W, dtype, What, k)
        np.testing.assert_array_equal(u16(oc_t), oc_o)
        np.testing.assert_array_equal(u16(ov_t), ov_o)
        W2 = oracle.outliers_apply(What, oc_o, ov_o)
        d = vq.vq3r_decode_outliers(idx_t, sc_t, cb_t, oc_t, ov_t).cpu().numpy()
        np.testing.assert_array_equal(d.view(np.uint32), W2.view(np.uint32))
        e_gpu = float(vq.vq3r_rel_frobenius_error_outliers(W_t, idx_t, sc_t, cb_t, oc_t, ov_t).cpu()[0])
        e_ref = oracle.rel_frobenius(W, dtype, W2)
        assert abs(e_gpu - e_ref) <= RELFRO_TOL * e_ref + 1e-300, (k, e_gpu, e_ref)
        y = torch.empty((B, rows), dtype=torch.float32, device=DEV)
        x_t = to_dev(xb, "bf16")
        vq.vq3r_gemv([dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=x_t, y=y)], B)
        vq.vq3r_gemv_outliers([dict(ocols=oc_t, ovals=ov_t, cols=cols, x=x_t, y=y)], B)
        assert gemv_rel_err(y.cpu().numpy(), oracle.gemv(W2, xb, "bf16")) <= GEMV_TOL
        results[k] = e_ref
    return results


def test_tiny_workload_budgets():
    cfg = wl.TINY
    W = synth.fill_rows(cfg["cols"], 0, cfg["rows"], cfg["seed"], wl.tag(0, wl.W1), synth.normal(), dtype="f32")
    cb, _ = oracle.lloyd_train(oracle.normalize_rows(W, "f32", oracle.row_scales(W, "f32")), cfg["lloyd_iters"])
    errs = check(W, "f32", cb, (1, 5, 64, 512))
    assert errs[512] < errs[64] < errs[5] < errs[1]


def test_exact_ties_go_to_lower_columns():
    """Zero codebooks decode to 0, so e = w; weights drawn from {-2, -1, 1, 2} tie in blocks, and budgets that
    end inside a block must take its lowest columns."""
    rng = np.random.default_rng(11)
    W = rng.choice([-2.0, -1.0, 1.0, 2.0], size=(40, 1024)).astype(np.float32)
    cb = np.zeros((3, 256, 8), dtype=np.float32)
    n2 = (np.abs(W) == 2).sum(axis=1)
    check(W, "f32", cb, (1, 100, int(n2.min()), int(n2.max()) + 3, 1024))


@pytest.mark.parametrize("rows,cols,dtype,ks", [(3, 40, "bf16", (1, 40)), (130, 800, "f16", (7, 33)),
                                                (257, 1032, "f32", (2, 129)), (5, 16384, "bf16", (1, 37, 700))])
def test_shapes_dtypes_and_the_column_limit(rows, cols, dtype, ks):
    rng = np.random.default_rng(rows + cols)
    Wf = (rng.standard_normal((rows, cols)) * np.exp(rng.standard_normal((rows, 1)))).astype(np.float32)
    W = Wf if dtype == "f32" else (f32_to_bf16_bits(Wf) if dtype == "bf16" else Wf.astype(np.float16).view(np.uint16))
    check(W, dtype, random_codebooks(rows), ks)


def test_sweep_distribution_outliers_reduce_the_error():
    """Rows of the 256-expert sweep distribution (Student-t(3), 0.1% of weights at +-20 sigma): with a budget of
    cols/512 the outliers are bit-exact and cut the relative error well below plain VQ3R's."""
    import importlib.util
    import os
    p = os.path.join(os.path.dirname(__file__), "golden", "make_codebooks.py")
    spec = importlib.util.spec_from_file_location("make_codebooks", p)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    cb = mod.load("sweep")
    rows, cols = wl.mat_shape(wl.W1)
    W = synth.fill_rows(cols, 0, 256, wl.SWEEP["seed"], wl.tag(3, wl.W1), wl.sweep_dist(), dtype="bf16")
    errs = check(W, "bf16", cb, (0, cols // 512, cols // 128))
    assert errs[cols // 512] < 0.9 * errs[0], errs


def test_grouped_sparse_add_over_expert_row_ranges():
    """One vq3r_gemv_outliers call over row ranges of two stacked matrices (as for experts), B = 3."""
    rng = np.random.default_rng(12)
    cb = random_codebooks(12)
    W = rng.standard_normal((1024, 256)).astype(np.float32)
    W_t = to_dev(W, "f32")
    cb_t = torch.from_numpy(cb).to(DEV)
    idx_t, sc_t = vq.vq3r_encode(W_t, cb_t)
    oc_t, ov_t = vq.vq3r_outliers(W_t, idx_t, sc_t, cb_t, 9)
    What = oracle.decode(*oracle.encode(W, "f32", cb), cb)
    W2 = oracle.outliers_apply(What, *oracle.outliers_select(W, "f32", What, 9))
    B = 3
    x = rng.standard_normal((2, B, 256)).astype(np.float32)
    mats, outs = [], []
    for j, (r0, n) in enumerate(((0, 512), (512, 512))):
        y = torch.empty((B, n), dtype=torch.float32, device=DEV)
        xt = to_dev(x[j], "f32")
        vq.vq3r_gemv([dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=xt, y=y, row0=r0, rows=n)], B)
        mats.append(dict(ocols=oc_t, ovals=ov_t, cols=256, x=xt, y=y, row0=r0, rows=n))
        outs.append((r0, n, y))
    vq.vq3r_gemv_outliers(mats, B)
    for j, (r0, n, y) in enumerate(outs):
        ref = oracle.gemv(W2[r0:r0 + n], x[j], "f32")
        assert gemv_rel_err(y.cpu().numpy(), ref) <= GEMV_TOL


def test_layer_stacked_outliers_sampled_rows():
    """Outliers of the 64-expert layer's stacked w1 (131072 x 7168 bf16, budget cols/512 = 14 per row, the
    benchmark's launch), bit-exact against the oracle on 256 sampled rows; the error with outliers of the whole
    matrix agrees with the decode-with-outliers kernel's output summed in binary64."""
    import importlib.util
    import os
    p = os.path.join(os.path.dirname(__file__), "golden", "make_codebooks.py")
    spec = importlib.util.spec_from_file_location("make_codebooks", p)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    cb = np.ascontiguousarray(mod.load("layer"))
    cfg = wl.LAYER
    rows, cols = wl.mat_shape(wl.W1)
    E, k = cfg["experts"], cols // 512
    W_t = torch.empty((E * rows, cols), dtype=torch.bfloat16, device=DEV)
    for e in range(E):
        synth.fill_rows_device(W_t[e * rows:(e + 1) * rows].data_ptr(), cols, 0, rows, cfg["seed"], wl.tag(e, wl.W1),
                               wl.expert_dist(), stream=torch.cuda.current_stream().cuda_stream)
    cb_t = torch.from_numpy(cb).to(DEV)
    idx_t, sc_t = vq.vq3r_encode(W_t, cb_t)
    oc_t, ov_t = vq.vq3r_outliers(W_t, idx_t, sc_t, cb_t, k)
    rng = np.random.default_rng(45)
    sample = np.sort(rng.choice(E * rows, 256, replace=False))
    Wh = np.stack([synth.fill_row_list(cols, [r % rows], cfg["seed"], wl.tag(int(r // rows), wl.W1),
                                       wl.expert_dist())[0] for r in sample])
    idx_o, sc_o = oracle.encode(Wh, "bf16", cb)
    sel = torch.from_numpy(sample).to(DEV)
    np.testing.assert_array_equal(idx_t[:, sel, :].cpu().numpy(), idx_o)
    oc_o, ov_o = oracle.outliers_select(Wh, "bf16", oracle.decode(idx_o, sc_o, cb), k)
    np.testing.assert_array_equal(u16(oc_t[sel]), oc_o)
    np.testing.assert_array_equal(u16(ov_t[sel]), ov_o)
    d = vq.vq3r_decode_outliers(idx_t, sc_t, cb_t, oc_t, ov_t)
    w = W_t.double()
    e2 = float(torch.sqrt(((w - d.double()) ** 2).sum() / (w ** 2).sum()))
    del d
    e = float(vq.vq3r_rel_frobenius_error_outliers(W_t, idx_t, sc_t, cb_t, oc_t, ov_t).cpu()[0])
    assert abs(e - e2) <= 1e-9 * e2


def _random_outliers(rng, rows, cols, k):
    """k distinct ascending columns per row and binary16 values (as vq3r_outliers lays them out)."""
    oc = np.zeros((rows, k), dtype=np.uint16)
    for i in range(rows):
        oc[i] = np.sort(rng.choice(cols, k, replace=False))
    ov = np.float16(rng.standard_normal((rows, k)) * 0.3).view(np.uint16)
    return oc, ov


@pytest.mark.parametrize("B,x_dtype,layout,per512", [(1, "bf16", "tiles", 3), (2, "bf16", "tiles", 3),
                                                     (5, "f32", "tiles", 1), (1, "f16", "tiles", 2),
                                                     (1, "bf16", "tiles", 4), (12, "bf16", "tiles", 3),
                                                     (3, "bf16", "planes", 3)])
def test_gemv_with_outliers_one_call(B, x_dtype, layout, per512):
    """vq3r_gemv_with_outliers over mixed matrices: several 512-row tiles with a ragged last one, a matrix
    without outliers between two with, a ragged last slab, two inputs x, up to per512 outliers per 512 columns.
    The lookup-table kernel starts y at the outliers' sums (tiles, B <= 10 or non-bf16 x); bf16 B = 12 and the
    plane layout take the two-launch path.  Against the oracle's binary64 product of the decoded weights with the
    outliers applied."""
    rng = np.random.default_rng(500 + B + per512)
    cb = random_codebooks(41)
    cb_t = torch.from_numpy(cb).to(DEV)
    p = per512
    specs = [(1030, 1024, 0, 2 * p), (300, 1024, 0, 0), (513, 2048, 1, 4 * p), (64, 1032, 1, 3 * p - 2)]
    xs = {}
    mats, refs = [], []
    for rows, cols, xk, k in specs:
        if (xk, cols) not in xs:
            xf = rng.standard_normal((B, cols)).astype(np.float32)
            xs[(xk, cols)] = (xf if x_dtype == "f32" else f32_to_bf16_bits(xf) if x_dtype == "bf16"
                              else xf.astype(np.float16).view(np.uint16))
        idx = rng.integers(0, 256, size=(3, rows, cols // 8), dtype=np.uint8)
        sc = np.float16(np.exp(rng.standard_normal(rows) * 0.5)).view(np.uint16)
        What = oracle.decode(idx, sc, cb)
        m = dict(idx=torch.from_numpy(idx).to(DEV), scales=torch.from_numpy(sc.view(np.int16)).to(DEV),
                 codebooks=cb_t, x=(xk, cols), y=torch.full((B, rows), float("nan"), device=DEV))
        if k:
            oc, ov = _random_outliers(rng, rows, cols, k)
            What = oracle.outliers_apply(What, oc, ov)
            m["otiles"] = vq.vq3r_pack_outliers(torch.from_numpy(oc.view(np.int16)).to(DEV),
                                                torch.from_numpy(ov.view(np.int16)).to(DEV))
        if layout == "tiles":
            m.update(idx=vq.vq3r_pack_tiles(m["idx"]), layout="tiles", cols=cols)
        refs.append(oracle.gemv(What, xs[(xk, cols)], x_dtype))
        mats.append(m)
    xdev = {kk: to_dev(v, x_dtype) for kk, v in xs.items()}
    for m in mats:
        m["x"] = xdev[m["x"]]
    vq.vq3r_gemv_with_outliers(mats, B)
    for m, ref in zip(mats, refs):
        y = m["y"].cpu().numpy()
        assert np.isfinite(y).all()
        assert gemv_rel_err(y, ref) <= GEMV_TOL
    assert vq.vq3r_device_error() == 0


def test_gemv_with_outliers_moe_decode_step_sampled_rows():
    """The 8-expert MoE decode step (24 matrices, B = 1, cols/512 outliers per row) in one call against the
    oracle on 32 sampled rows of every matrix.  Outlier columns: one per 512-column stretch of the row."""
    rng = np.random.default_rng(77)
    cb = random_codebooks(43)
    cb_t = torch.from_numpy(cb).to(DEV)
    B = 1
    x1 = f32_to_bf16_bits(rng.standard_normal((B, 7168)).astype(np.float32))
    x1_t = to_dev(x1, "bf16")
    mats, hosts = [], []
    for e in range(8):
        x2 = f32_to_bf16_bits(rng.standard_normal((B, 2048)).astype(np.float32))
        x2_t = to_dev(x2, "bf16")
        for rows, cols, x_t, x in ((2048, 7168, x1_t, x1), (2048, 7168, x1_t, x1), (7168, 2048, x2_t, x2)):
            idx_t = torch.randint(0, 256, (3, rows, cols // 8), dtype=torch.uint8, device=DEV)
            sc = np.float16(np.exp(rng.standard_normal(rows) * 0.5)).view(np.uint16)
            k = cols // 512
            oc = (rng.integers(0, 512, size=(rows, k)) + 512 * np.arange(k)).astype(np.uint16)
            ov = np.float16(rng.standard_normal((rows, k))).view(np.uint16)
            m = dict(idx=vq.vq3r_pack_tiles(idx_t), layout="tiles", cols=cols,
                     scales=torch.from_numpy(sc.view(np.int16)).to(DEV), codebooks=cb_t, x=x_t,
                     y=torch.empty((B, rows), device=DEV),
                     otiles=vq.vq3r_pack_outliers(torch.from_numpy(oc.view(np.int16)).to(DEV),
                                                  torch.from_numpy(ov.view(np.int16)).to(DEV)))
            mats.append(m)
            hosts.append((idx_t, sc, oc, ov, x))
    vq.vq3r_gemv_with_outliers(mats, B)
    torch.cuda.synchronize()
    for m, (idx_t, sc, oc, ov, x) in zip(mats, hosts):
        rows = sc.shape[0]
        sample = np.sort(rng.choice(rows, 32, replace=False))
        idx = idx_t[:, torch.from_numpy(sample).to(DEV), :].cpu().numpy()
        What = oracle.outliers_apply(oracle.decode(idx, sc[sample], cb), oc[sample], ov[sample])
        ref = oracle.gemv(What, x, "bf16")
        assert gemv_rel_err(m["y"][:, torch.from_numpy(sample).to(DEV)].cpu().numpy(), ref) <= GEMV_TOL
    assert vq.vq3r_device_error() == 0


@pytest.mark.parametrize("rows,k", [(1, 1), (511, 3), (512, 14), (1300, 5)])
def test_pack_outliers_layout(rows, k):
    """The outlier-tile layout written out from its definition: word (t, q, r) = ocols[512 t + r][q] |
    ovals[512 t + r][q] << 16, all ones past the last row."""
    rng = np.random.default_rng(rows + k)
    oc = rng.integers(0, 16384, size=(rows, k)).astype(np.uint16)
    ov = rng.integers(0, 65536, size=(rows, k)).astype(np.uint16)
    got = vq.vq3r_pack_outliers(torch.from_numpy(oc.view(np.int16)).to(DEV),
                                torch.from_numpy(ov.view(np.int16)).to(DEV)).cpu().numpy().view(np.uint32)
    n_tiles = (rows + 511) // 512
    want = np.full((n_tiles, k, 512), 0xFFFFFFFF, dtype=np.uint32)
    for i in range(rows):
        for q in range(k):
            want[i // 512, q, i % 512] = int(oc[i, q]) | (int(ov[i, q]) << 16)
    np.testing.assert_array_equal(got, want)
    assert vq.lib().vq3r_outliers_tiles_size(rows, k) == got.nbytes
