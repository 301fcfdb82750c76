"""VQ4P (4 stages x 64 codewords, 6-bit indices packed in three byte planes) on the CUDA path vs the oracle,
through the C ABI.

Bars as for VQ3R: packed index planes, scales, decoded weights and trained codebooks bit-exact; the relative
Frobenius error within 1e-9 relative.  Oracle inputs come from the host generator or the oracle itself.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as wl
from vq3r_cases import GEMV_TOL, RELFRO_TOL, f32_to_bf16_bits, gemv_rel_err

pytestmark = pytest.mark.gpu

vq = pytest.importorskip("residual_vector_quantization_b200")
DEV = "cuda"


def to_dev(a, dtype):
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(DEV)
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def host_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def random_codebooks4(seed):
    """Geometrically shrinking stage codebooks [4][64][8], as a trained residual codebook set looks."""
    rng = np.random.default_rng(seed)
    return np.stack([rng.standard_normal((64, 8)) * 0.5 ** s for s in range(4)]).astype(np.float32)


def check(Wnp, dtype, cb):
    """Bit-exact VQ4P encode and decode (f32 and f16 outputs) and the error metric on one matrix."""
    W_t = to_dev(Wnp, dtype)
    cb_t = torch.from_numpy(np.ascontiguousarray(cb)).to(DEV)
    pl_t, sc_t = vq.vq4p_encode(W_t, cb_t)
    pl_o, sc_o = oracle.vq4p_encode(Wnp, dtype, cb)
    np.testing.assert_array_equal(sc_t.cpu().numpy().view(np.uint16), sc_o)
    np.testing.assert_array_equal(pl_t.cpu().numpy(), pl_o)
    Wd_o = oracle.vq4p_decode(pl_o, sc_o, cb)
    d32 = vq.vq4p_decode(pl_t, sc_t, cb_t, torch.float32).cpu().numpy()
    np.testing.assert_array_equal(d32.view(np.uint32), Wd_o.view(np.uint32))
    d16 = vq.vq4p_decode(pl_t, sc_t, cb_t, torch.float16)
    np.testing.assert_array_equal(host_bits(d16), oracle.vq4p_decode(pl_o, sc_o, cb, out="f16"))
    if Wnp.shape[0] > 0 and np.any(Wd_o != 0):
        e_gpu = float(vq.vq4p_rel_frobenius_error(W_t, pl_t, sc_t, cb_t).cpu()[0])
        e_ref = oracle.rel_frobenius(Wnp, dtype, Wd_o)
        assert abs(e_gpu - e_ref) <= RELFRO_TOL * e_ref
    return W_t, pl_t, sc_t, cb_t, pl_o, sc_o


@pytest.fixture(scope="module")
def tiny():
    cfg = wl.TINY
    W = synth.fill_rows(cfg["cols"], 0, cfg["rows"], cfg["seed"], wl.tag(0, wl.W1), synth.normal(), dtype="f32")
    vecs = oracle.normalize_rows(W, "f32", oracle.row_scales(W, "f32")).reshape(-1, 8)
    cb, tr = oracle.vq4p_train(vecs, cfg["lloyd_iters"])
    return W, vecs, cb, tr


def test_tiny_workload_bit_exact(tiny):
    W, _, cb, _ = tiny
    check(W, "f32", cb)


def test_tiny_training_bit_exact(tiny):
    """VQ4P codebooks (10 Lloyd iterations, 4 stages of 64, all 16384 tiny vectors) trained on the GPU equal the
    oracle's bit for bit; the distortion trace agrees to 1e-12."""
    _, vecs, cb, tr = tiny
    cb_t, tr_t = vq.vq4p_train(torch.from_numpy(np.ascontiguousarray(vecs)).to(DEV), wl.TINY["lloyd_iters"])
    np.testing.assert_array_equal(cb_t.cpu().numpy().view(np.uint32), cb.view(np.uint32))
    np.testing.assert_allclose(tr_t.cpu().numpy(), tr, rtol=1e-12)


@pytest.mark.parametrize("n,iters,nstages,dup", [(64, 3, 4, False), (1000, 5, 4, True), (4099, 0, 2, False),
                                                 (300, 7, 1, True)])
def test_training_small_cases_bit_exact(n, iters, nstages, dup):
    """n = 64 (every vector its own centroid), duplicates (empty clusters keep their centroid), no iterations,
    fewer stages, ragged counts."""
    rng = np.random.default_rng(n + iters + 7)
    vecs = (rng.standard_normal((n, 8)) * np.exp(rng.standard_normal((n, 1)))).astype(np.float32)
    if dup:
        vecs[:] = vecs[rng.integers(0, 40, n)]
    cb_o, tr_o = oracle.vq4p_train(vecs, iters)
    cb_t, tr_t = vq.vq4p_train(torch.from_numpy(vecs).to(DEV), iters, nstages)
    np.testing.assert_array_equal(cb_t.cpu().numpy().view(np.uint32), cb_o[:nstages].view(np.uint32))
    np.testing.assert_allclose(tr_t.cpu().numpy(), tr_o[:nstages], rtol=1e-12, atol=1e-300)


@pytest.mark.parametrize("rows,cols,dtype", [(1, 8, "f32"), (3, 40, "bf16"), (130, 800, "bf16"),
                                             (257, 1032, "f16"), (1025, 2048, "bf16"), (5, 4104, "f32")])
def test_shapes_and_dtypes(rows, cols, dtype):
    rng = np.random.default_rng(rows * 5 + cols)
    cb = random_codebooks4(rows + cols)
    Wf = (rng.standard_normal((rows, cols)) * np.exp(rng.standard_normal((rows, 1)))).astype(np.float32)
    if dtype == "f32":
        W = Wf
    elif dtype == "bf16":
        W = f32_to_bf16_bits(Wf)
    else:
        W = Wf.astype(np.float16).view(np.uint16)
    check(W, dtype, cb)


def test_ties_take_the_lowest_index():
    """Every codeword of every stage appears twice (rows j and j + 32): all decisions are exact ties between a
    pair, and the lower index must win on the GPU as in the oracle."""
    rng = np.random.default_rng(31)
    half = rng.standard_normal((4, 32, 8)).astype(np.float32) * (0.5 ** np.arange(4, dtype=np.float32))[:, None, None]
    cb = np.ascontiguousarray(np.concatenate([half, half], axis=1))
    W = rng.standard_normal((64, 512)).astype(np.float32)
    _, pl_t, _, _, pl_o, _ = check(W, "f32", cb)
    assert (oracle.vq4p_unpack(pl_o) < 32).all()


def test_planted_exact_case():
    """W = scale * C1[i1] exactly, with stage 2-4 codeword 0 the zero vector: the indices are (i1, 0, 0, 0) and
    the error is exactly 0."""
    rng = np.random.default_rng(32)
    signs = np.array([[1.0 if (j >> k) & 1 else -1.0 for k in range(8)] for j in range(256)], np.float32)
    cb = random_codebooks4(9)
    cb[0] = signs[rng.choice(256, 64, replace=False)]
    cb[1:, 0] = 0.0
    pi = rng.integers(0, 64, size=(16, 64))
    s = np.array([0.75, 3.0, 2.0 ** -6, 1.5] * 4, dtype=np.float32)
    W = (cb[0][pi].reshape(16, 512) * s[:, None]).astype(np.float32)
    W_t, pl_t, sc_t, cb_t, pl_o, _ = check(W, "f32", cb)
    idx4 = oracle.vq4p_unpack(pl_t.cpu().numpy())
    np.testing.assert_array_equal(idx4[0], pi)
    assert (idx4[1:] == 0).all()
    assert float(vq.vq4p_rel_frobenius_error(W_t, pl_t, sc_t, cb_t).cpu()[0]) == 0.0


def test_empty_matrix_is_a_noop():
    W_t = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    pl, sc = vq.vq4p_encode(W_t, torch.zeros((4, 64, 8), device=DEV))
    assert pl.shape == (3, 0, 8) and sc.shape == (0,)
    out = vq.vq4p_decode(pl, sc, torch.zeros((4, 64, 8), device=DEV))
    assert out.shape == (0, 64)


def test_expert_w2_full_matrix_bit_exact():
    """A full 7168 x 2048 bf16 expert matrix with the layer's VQ4P codebooks: every index, scale and decoded
    weight bit-exact; VQ4P's error sits above VQ3R's on the same matrix (smaller codebooks, page §5)."""
    import importlib.util
    import os
    p = os.path.join(os.path.dirname(__file__), "golden", "make_codebooks.py")
    spec = importlib.util.spec_from_file_location("make_codebooks", p)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    cb4, cb3 = mod.load("vq4p_layer"), mod.load("layer")
    rows, cols = wl.mat_shape(wl.W2)
    W = synth.fill_rows(cols, 0, rows, wl.LAYER["seed"], wl.tag(0, wl.W2), wl.expert_dist(), dtype="bf16")
    W_t, pl_t, sc_t, cb_t, pl_o, sc_o = check(W, "bf16", cb4)
    e4 = float(vq.vq4p_rel_frobenius_error(W_t, pl_t, sc_t, cb_t).cpu()[0])
    cb3_t = torch.from_numpy(np.ascontiguousarray(cb3)).to(DEV)
    idx3, sc3 = vq.vq3r_encode(W_t, cb3_t)
    e3 = float(vq.vq3r_rel_frobenius_error(W_t, idx3, sc3, cb3_t).cpu()[0])
    assert 0.1 < e3 < e4 < 0.4, (e3, e4)


def test_layer_stacked_encode_sampled_rows():
    """VQ4P encode of the 64-expert layer's stacked w1 (131072 x 7168 bf16, the benchmark's launch), bit-exact
    against the oracle on 256 sampled rows (planes and scales); decode of those rows bit-exact."""
    import importlib.util
    import os
    p = os.path.join(os.path.dirname(__file__), "golden", "make_codebooks.py")
    spec = importlib.util.spec_from_file_location("make_codebooks", p)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    cb = np.ascontiguousarray(mod.load("vq4p_layer"))
    cfg = wl.LAYER
    rows, cols = wl.mat_shape(wl.W1)
    E = cfg["experts"]
    W_t = torch.empty((E * rows, cols), dtype=torch.bfloat16, device=DEV)
    for e in range(E):
        synth.fill_rows_device(W_t[e * rows:(e + 1) * rows].data_ptr(), cols, 0, rows, cfg["seed"], wl.tag(e, wl.W1),
                               wl.expert_dist(), stream=torch.cuda.current_stream().cuda_stream)
    cb_t = torch.from_numpy(cb).to(DEV)
    pl_t, sc_t = vq.vq4p_encode(W_t, cb_t)
    d_t = vq.vq4p_decode(pl_t, sc_t, cb_t)
    rng = np.random.default_rng(44)
    sample = np.sort(rng.choice(E * rows, 256, replace=False))
    Wh = np.stack([synth.fill_row_list(cols, [r % rows], cfg["seed"], wl.tag(int(r // rows), wl.W1),
                                       wl.expert_dist())[0] for r in sample])
    sel = torch.from_numpy(sample).to(DEV)
    np.testing.assert_array_equal(host_bits(W_t[sel]), Wh)  # the two generators agree
    pl_o, sc_o = oracle.vq4p_encode(Wh, "bf16", cb)
    np.testing.assert_array_equal(sc_t[sel].cpu().numpy().view(np.uint16), sc_o)
    np.testing.assert_array_equal(pl_t[:, sel, :].cpu().numpy(), pl_o)
    np.testing.assert_array_equal(d_t[sel].cpu().numpy().view(np.uint32),
                                  oracle.vq4p_decode(pl_o, sc_o, cb).view(np.uint32))


def _gemv_case(rng, specs, B, x_dtype, seed):
    """Random VQ4P matrices (every 24-bit index word possible), binary16 scales, per-group codebooks and x;
    -> (device descriptor dicts in the tiled layout, binary64 oracle outputs)."""
    xs, mats, refs = {}, [], []
    for rows, cols, cbk, xk in specs:
        cb = random_codebooks4(seed + cbk)
        if (xk, cols) not in xs:
            xf = rng.standard_normal((B, cols)).astype(np.float32)
            xs[(xk, cols)] = (xf if x_dtype == "f32" else f32_to_bf16_bits(xf) if x_dtype == "bf16"
                              else xf.astype(np.float16).view(np.uint16))
        pl = rng.integers(0, 256, size=(3, rows, cols // 8), dtype=np.uint8)
        sc = np.float16(np.exp(rng.standard_normal(rows) * 0.5)).view(np.uint16)
        refs.append(oracle.vq4p_gemv(pl, sc, cb, xs[(xk, cols)], x_dtype))
        pl_t = torch.from_numpy(pl).to(DEV)
        mats.append(dict(idx=vq.vq3r_pack_tiles(pl_t), layout="tiles", cols=cols,
                         scales=torch.from_numpy(sc.view(np.int16)).to(DEV),
                         codebooks=torch.from_numpy(np.ascontiguousarray(cb)).to(DEV),
                         x=(xk, cols), y=torch.full((B, rows), float("nan"), device=DEV)))
    xdev = {k: to_dev(v, x_dtype) for k, v in xs.items()}
    for m in mats:
        m["x"] = xdev[m["x"]]
    return mats, refs


@pytest.mark.parametrize("B,x_dtype", [(1, "bf16"), (1, "f32"), (1, "f16"), (2, "bf16"), (3, "f16"), (8, "bf16"),
                                       (17, "f32"), (32, "bf16")])
def test_gemv_grouped_matches_oracle(B, x_dtype):
    """vq4p_gemv over mixed matrices (ragged rows and slabs, two codebook sets, two x per width) against the
    oracle's binary64 product of the decoded weights; one token (one table per slab), token pairs with an odd
    count (a pair with one token), every x dtype."""
    rng = np.random.default_rng(900 + 10 * B + len(x_dtype))
    specs = [(300, 1032, 0, 0), (129, 1032, 0, 0), (64, 200, 1, 1), (513, 2048, 1, 0), (1, 8, 0, 2)]
    mats, refs = _gemv_case(rng, specs, B, x_dtype, 70)
    vq.vq4p_gemv(mats, B)
    for m, ref in zip(mats, refs):
        y = m["y"].cpu().numpy()
        assert np.isfinite(y).all()  # every output written
        assert gemv_rel_err(y, ref) <= GEMV_TOL
    assert vq.vq3r_device_error() == 0


@pytest.mark.parametrize("B", [1, 4])
def test_gemv_moe_decode_step_sampled_rows(B):
    """The 8-expert MoE decode step's shapes (w1, w3: 2048 x 7168; w2: 7168 x 2048; one call, 24 matrices) with
    random VQ4P indices: 48 sampled rows of every matrix against the oracle."""
    rng = np.random.default_rng(950 + B)
    cb = random_codebooks4(5)
    cb_t = torch.from_numpy(np.ascontiguousarray(cb)).to(DEV)
    x1 = f32_to_bf16_bits(rng.standard_normal((B, 7168)).astype(np.float32))
    x2 = f32_to_bf16_bits(rng.standard_normal((B, 2048)).astype(np.float32))
    x1_t, x2_t = to_dev(x1, "bf16"), to_dev(x2, "bf16")
    mats, hosts = [], []
    for e in range(8):
        for rows, cols, x_t, x in ((2048, 7168, x1_t, x1), (2048, 7168, x1_t, x1), (7168, 2048, x2_t, x2)):
            pl_t = torch.randint(0, 256, (3, rows, cols // 8), dtype=torch.uint8, device=DEV)
            sc_t = torch.from_numpy(np.float16(np.exp(rng.standard_normal(rows) * 0.5)).view(np.int16)).to(DEV)
            mats.append(dict(idx=vq.vq3r_pack_tiles(pl_t), layout="tiles", cols=cols, scales=sc_t, codebooks=cb_t,
                             x=x_t, y=torch.empty((B, rows), device=DEV)))
            hosts.append((pl_t, sc_t, x))
    vq.vq4p_gemv(mats, B)
    torch.cuda.synchronize()
    for m, (pl_t, sc_t, x) in zip(mats, hosts):
        rows = pl_t.shape[1]
        sample = np.sort(rng.choice(rows, 48, replace=False))
        sel = torch.from_numpy(sample).to(DEV)
        pl = pl_t[:, sel, :].cpu().numpy()
        sc = sc_t[sel].cpu().numpy().view(np.uint16)
        ref = oracle.vq4p_gemv(pl, sc, cb, x, "bf16")
        y = m["y"][:, sel].cpu().numpy()
        # the tolerance's rms term comes from the sampled rows
        assert gemv_rel_err(y, ref) <= GEMV_TOL
    assert vq.vq3r_device_error() == 0


def test_gemv_rejects_the_planes_layout():
    pl = torch.zeros((3, 4, 2), dtype=torch.uint8, device=DEV)
    m = dict(idx=pl, scales=torch.zeros(4, dtype=torch.int16, device=DEV), codebooks=torch.zeros((4, 64, 8), device=DEV),
             x=torch.zeros((1, 16), dtype=torch.bfloat16, device=DEV), y=torch.empty((1, 4), device=DEV))
    with pytest.raises(vq.VQ3RError):
        vq.vq4p_gemv([m], 1)
