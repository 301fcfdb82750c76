"""CUDA path vs the CPU oracle, through the C ABI (residual_vector_quantization_b200).

Bars: indices, scales and decoded weights bit-exact; relative Frobenius
error within 1e-9 relative; GEMV within 2e-3 max relative error (rms(y)
floor) against the binary64 oracle GEMV.  Every oracle input comes from the
host generator (synth) or from the oracle itself, never from the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as wl
from vq3r_cases import (GEMM_TOL, GEMV_TOL, RELFRO_TOL, energy8_vectors, f32_to_bf16_bits, gemv_rel_err, random_codebooks,
                        sign_pattern_codebooks)

pytestmark = pytest.mark.gpu

vq = pytest.importorskip("residual_vector_quantization_b200")
DEV = "cuda"


def to_dev(a, dtype):
    """numpy host array -> device tensor: f32 as float32, bf16/f16 from uint16 bit patterns."""
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(DEV)
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def host_bits(t):
    """device bf16/f16 tensor -> numpy uint16 bit patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def gpu_encode(W_t, cb):
    idx, sc = vq.vq3r_encode(W_t, torch.from_numpy(cb).to(DEV))
    torch.cuda.synchronize()
    return idx, sc


def check_encode_decode(Wnp, dtype, cb):
    """Full bit-exact parity of encode and decode on one matrix; returns device tensors."""
    W_t = to_dev(Wnp, dtype)
    idx_t, sc_t = gpu_encode(W_t, cb)
    idx_o, sc_o = oracle.encode(Wnp, dtype, cb)
    np.testing.assert_array_equal(sc_t.cpu().numpy().view(np.uint16), sc_o)
    np.testing.assert_array_equal(idx_t.cpu().numpy(), idx_o)
    cb_t = torch.from_numpy(cb).to(DEV)
    d32 = vq.vq3r_decode(idx_t, sc_t, cb_t, torch.float32).cpu().numpy()
    np.testing.assert_array_equal(d32.view(np.uint32), oracle.decode(idx_o, sc_o, cb).view(np.uint32))
    d16 = vq.vq3r_decode(idx_t, sc_t, cb_t, torch.float16)
    np.testing.assert_array_equal(host_bits(d16), oracle.decode(idx_o, sc_o, cb, out="f16"))
    return W_t, idx_t, sc_t, cb_t, idx_o, sc_o


def as_layout(mats, layout):
    """GEMV descriptors in the requested index layout (tiles: packed with vq3r_pack_tiles)."""
    if layout == "planes":
        return mats
    out = []
    for m in mats:
        idx = m["idx"]
        out.append(dict(m, idx=vq.vq3r_pack_tiles(idx), layout="tiles", cols=idx.shape[2] * 8))
    return out


def tiles_reference(idx):
    """The tiled layout of index planes [3][rows][V], written out from its definition."""
    _, rows, V = idx.shape
    n_slabs, n_tiles = -(-V // 64), -(-rows // 512)
    out = np.zeros((3, n_slabs, n_tiles, 512, 64), dtype=np.uint8)
    for s in range(3):
        for slab in range(n_slabs):
            for t in range(n_tiles):
                blk = np.zeros((512, 64), np.uint8)
                src = idx[s, t * 512:(t + 1) * 512, slab * 64:(slab + 1) * 64]
                blk[:src.shape[0], :src.shape[1]] = src
                swap = (np.arange(512) >> 2) & 1
                for c in range(64):
                    dst = 16 * (c >> 4) + 8 * (((c >> 3) & 1) ^ swap) + (c & 7)
                    out[s, slab, t, np.arange(512), dst] = blk[:, c]
    return out.reshape(-1)


# ------------------------------------------------------------------ tiny workload, end to end

@pytest.fixture(scope="module")
def tiny():
    cfg = wl.TINY
    W = synth.fill_rows(cfg["cols"], 0, cfg["rows"], cfg["seed"], wl.tag(0, wl.W1), synth.normal(), dtype="f32")
    sc = oracle.row_scales(W, "f32")
    cb, _ = oracle.lloyd_train(oracle.normalize_rows(W, "f32", sc), cfg["lloyd_iters"])
    return W, cb


def test_tiny_encode_decode_bit_exact(tiny):
    W, cb = tiny
    check_encode_decode(W, "f32", cb)


def test_tiny_rel_frobenius(tiny):
    W, cb = tiny
    W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(W, "f32", cb)
    e_gpu = float(vq.vq3r_rel_frobenius_error(W_t, idx_t, sc_t, cb_t).cpu()[0])
    e_ref = oracle.rel_frobenius(W, "f32", oracle.decode(idx_o, sc_o, cb))
    assert abs(e_gpu - e_ref) <= RELFRO_TOL * e_ref


@pytest.mark.parametrize("layout", ["planes", "tiles"])
@pytest.mark.parametrize("B", [1, 4, 8, 32])
def test_tiny_gemv(tiny, B, layout):
    W, cb = tiny
    W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(W, "f32", cb)
    x = synth.fill_rows(W.shape[1], 0, B, wl.TINY_SEED, wl.tag(0, wl.X_GATEUP), synth.normal(), dtype="f32")
    y_t = torch.empty((B, W.shape[0]), dtype=torch.float32, device=DEV)
    vq.vq3r_gemv(as_layout([dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=to_dev(x, "f32"), y=y_t)], layout), B)
    y_ref = oracle.gemv(oracle.decode(idx_o, sc_o, cb), x, "f32")
    assert gemv_rel_err(y_t.cpu().numpy(), y_ref) <= GEMV_TOL


# ------------------------------------------------------------------ shapes, dtypes, ragged tails

@pytest.mark.parametrize("rows,cols,dtype", [(1, 8, "f32"), (3, 40, "bf16"), (130, 800, "bf16"), (257, 1032, "f16"),
                                             (64, 7168, "bf16"), (1025, 2048, "bf16"), (5, 4104, "f32")])
def test_shapes_and_dtypes(rows, cols, dtype):
    rng = np.random.default_rng(rows * 7 + cols)
    cb = random_codebooks(rows + cols)
    Wf = (rng.standard_normal((rows, cols)) * np.exp(rng.standard_normal((rows, 1)))).astype(np.float32)
    if dtype == "f32":
        W = Wf
    elif dtype == "bf16":
        W = f32_to_bf16_bits(Wf)
    else:
        W = Wf.astype(np.float16).view(np.uint16)
    W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(W, dtype, cb)
    for B in (1, 3):
        x = rng.standard_normal((B, cols)).astype(np.float32)
        xb = f32_to_bf16_bits(x)
        y_ref = oracle.gemv(oracle.decode(idx_o, sc_o, cb), xb, "bf16")
        for layout in ("planes", "tiles"):
            y_t = torch.empty((B, rows), dtype=torch.float32, device=DEV)
            vq.vq3r_gemv(as_layout([dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=to_dev(xb, "bf16"), y=y_t)],
                                   layout), B)
            assert gemv_rel_err(y_t.cpu().numpy(), y_ref) <= GEMV_TOL, layout
    e_gpu = float(vq.vq3r_rel_frobenius_error(W_t, idx_t, sc_t, cb_t).cpu()[0])
    e_ref = oracle.rel_frobenius(W, dtype, oracle.decode(idx_o, sc_o, cb))
    assert abs(e_gpu - e_ref) <= RELFRO_TOL * e_ref


def test_ties_take_the_lowest_index():
    """Sign-pattern codebooks and residual components that are exactly 0: every
    tie is exact, and the lowest index must win on the GPU as in the oracle."""
    rng = np.random.default_rng(21)
    cb = sign_pattern_codebooks()
    V, rows = 64, 96
    W = energy8_vectors(rng, rows * V).reshape(rows, V * 8)
    W[:, ::3] = 0.0  # more ties (rows keep a nonzero RMS)
    check_encode_decode(W, "f32", cb)
    perm = rng.permutation(256)
    check_encode_decode(W, "f32", np.ascontiguousarray(cb[:, perm, :]))


def test_encode_tie_that_a_fused_multiply_add_would_break():
    """A vector whose two best stage-1 codewords (37 and 61) tie exactly under the distance definition (every
    binary32 operation rounded, k ascending) while a fused d + e * e accumulation makes 61 strictly closer.
    The lowest index must win, as in the oracle.  (Found as a mismatch in a seeded 513 x 2048 matrix: the
    paired add and multiply of the encoder had been contracted into fused multiply-adds.)"""
    rng = np.random.default_rng(513 * 7 + 2048 + 300)
    cb = random_codebooks(513 + 2048)
    W = f32_to_bf16_bits(rng.standard_normal((513, 2048)).astype(np.float32))[500:501]
    # the tie, checked on the host: equal with per-operation rounding, 61 first with fused accumulation
    s = np.float32(oracle.fp16_to_double(int(oracle.row_scales(W, "bf16")[0])))
    r = ((W[0, 160:168].astype(np.uint32) << 16).view(np.float32) / s).astype(np.float32)

    def dist(c, fused):
        acc = np.float32(0.0)
        for k in range(8):
            e = np.float32(r[k] - c[k])
            acc = np.float32(np.float64(e) * np.float64(e) + np.float64(acc)) if fused else np.float32(acc + np.float32(e * e))
        return acc
    assert dist(cb[0, 37], False) == dist(cb[0, 61], False)
    assert dist(cb[0, 61], True) < dist(cb[0, 37], True)
    W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(W, "bf16", cb)
    assert idx_o[0, 0, 20] == 37


def test_encode_near_twin_codewords():
    """Every codeword of every stage has a twin (index + 128) perturbed in one coordinate by 0 ulps (an exact tie)
    up to 2^-12 relative, so the two best screening values of most vectors lie on either side of the encoder's
    margin: the winners it accepts without the definition's scan and the ones it re-scans must both equal the
    oracle's indices."""
    rng = np.random.default_rng(41)
    cb = random_codebooks(41)
    for s in range(3):
        for j in range(128):
            k = j % 8
            c = cb[s, j].copy()
            if j % 4 == 0:
                pass                                             # exact duplicate
            elif j % 4 == 1:
                c[k] = np.nextafter(c[k], np.float32(np.inf))    # 1 ulp
            else:
                c[k] = np.float32(c[k] * (1 + 2.0 ** -rng.integers(12, 24)))
            cb[s, 128 + j] = c
    W = rng.standard_normal((192, 1024)).astype(np.float32)
    # every third row is made of stage-1 codewords (close to a codeword and its twin after the row's scaling)
    W[::3, :] = cb[0][rng.integers(0, 256, size=(64, 128))].reshape(64, 1024)
    check_encode_decode(W, "f32", cb)
    check_encode_decode(f32_to_bf16_bits(W), "bf16", cb)


def test_scale_limits_zero_rows_and_subnormals():
    rng = np.random.default_rng(22)
    cb = random_codebooks(5)
    W = rng.standard_normal((8, 512)).astype(np.float32)
    W[0] = 0.0                       # zero row -> scale 0, r = 0
    W[1] *= 1e6                      # RMS above 65504 -> saturated scale
    W[2] *= 2.0 ** -20               # binary16 subnormal scale
    W[3] *= 2.0 ** -30               # scale underflows to 0
    W[4] = 1 + 2.0 ** -11            # RMS on a binary16 midpoint (ties to even)
    W[5] = 1 + 3 * 2.0 ** -11
    check_encode_decode(W, "f32", cb)


def test_planted_exact_case():
    rng = np.random.default_rng(23)
    cb = sign_pattern_codebooks()
    cb[0] = cb[0][rng.permutation(256)]
    cb[1] = rng.standard_normal((256, 8)).astype(np.float32) * 0.3
    cb[2] = rng.standard_normal((256, 8)).astype(np.float32) * 0.1
    cb[1, 0] = 0.0
    cb[2, 0] = 0.0
    pi = rng.integers(0, 256, size=(16, 64))
    s = np.array([0.75, 3.0, 2.0 ** -6, 1.5] * 4, dtype=np.float32)
    W = (cb[0][pi].reshape(16, 512) * s[:, None]).astype(np.float32)
    W_t, idx_t, sc_t, cb_t, idx_o, _ = check_encode_decode(W, "f32", cb)
    np.testing.assert_array_equal(idx_t.cpu().numpy()[0], pi)
    assert float(vq.vq3r_rel_frobenius_error(W_t, idx_t, sc_t, cb_t).cpu()[0]) == 0.0


def test_empty_matrix_is_a_noop():
    W_t = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    idx, sc = vq.vq3r_encode(W_t, torch.zeros((3, 256, 8), device=DEV))
    assert idx.shape == (3, 0, 8) and sc.shape == (0,)


@pytest.mark.parametrize("rows,cols", [(3, 40), (130, 800), (1025, 2048), (600, 7168)])
def test_pack_tiles_layout(rows, cols):
    rng = np.random.default_rng(rows + cols)
    idx = rng.integers(0, 256, size=(3, rows, cols // 8), dtype=np.uint8)
    packed = vq.vq3r_pack_tiles(torch.from_numpy(idx).to(DEV)).cpu().numpy()
    assert packed.size == vq.vq3r_tiles_size(rows, cols)
    np.testing.assert_array_equal(packed, tiles_reference(idx))


@pytest.mark.parametrize("layout", ["planes", "tiles"])
def test_grouped_gemv_mixed_matrices(layout):
    """One call over matrices of different shapes, codebooks and inputs."""
    rng = np.random.default_rng(24)
    specs = [(300, 1024, 0, 0), (129, 1024, 0, 0), (64, 512, 1, 1), (200, 1024, 2, 0), (33, 1024, 0, 2)]
    B = 4
    xs = {}
    mats, refs = [], []
    for rows, cols, cbk, xk in specs:
        cb = random_codebooks(100 + cbk)
        if (xk, cols) not in xs:
            xs[(xk, cols)] = f32_to_bf16_bits(rng.standard_normal((B, cols)).astype(np.float32))
        x = xs[(xk, cols)]
        W = f32_to_bf16_bits(rng.standard_normal((rows, cols)).astype(np.float32))
        W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(W, "bf16", cb)
        y_t = torch.empty((B, rows), dtype=torch.float32, device=DEV)
        mats.append(dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=None, y=y_t, key=(xk, cols)))
        refs.append(oracle.gemv(oracle.decode(idx_o, sc_o, cb), x, "bf16"))
    xdev = {k: to_dev(v, "bf16") for k, v in xs.items()}
    for m in mats:
        m["x"] = xdev[m.pop("key")]
    vq.vq3r_gemv(as_layout(mats, layout), B)
    for m, ref in zip(mats, refs):
        assert gemv_rel_err(m["y"].cpu().numpy(), ref) <= GEMV_TOL


@pytest.mark.parametrize("B", [8, 9, 12, 24, 32])
def test_grouped_gemv_many_tokens(B):
    """Many tokens, bf16 x, tiled layout, matrices with different codebooks: B <= 10 on the two-token lookup
    tables (an odd B leaves a pair with one token), B >= 11 on the tensor cores with the weights rebuilt in
    bf16 hi + lo (mma.sync, since the codebooks differ): ragged rows (not multiples of 128), partial last
    slabs, partly filled 8-token tiles, mixed groups."""
    rng = np.random.default_rng(80 + B)
    specs = [(300, 1032, 0, 0), (129, 1032, 0, 0), (64, 200, 1, 1), (513, 2048, 2, 0), (33, 1032, 0, 2)]
    xs = {}
    mats, refs = [], []
    for rows, cols, cbk, xk in specs:
        cb = random_codebooks(300 + cbk)
        if (xk, cols) not in xs:
            xs[(xk, cols)] = f32_to_bf16_bits(rng.standard_normal((B, cols)).astype(np.float32))
        x = xs[(xk, cols)]
        W = f32_to_bf16_bits(rng.standard_normal((rows, cols)).astype(np.float32))
        W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(W, "bf16", cb)
        y_t = torch.full((B, rows), float("nan"), dtype=torch.float32, device=DEV)
        mats.append(dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=None, y=y_t, key=(xk, cols)))
        refs.append(oracle.gemv(oracle.decode(idx_o, sc_o, cb), x, "bf16"))
    xdev = {k: to_dev(v, "bf16") for k, v in xs.items()}
    for m in mats:
        m["x"] = xdev[m.pop("key")]
    vq.vq3r_gemv(as_layout(mats, "tiles"), B)
    for m, ref in zip(mats, refs):
        y = m["y"].cpu().numpy()
        assert np.isfinite(y).all()  # every output written
        assert gemv_rel_err(y, ref) <= GEMV_TOL


@pytest.mark.parametrize("B", [17, 24, 32])
def test_grouped_gemv_tensor_memory_kernel(B):
    """17..32 tokens, bf16 x, tiled layout and one codebook set for the whole call run on the tcgen05 kernel
    (weights rebuilt in bf16 hi + lo into tensor memory): ragged rows (not multiples of 128), columns that end
    in the middle of a 16-column step (cols % 16 == 8), partial last slabs, a matrix of one step, mixed x
    groups, and the K-step split across warp-groups that cuts tiles in the middle."""
    rng = np.random.default_rng(90 + B)
    cb = random_codebooks(401)
    specs = [(300, 1032, 0), (129, 1032, 0), (64, 200, 1), (513, 2048, 2), (33, 1032, 0), (7, 8, 3), (2048, 7168, 4)]
    xs = {}
    mats, refs = [], []
    for rows, cols, xk in specs:
        if (xk, cols) not in xs:
            xs[(xk, cols)] = f32_to_bf16_bits(rng.standard_normal((B, cols)).astype(np.float32))
        x = xs[(xk, cols)]
        W = f32_to_bf16_bits((rng.standard_normal((rows, cols)) * np.exp(rng.standard_normal((rows, 1)))).astype(np.float32))
        W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(W, "bf16", cb)
        y_t = torch.full((B, rows), float("nan"), dtype=torch.float32, device=DEV)
        mats.append(dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=None, y=y_t, key=(xk, cols)))
        refs.append(oracle.gemv(oracle.decode(idx_o, sc_o, cb), x, "bf16"))
    xdev = {k: to_dev(v, "bf16") for k, v in xs.items()}
    cb_t = mats[0]["codebooks"]
    for m in mats:
        m["x"] = xdev[m.pop("key")]
        m["codebooks"] = cb_t  # one codebook tensor for the whole call
    ws = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    tiled = as_layout(mats, "tiles")
    for _ in range(2):  # twice: the second call reuses the workspace's grid-barrier counts
        for m in mats:
            m["y"].fill_(float("nan"))
        vq.vq3r_gemv(tiled, B, workspace=ws)
        for m, ref in zip(mats, refs):
            y = m["y"].cpu().numpy()
            assert np.isfinite(y).all()  # every output written
            assert gemv_rel_err(y, ref) <= GEMV_TOL
    assert vq.vq3r_device_error() == 0


@pytest.mark.parametrize("B", [1, 3])
def test_gemv_cuda_graph_replays(B):
    """A tiled GEMV captured once in a CUDA graph and replayed with new inputs: every replay repeats the
    captured kernel arguments, so the kernel's zeroing of y and its grid barrier (kept in the workspace
    header) must work from the state the previous replay left."""
    rng = np.random.default_rng(90 + B)
    cb = random_codebooks(400)
    specs = [(1100, 1032), (70, 1032)]
    mats, decoded = [], []
    x_t = torch.zeros((B, 1032), dtype=torch.float32, device=DEV)
    for rows, cols in specs:
        W = rng.standard_normal((rows, cols)).astype(np.float32)
        W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(W, "f32", cb)
        mats.append(dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=x_t,
                         y=torch.zeros((B, rows), dtype=torch.float32, device=DEV)))
        decoded.append(oracle.decode(idx_o, sc_o, cb))
    mats = as_layout(mats, "tiles")
    ws = torch.zeros(max(vq.vq3r_gemv_workspace_size(mats, B), 16), dtype=torch.uint8, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        vq.vq3r_gemv(mats, B, workspace=ws)  # warm-up outside the capture (first-call device setup)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        vq.vq3r_gemv(mats, B, workspace=ws)
    for rep in range(4):
        x = rng.standard_normal((B, 1032)).astype(np.float32)
        x_t.copy_(torch.from_numpy(x))
        for m in mats:
            m["y"].fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for m, Wd in zip(mats, decoded):
            y = m["y"].cpu().numpy()
            assert np.isfinite(y).all(), rep
            assert gemv_rel_err(y, oracle.gemv(Wd, x, "f32")) <= GEMV_TOL, rep
    assert vq.vq3r_device_error() == 0
    del g


# ------------------------------------------------------------------ error statuses

def test_error_statuses():
    cb = torch.zeros((3, 256, 8), device=DEV)
    with pytest.raises(vq.VQ3RError) as e:
        vq.vq3r_encode(torch.zeros((4, 12), device=DEV), cb)
    assert e.value.status == 2
    buf = torch.zeros(4 * 16 + 1, device=DEV)
    with pytest.raises(vq.VQ3RError) as e:
        vq.vq3r_encode(buf[1:].view(4, 16), cb)  # 4-byte offset: not 16-byte aligned
    assert e.value.status == 3
    W = torch.zeros((4, 16), device=DEV)
    idx, sc = vq.vq3r_encode(W, cb)
    y = torch.empty((1, 4), device=DEV)
    m = [dict(idx=idx, scales=sc, codebooks=cb, x=torch.zeros((1, 16), device=DEV), y=y)]
    with pytest.raises(vq.VQ3RError) as e:
        vq.vq3r_gemv(m, 33)
    assert e.value.status == 5
    with pytest.raises(vq.VQ3RError) as e:
        vq.vq3r_gemv(m, 1, workspace=torch.empty(16, dtype=torch.uint8, device=DEV))
    assert e.value.status == 7
    assert vq.vq3r_device_error() == 0


# ------------------------------------------------------------------ full-size workloads, sampled rows

def load_codebooks(name):
    import importlib.util
    import os
    p = os.path.join(os.path.dirname(__file__), "golden", "make_codebooks.py")
    spec = importlib.util.spec_from_file_location("make_codebooks", p)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return np.ascontiguousarray(mod.load(name))


def device_matrix(experts, kind, seed, dist):
    """Rows of `kind` for the listed experts stacked into one bf16 device tensor."""
    rows, cols = wl.mat_shape(kind)
    W = torch.empty((len(experts) * rows, cols), dtype=torch.bfloat16, device=DEV)
    for i, e in enumerate(experts):
        synth.fill_rows_device(W[i * rows:(i + 1) * rows].data_ptr(), cols, 0, rows, seed, wl.tag(e, kind), dist,
                               stream=torch.cuda.current_stream().cuda_stream)
    return W


def host_rows(experts, kind, seed, dist, stacked_rows):
    rows, cols = wl.mat_shape(kind)
    out = np.empty((len(stacked_rows), cols), dtype=np.uint16)
    for i, r in enumerate(stacked_rows):
        e = experts[r // rows]
        out[i] = synth.fill_row_list(cols, [r % rows], seed, wl.tag(e, kind), dist)[0]
    return out


@pytest.mark.parametrize("kind", [wl.W1, wl.W2])
def test_layer_stacked_encode_sampled_rows(kind):
    """Encode of a 64-expert layer matrix stacked into one call (the benchmark's
    launch), bit-exact against the oracle on 256 sampled rows."""
    cfg = wl.LAYER
    cb = load_codebooks("layer")
    experts = list(range(cfg["experts"]))
    W_t = device_matrix(experts, kind, cfg["seed"], wl.expert_dist())
    idx_t, sc_t = gpu_encode(W_t, cb)
    rng = np.random.default_rng(kind)
    sample = np.sort(rng.choice(W_t.shape[0], 256, replace=False))
    Wh = host_rows(experts, kind, cfg["seed"], wl.expert_dist(), sample)
    np.testing.assert_array_equal(host_bits(W_t[torch.from_numpy(sample).to(DEV)]), Wh)  # generators agree
    idx_o, sc_o = oracle.encode(Wh, "bf16", cb)
    sel = torch.from_numpy(sample).to(DEV)
    np.testing.assert_array_equal(sc_t[sel].cpu().numpy().view(np.uint16), sc_o)
    np.testing.assert_array_equal(idx_t[:, sel, :].cpu().numpy(), idx_o)


def test_expert_w2_full_matrix_bit_exact_and_error():
    """The single-expert workload's down projection w2 (7168 x 2048 bf16, Student-t(4) x log-normal rows, seed
    1) at full size: indices, scales and fp32 / fp16 decode bit-exact against the oracle on every row, and the
    error kernel within 1e-9 of the oracle's binary64 rel-Frobenius over the whole matrix."""
    cfg = wl.EXPERT
    cb = load_codebooks("expert")
    rows, cols = wl.mat_shape(wl.W2)
    Wh = synth.fill_rows(cols, 0, rows, cfg["seed"], wl.tag(0, wl.W2), wl.expert_dist())
    W_t = device_matrix([0], wl.W2, cfg["seed"], wl.expert_dist())
    np.testing.assert_array_equal(host_bits(W_t), Wh)  # the two generators agree on every element
    W_t, idx_t, sc_t, cb_t, idx_o, sc_o = check_encode_decode(Wh, "bf16", cb)
    e = float(vq.vq3r_rel_frobenius_error(W_t, idx_t, sc_t, cb_t).cpu()[0])
    e_ref = oracle.rel_frobenius(Wh, "bf16", oracle.decode(idx_o, sc_o, cb))
    assert abs(e - e_ref) <= RELFRO_TOL * e_ref, (e, e_ref)
    assert 0.1 < e_ref < 0.3  # sanity band, not parity


@pytest.mark.parametrize("layout", ["planes", "tiles"])
@pytest.mark.parametrize("B", [1, 4, 8, 32])
def test_moe_decode_step_gemv_sampled_rows(B, layout):
    """The MoE decode step (8 experts of the layer; gate/up in one call, down in
    one call) at full size against the binary64 oracle on sampled rows."""
    cfg = wl.LAYER
    cb = load_codebooks("layer")
    cb_t = torch.from_numpy(cb).to(DEV)
    experts = list(range(8))
    x_up = synth.fill_rows(wl.HIDDEN, 0, B, wl.ACT_SEED, wl.tag(0, wl.X_GATEUP), synth.normal())
    x_dn = [synth.fill_rows(wl.INTER, 0, B, wl.ACT_SEED, wl.tag(e, wl.X_DOWN), synth.normal()) for e in experts]
    x_up_t = to_dev(x_up, "bf16")
    phase1, phase2, checks = [], [], []
    rng = np.random.default_rng(B)
    for e in experts:
        for kind in (wl.W1, wl.W3, wl.W2):
            rows, cols = wl.mat_shape(kind)
            W_t = device_matrix([e], kind, cfg["seed"], wl.expert_dist())
            idx_t, sc_t = gpu_encode(W_t, cb)
            del W_t
            y_t = torch.empty((B, rows), dtype=torch.float32, device=DEV)
            if kind == wl.W2:
                phase2.append(dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=to_dev(x_dn[e], "bf16"), y=y_t))
            else:
                phase1.append(dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=x_up_t, y=y_t))
            sample = np.sort(rng.choice(rows, 24, replace=False))
            checks.append((y_t, e, kind, sample, x_dn[e] if kind == wl.W2 else x_up))
    vq.vq3r_gemv(as_layout(phase1, layout), B)
    vq.vq3r_gemv(as_layout(phase2, layout), B)
    torch.cuda.synchronize()
    worst = 0.0
    for y_t, e, kind, sample, x in checks:
        Wh = host_rows([e], kind, cfg["seed"], wl.expert_dist(), sample)
        idx_o, sc_o = oracle.encode(Wh, "bf16", cb)
        y_ref = oracle.gemv(oracle.decode(idx_o, sc_o, cb), x, "bf16")
        y = y_t.cpu().numpy()[:, sample]
        worst = max(worst, gemv_rel_err(y, y_ref))
    assert worst <= GEMV_TOL, worst


@pytest.mark.parametrize("kind", [wl.W1, wl.W2])
def test_sweep_256_experts_sampled_rows(kind):
    """The 256-expert scale sweep (Student-t(3) rows with 0.1% outliers at 20 sigma): one stacked matrix of all
    experts encoded in one call and bit-exact on 256 sampled rows; one expert's rel-Frobenius error consistent
    with its decode; and the GEMV over all 256 experts at B = 1 (both layouts), 4 and 32 (tiled) within the
    tolerance on the sampled rows."""
    cfg = wl.SWEEP
    cb = load_codebooks("sweep")
    cb_t = torch.from_numpy(cb).to(DEV)
    dist = wl.sweep_dist()
    experts = list(range(cfg["experts"]))
    rows, cols = wl.mat_shape(kind)
    W_t = device_matrix(experts, kind, cfg["seed"], dist)
    idx_t, sc_t = gpu_encode(W_t, cb)
    rng = np.random.default_rng(500 + kind)
    sample = np.sort(rng.choice(W_t.shape[0], 256, replace=False))
    sel = torch.from_numpy(sample).to(DEV)
    Wh = host_rows(experts, kind, cfg["seed"], dist, sample)
    np.testing.assert_array_equal(host_bits(W_t[sel]), Wh)  # generators agree
    idx_o, sc_o = oracle.encode(Wh, "bf16", cb)
    np.testing.assert_array_equal(sc_t[sel].cpu().numpy().view(np.uint16), sc_o)
    np.testing.assert_array_equal(idx_t[:, sel, :].cpu().numpy(), idx_o)

    # one expert (the last), a row range of the stacked arrays: every row of its indices and scales bit-exact,
    # and the error kernel within 1e-9 of the oracle's binary64 rel-Frobenius of the whole expert matrix
    e_last = cfg["experts"] - 1
    e0 = e_last * rows
    W_e, sc_e = W_t[e0:], sc_t[e0:]
    idx_e = idx_t[:, e0:, :].contiguous()
    We_h = synth.fill_rows(cols, 0, rows, cfg["seed"], wl.tag(e_last, kind), dist)
    idx_eo, sc_eo = oracle.encode(We_h, "bf16", cb)
    np.testing.assert_array_equal(sc_e.cpu().numpy().view(np.uint16), sc_eo)
    np.testing.assert_array_equal(idx_e.cpu().numpy(), idx_eo)
    err = float(vq.vq3r_rel_frobenius_error(W_e, idx_e, sc_e, cb_t).cpu()[0])
    err_ref = oracle.rel_frobenius(We_h, "bf16", oracle.decode(idx_eo, sc_eo, cb))
    assert abs(err - err_ref) <= RELFRO_TOL * err_ref, (err, err_ref)
    del W_t, W_e, idx_e
    torch.cuda.empty_cache()

    W_ref = oracle.decode(idx_o, sc_o, cb)
    tiles = vq.vq3r_pack_tiles(idx_t)
    for B, layouts in ((1, ("planes", "tiles")), (4, ("tiles",)), (32, ("tiles",))):
        x = synth.fill_rows(cols, 0, B, wl.ACT_SEED, wl.tag(900 + kind, wl.X_GATEUP), synth.normal())
        y_ref = oracle.gemv(W_ref, x, "bf16")
        for layout in layouts:
            y_t = torch.full((B, idx_t.shape[1]), float("nan"), dtype=torch.float32, device=DEV)
            m = dict(idx=idx_t, scales=sc_t, codebooks=cb_t, x=to_dev(x, "bf16"), y=y_t)
            if layout == "tiles":
                m.update(idx=tiles, layout="tiles", cols=cols)
            vq.vq3r_gemv([m], B)
            y = y_t[:, sel].cpu().numpy()
            assert np.isfinite(y).all()
            assert gemv_rel_err(y, y_ref) <= GEMV_TOL, (B, layout)
    assert vq.vq3r_device_error() == 0


# ------------------------------------------------------------------ prefill product on the tensor cores

@pytest.mark.parametrize("specs", [
    [(128, 64, 1)],                        # one tile, one token, one step
    [(130, 72, 5)],                        # ragged rows (2 blocks), ragged last step (9 vectors)
    [(300, 1032, 257)],                    # 3 row blocks, two token tiles (one of a single token)
    [(513, 2048, 300)],                    # a row block past a 512-row tile, 32 steps
    [(64, 520, 600), (200, 512, 40), (0, 64, 7), (96, 128, 0)],  # one call, several matrices, empty ones
])
def test_gemm_parity(specs):
    """The prefill product against the binary64 product of the bf16-rounded decoded weights (the oracle), on
    ragged rows, columns and token counts."""
    rng = np.random.default_rng(sum(r * 7 + c + t for r, c, t in specs))
    mats, refs = [], []
    for rows, cols, T in specs:
        cb = random_codebooks(rows + cols)
        W = f32_to_bf16_bits(rng.standard_normal((max(rows, 1), cols)).astype(np.float32))[:rows]
        W_t = to_dev(W, "bf16")
        idx_t, sc_t = gpu_encode(W_t, cb) if rows else (torch.zeros((3, 0, cols // 8), dtype=torch.uint8, device=DEV),
                                                      torch.zeros(0, dtype=torch.int16, device=DEV))
        x = f32_to_bf16_bits(rng.standard_normal((T, cols)).astype(np.float32))
        y_t = torch.full((T, rows), float("nan"), dtype=torch.float32, device=DEV)
        tiles = vq.vq3r_pack_tiles(idx_t) if rows else torch.zeros(16, dtype=torch.uint8, device=DEV)
        mats.append(dict(idx=tiles, scales=sc_t, codebooks=torch.from_numpy(cb).to(DEV), cols=cols,
                         x=to_dev(x, "bf16"), y=y_t))
        if rows and T:
            idx_o, sc_o = oracle.encode(W, "bf16", cb)
            refs.append(oracle.gemm(idx_o, sc_o, cb, x))
        else:
            refs.append(None)
    vq.vq3r_gemm(mats)
    torch.cuda.synchronize()
    assert vq.vq3r_device_error() == 0
    for m, ref in zip(mats, refs):
        if ref is None:
            continue
        y = m["y"].cpu().numpy()
        assert np.isfinite(y).all()  # every output written
        assert gemv_rel_err(y, ref) <= GEMM_TOL


def test_gemm_moe_prefill_sampled_rows():
    """Prefill of 8 experts' gate projections (2048 x 7168 each, rows of one packed stacked matrix) with a
    different number of routed tokens per expert, in one call; 24 sampled rows of every expert against the
    oracle."""
    cfg = wl.LAYER
    cb = load_codebooks("layer")
    cb_t = torch.from_numpy(cb).to(DEV)
    experts = list(range(8))
    rows, cols = wl.mat_shape(wl.W1)
    W_t = device_matrix(experts, wl.W1, cfg["seed"], wl.expert_dist())
    idx_t, sc_t = gpu_encode(W_t, cb)
    del W_t
    tiles = vq.vq3r_pack_tiles(idx_t)
    rng = np.random.default_rng(33)
    mats, checks = [], []
    for e in experts:
        T = 64 + 97 * e  # 64 .. 743 tokens
        x = synth.fill_rows(cols, 0, T, wl.ACT_SEED, wl.tag(100 + e, wl.X_GATEUP), synth.normal())
        y_t = torch.full((T, rows), float("nan"), dtype=torch.float32, device=DEV)
        mats.append(dict(idx=tiles, scales=sc_t, codebooks=cb_t, cols=cols, row0=e * rows, rows=rows,
                         x=to_dev(x, "bf16"), y=y_t))
        checks.append((e, x, y_t, np.sort(rng.choice(rows, 24, replace=False))))
    vq.vq3r_gemm(mats)
    torch.cuda.synchronize()
    assert vq.vq3r_device_error() == 0
    worst = 0.0
    for e, x, y_t, sample in checks:
        Wh = host_rows([e], wl.W1, cfg["seed"], wl.expert_dist(), sample)
        idx_o, sc_o = oracle.encode(Wh, "bf16", cb)
        ref = oracle.gemm(idx_o, sc_o, cb, x)
        y = y_t.cpu().numpy()
        assert np.isfinite(y).all()
        # the per-token rms floor is taken over the sampled rows
        worst = max(worst, gemv_rel_err(y[:, sample], ref))
    assert worst <= GEMM_TOL, worst


# ------------------------------------------------------------------ codebook training (Lloyd) on the GPU

def test_train_tiny_workload_bit_exact(tiny):
    """The tiny workload's codebooks (10 Lloyd iterations on all 16384 vectors) trained on the GPU equal the
    oracle's bit for bit; the distortion trace agrees to 1e-12."""
    W, cb = tiny
    cfg = wl.TINY
    vecs = oracle.normalize_rows(W, "f32", oracle.row_scales(W, "f32")).reshape(-1, 8)
    _, tr_o = oracle.lloyd_train(vecs, cfg["lloyd_iters"])
    cb_t, tr_t = vq.vq3r_train(torch.from_numpy(np.ascontiguousarray(vecs)).to(DEV), cfg["lloyd_iters"])
    np.testing.assert_array_equal(cb_t.cpu().numpy().view(np.uint32), cb.view(np.uint32))
    np.testing.assert_allclose(tr_t.cpu().numpy(), tr_o, rtol=1e-12)


@pytest.mark.parametrize("n,iters,nstages,dup", [(256, 3, 3, False), (1000, 5, 3, True), (4099, 0, 2, False),
                                                 (3000, 7, 1, True)])
def test_train_small_cases_bit_exact(n, iters, nstages, dup):
    """n = 256 (every vector its own centroid), duplicated vectors (empty clusters keep their centroid), no
    iterations, fewer stages, a ragged vector count."""
    rng = np.random.default_rng(n + iters)
    vecs = (rng.standard_normal((n, 8)) * np.exp(rng.standard_normal((n, 1)))).astype(np.float32)
    if dup:  # only 100 distinct vectors after the first 256: most clusters end up empty
        vecs[256:] = vecs[rng.integers(0, 100, n - 256)]
        vecs[:256] = vecs[rng.integers(0, 100, 256)]
    cb_o, tr_o = oracle.lloyd_train(vecs, iters, nstages)
    cb_t, tr_t = vq.vq3r_train(torch.from_numpy(vecs).to(DEV), iters, nstages)
    np.testing.assert_array_equal(cb_t.cpu().numpy().view(np.uint32), cb_o.view(np.uint32))
    np.testing.assert_allclose(tr_t.cpu().numpy(), tr_o, rtol=1e-12, atol=1e-300)


def test_train_reproduces_the_expert_codebooks():
    """The single-expert workload's stored codebooks (tests/golden/codebooks_expert.txt, written by the oracle:
    65536 sampled normalised vectors, 20 iterations, 3 stages) retrained on the GPU, bit for bit."""
    import importlib.util
    import os
    p = os.path.join(os.path.dirname(__file__), "golden", "make_codebooks.py")
    spec = importlib.util.spec_from_file_location("make_codebooks", p)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    cfg = wl.EXPERT
    vecs = mod.training_vectors(cfg["seed"], wl.expert_dist(), [0], cfg["train_vectors"])
    cb_t, tr_t = vq.vq3r_train(torch.from_numpy(vecs).to(DEV), cfg["lloyd_iters"])
    np.testing.assert_array_equal(cb_t.cpu().numpy().view(np.uint32), mod.load("expert").view(np.uint32))
