"""Pins of the CPU oracle against what the source pages and the mathematics
fix, independent of the oracle's own code.

Page: "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验"
(xdnf.cn/news/289497), §2 (format, reconstruction rule, Lloyd codebooks),
§3.1 (relative Frobenius error, rtn4-row, vq2), §4 (greedy single pass),
§5 (the VQ4P sibling: 4 stages x 64 entries, 6-bit packed indices).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth
from synth import workloads as wl

K, D = 256, 8


from vq3r_cases import energy8_vectors, sign_pattern_codebooks  # noqa: E402


# ---------------------------------------------------------------- generator

def test_philox_known_answers():
    """Philox4x32-10 known-answer vectors (Salmon et al., SC'11, Random123 KAT)."""
    assert synth.philox([0, 0, 0, 0], [0, 0]) == [0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8]
    assert synth.philox([0xffffffff] * 4, [0xffffffff] * 2) == [0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd]
    assert synth.philox([0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344], [0xa4093822, 0x299f31d0]) == \
        [0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1]


def test_generator_moments_and_row_independence():
    d = synth.normal()
    a = synth.fill_rows(4096, 0, 64, 7, 3, d, dtype="f32")
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    # any row range regenerates the same values
    b = synth.fill_rows(4096, 17, 5, 7, 3, d, dtype="f32")
    np.testing.assert_array_equal(a[17:22], b)
    c = synth.fill_row_list(4096, [40, 2, 40], 7, 3, d, dtype="f32")
    np.testing.assert_array_equal(c[0], a[40])
    np.testing.assert_array_equal(c[1], a[2])
    t = synth.fill_rows(2048, 0, 64, 7, 3, synth.student_t(4), dtype="f32").astype(np.float64)
    # Student-t(4) variance = df / (df - 2) = 2
    assert abs(t.var() - 2.0) < 0.15


def test_sweep_distribution_outliers_and_row_factors():
    """The scale-sweep recipe: Student-t(3) values times a log-normal(0, 0.5) row factor, with 0.1% of the
    positions replaced by +-20 sigma (sigma = sqrt(3), the t(3) standard deviation) times the row factor."""
    rows, cols, seed, tag = 256, 4096, 4, 8
    full = synth.fill_rows(cols, 0, rows, seed, tag, wl.sweep_dist(), dtype="f32").astype(np.float64)
    plain = synth.fill_rows(cols, 0, rows, seed, tag, synth.student_t(3, row_sigma=0.5), dtype="f32")
    unit = synth.fill_rows(cols, 0, rows, seed, tag, synth.student_t(3), dtype="f32").astype(np.float64)
    rowf = plain.astype(np.float64) / unit
    rowf_row = np.median(rowf, axis=1)
    # one factor per row, log-normal with sigma 0.5
    assert np.allclose(rowf, rowf_row[:, None], rtol=1e-6)
    assert abs(np.log(rowf_row).std() - 0.5) < 0.08 and abs(np.log(rowf_row).mean()) < 0.1
    # t(3) against its closed-form CDF, F(t) = 1/2 + (atan(u) + u / (1 + u^2)) / pi with u = t / sqrt(3):
    # P(|t| <= a) = 2 F(a) - 1 (sd of the empirical fraction < 0.0005 at this size)
    for a in (0.25, 0.7649, 1.5, 4.0, 10.0):
        u = a / math.sqrt(3.0)
        expect = 2.0 * (0.5 + (math.atan(u) + u / (1.0 + u * u)) / math.pi) - 1.0
        assert abs((np.abs(unit) <= a).mean() - expect) < 0.003, a
    # outliers: about 0.1% of the positions, exactly +-20 sqrt(3) x row factor, either sign
    out = full != plain
    n = out.sum()
    assert 850 < n < 1250, n  # binomial(1 048 576, 1e-3): mean 1049, sd 32
    mag = np.abs(full[out]) / np.broadcast_to(rowf_row[:, None], full.shape)[out]
    assert np.allclose(mag, 20.0 * np.sqrt(3.0), rtol=1e-6)
    assert 0.4 < (full[out] > 0).mean() < 0.6


def test_sample_without_replacement():
    s = synth.sample(5, 9, 100000, 5000)
    assert len(np.unique(s)) == 5000 and s.min() >= 0 and s.max() < 100000
    assert abs(s.mean() - 50000) < 2000
    np.testing.assert_array_equal(s[:100], synth.sample(5, 9, 100000, 100))


# ---------------------------------------------------------------- conversions

def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-8, 5, 2000),
                         [0.0, -0.0, 1.0, 65504.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14]])
    for x in xs:
        assert oracle.fp16_from_double_sat(x) == int(np.float16(x).view(np.uint16)), x
        h = int(np.float16(x).view(np.uint16))
        assert oracle.fp16_to_double(h) == float(np.float16(x))


def test_fp16_midpoints_and_saturation():
    assert oracle.fp16_from_double_sat(1 + 2 ** -11) == 0x3C00          # tie -> even (1.0)
    assert oracle.fp16_from_double_sat(1 + 3 * 2 ** -11) == 0x3C02      # tie -> even (1 + 2^-9)
    assert oracle.fp16_from_double_sat(65520.0) == 0x7BFF               # saturating reading
    assert oracle.fp16_from_double_sat(1e9) == 0x7BFF
    assert oracle.fp16_from_float(65520.0) == 0x7C00                    # plain conversion: inf
    assert oracle.fp16_from_double_sat(2.0 ** -25) == 0x0000            # tie -> even (0)
    assert oracle.fp16_from_double_sat(3 * 2.0 ** -25) == 0x0002


# ---------------------------------------------------------------- scale (§2)

@pytest.mark.parametrize("cols", [8, 512, 2048, 7168])
def test_scale_of_constant_magnitude_rows(cols):
    rng = np.random.default_rng(cols)
    for m in [2.0 ** -10, 0.25, 1.0, 4.0, 1024.0]:
        W = (rng.choice([-1.0, 1.0], size=(3, cols)) * m).astype(np.float32)
        sc = oracle.row_scales(W, "f32")
        assert all(oracle.fp16_to_double(s) == m for s in sc)


def test_scale_rne_midpoints_and_limits():
    W = np.full((4, 1024), 1 + 2 ** -11, dtype=np.float32)
    W[1] = 1 + 3 * 2 ** -11
    W[2] = 70000.0
    W[3] = 2.0 ** -20
    sc = oracle.row_scales(W, "f32")
    assert list(sc) == [0x3C00, 0x3C02, 0x7BFF, 0x0010]
    assert oracle.row_scales(np.zeros((1, 64), np.float32), "f32")[0] == 0


def test_scale_equals_correctly_rounded_rms():
    """binary16(sqrt(mean w^2)) with the mean taken exactly (math.fsum)."""
    rng = np.random.default_rng(1)
    for cols in (8, 512, 7168):
        W = (rng.standard_normal((16, cols)) * np.exp(rng.standard_normal((16, 1)))).astype(np.float32)
        sc = oracle.row_scales(W, "f32")
        for i in range(16):
            ss = math.fsum(float(w) * float(w) for w in W[i])
            ref = np.float16(math.sqrt(ss / cols))
            assert sc[i] == int(ref.view(np.uint16))


# ---------------------------------------------------------------- encode/decode closed forms

def _greedy_scalar_levels(r):
    """Per-dimension greedy binary expansion with step a, a/2, a/4 (a = 1),
    exact in rationals; a zero residual takes the positive codeword."""
    bits = np.zeros((3, D), dtype=np.int64)
    w = np.zeros(D, dtype=np.float64)
    for k in range(D):
        e = Fraction(float(r[k]))
        acc = Fraction(0)
        for s, step in enumerate([Fraction(1), Fraction(1, 2), Fraction(1, 4)]):
            neg = e < 0
            bits[s, k] = 1 if neg else 0
            c = -step if neg else step
            e -= c
            acc += c
        w[k] = float(acc)
    return bits, w


def test_sign_pattern_codebooks_equal_scalar_quantizer():
    """With sign-pattern codebooks (+-1, +-1/2, +-1/4) greedy RVQ is the uniform
    8-level scalar quantizer +-{1.75, 1.25, 0.75, 0.25} per dimension, ties to
    the lower index (positive codeword); all arithmetic is exact."""
    rng = np.random.default_rng(2)
    cb = sign_pattern_codebooks()
    V, rows = 16, 24
    W = energy8_vectors(rng, rows * V).reshape(rows, V * D)
    idx, sc = oracle.encode(W, "f32", cb)
    assert all(s == 0x3C00 for s in sc)  # RMS exactly 1
    What = oracle.decode(idx, sc, cb)
    for i in range(rows):
        for v in range(V):
            bits, w = _greedy_scalar_levels(W[i, v * D:(v + 1) * D])
            for s in range(3):
                assert idx[s, i, v] == int(sum(int(b) << k for k, b in enumerate(bits[s])))
            np.testing.assert_array_equal(What[i, v * D:(v + 1) * D], w.astype(np.float32))


def test_permuted_sign_codebooks_tie_goes_to_lowest_index():
    rng = np.random.default_rng(3)
    cb = sign_pattern_codebooks()
    perm = rng.permutation(K)
    cbp = cb[:, perm, :]
    r = energy8_vectors(rng, 200)
    r[:, 0] = 0.0  # force a tie in dimension 0 at stage 1
    idx, _ = oracle.encode_vectors(r, cbp, nstages=1)
    for i in range(200):
        # codewords whose signs match every nonzero dimension all tie; lowest position wins
        cand = []
        for pos in range(K):
            j = perm[pos]
            ok = all(r[i, k] == 0 or ((j >> k) & 1) == (1 if r[i, k] < 0 else 0) for k in range(D))
            if ok:
                cand.append(pos)
        assert idx[i, 0] == min(cand)


def test_planted_exact_reconstruction():
    """Rows s * C1[pi(v)] with +-1 sign-pattern C1 and zero codeword 0 in C2, C3:
    scale = s exactly, indices (pi(v), 0, 0), decode exact, error 0."""
    rng = np.random.default_rng(4)
    cb = sign_pattern_codebooks()
    cb[0] = cb[0][rng.permutation(K)]
    cb[1] = rng.standard_normal((K, D)).astype(np.float32) * 0.3
    cb[2] = rng.standard_normal((K, D)).astype(np.float32) * 0.1
    cb[1, 0] = 0.0
    cb[2, 0] = 0.0
    rows, V = 12, 32
    pi = rng.integers(0, K, size=(rows, V))
    svals = np.array([0.75, 3.0, 2.0 ** -6, 1.5, 40.0, 0.125] * 2, dtype=np.float32)
    W = (cb[0][pi].reshape(rows, V * D) * svals[:, None]).astype(np.float32)
    Wb = synth.bf16_bits_to_f32((W.view(np.uint32) >> 16).astype(np.uint16))
    np.testing.assert_array_equal(Wb, W)  # exactly representable in bf16 too
    for dt, Win in (("f32", W), ("bf16", (W.view(np.uint32) >> 16).astype(np.uint16))):
        idx, sc = oracle.encode(Win, dt, cb)
        np.testing.assert_array_equal([oracle.fp16_to_double(s) for s in sc], svals.astype(np.float64))
        np.testing.assert_array_equal(idx[0], pi)
        assert not idx[1].any() and not idx[2].any()
        What = oracle.decode(idx, sc, cb)
        np.testing.assert_array_equal(What, W)
        assert oracle.rel_frobenius(Win, dt, What) == 0.0


def test_zero_row_and_zero_scale():
    cb = sign_pattern_codebooks()
    W = np.zeros((2, 16), np.float32)
    W[1] = 2.0 ** -30  # RMS underflows binary16 -> scale 0 -> r = 0
    idx, sc = oracle.encode(W, "f32", cb)
    assert list(sc) == [0, 0]
    What = oracle.decode(idx, sc, cb)
    assert not What.any()


def test_bits_per_weight_is_three():
    rng = np.random.default_rng(5)
    cb = rng.standard_normal((3, K, D)).astype(np.float32)
    for rows, cols in ((3, 8), (5, 512), (2, 7168)):
        W = rng.standard_normal((rows, cols)).astype(np.float32)
        idx, sc = oracle.encode(W, "f32", cb)
        assert idx.nbytes == 3 * rows * cols // 8
        assert idx.nbytes * 8 / (rows * cols) == 3.0
        assert sc.nbytes * 8 / (rows * cols) == 16 / cols


# ---------------------------------------------------------------- greedy vs exhaustive

def test_exhaustive_joint_search_lower_bounds_greedy():
    rng = np.random.default_rng(6)
    cb = (rng.standard_normal((3, K, D)) * np.array([1.0, 0.5, 0.25])[:, None, None]).astype(np.float32)
    r = rng.standard_normal((6, D)).astype(np.float32)
    idx, _ = oracle.encode_vectors(r, cb)
    g = cb[0][idx[:, 0]].astype(np.float64) + cb[1][idx[:, 1]] + cb[2][idx[:, 2]]
    greedy_err = ((r.astype(np.float64) - g) ** 2).sum(1)
    bidx, berr = oracle.bruteforce_joint(r, cb)
    assert np.all(berr <= greedy_err + 1e-12)
    # the exhaustive result is the reported triple's error
    bj = cb[0][bidx[:, 0]].astype(np.float64) + cb[1][bidx[:, 1]] + cb[2][bidx[:, 2]]
    np.testing.assert_allclose(((r.astype(np.float64) - bj) ** 2).sum(1), berr, rtol=1e-12)


def test_exhaustive_finds_a_planted_joint_optimum_that_greedy_misses():
    """Codebooks built so that each test vector r = e_m (unit vector of dim m) has exactly one triple summing to
    it, C1[b] + C2[p] + C3[z3] = 0.5 e_m + 0.5 e_m + 0, while greedy is lured by C1[a] = 0.875 e_m (distance
    1/64 against 1/4 for C1[b]) and then takes the zero codewords, ending at error exactly 1/64.  Every other
    codeword sits at 64 + j on dimension 7 (all positive, so no two of them cancel).  The planted indices sit at
    the ends and the middle of each range (b = 255 for one vector, p = 255 for another, z3 = 255 for all), so a
    search that skipped any part of a range, or mixed up which stage a codebook belongs to, returns another
    triple or a non-zero error.  All values are dyadic: the expected errors are exact in binary64."""
    cb = np.zeros((3, K, D), np.float32)
    for s in range(3):
        cb[s, :, 7] = 64.0 + np.arange(K)
    z2, z3 = 7, 255
    cb[1, z2] = 0.0
    cb[2, z3] = 0.0
    plants = [(0, 0, 255, 17), (1, 1, 3, 255), (2, 2, 128, 129), (3, 254, 200, 0), (4, 100, 5, 254)]
    for m, a, b, p in plants:
        cb[0, a] = 0.0
        cb[0, a, m] = 0.875
        cb[0, b] = 0.0
        cb[0, b, m] = 0.5
        cb[1, p] = 0.0
        cb[1, p, m] = 0.5
    r = np.zeros((len(plants), D), np.float32)
    for i, (m, _, _, _) in enumerate(plants):
        r[i, m] = 1.0
    # greedy: the lure, then the zero codewords; error 1/64
    idx, res = oracle.encode_vectors(r, cb)
    np.testing.assert_array_equal(idx, [[a, z2, z3] for _, a, _, _ in plants])
    np.testing.assert_array_equal((res.astype(np.float64) ** 2).sum(1), np.full(len(plants), 1.0 / 64))
    # exhaustive: the planted triple, error exactly zero
    bidx, berr = oracle.bruteforce_joint(r, cb)
    np.testing.assert_array_equal(bidx, [[b, p, z3] for _, _, b, p in plants])
    np.testing.assert_array_equal(berr, np.zeros(len(plants)))


def test_exhaustive_equals_greedy_when_later_stages_are_zero():
    rng = np.random.default_rng(7)
    cb = np.zeros((3, K, D), np.float32)
    cb[0] = rng.standard_normal((K, D))
    r = rng.standard_normal((4, D)).astype(np.float32)
    idx, _ = oracle.encode_vectors(r, cb)
    bidx, _ = oracle.bruteforce_joint(r, cb)
    np.testing.assert_array_equal(bidx[:, 0], idx[:, 0])


# ---------------------------------------------------------------- Lloyd (§2, §4)

def test_lloyd_recovers_separated_centres():
    rng = np.random.default_rng(8)
    centres = (rng.integers(-64, 64, size=(K, D)) * 4.0).astype(np.float32)
    centres[:, 0] = np.arange(K) * 8.0  # all distinct and far apart
    off = np.zeros((4, D), np.float32)
    off[0, 1], off[1, 1], off[2, 2], off[3, 2] = 0.125, -0.125, 0.25, -0.25
    pts = (centres[None, :, :] + off[:, None, :]).reshape(-1, D)  # first 256 = one per cluster
    cb, tr = oracle.lloyd_train(pts, iters=2, nstages=1)
    np.testing.assert_array_equal(cb[0], centres)
    assert tr[0, -1] == pytest.approx(K * (2 * 0.125 ** 2 + 2 * 0.25 ** 2))


def test_lloyd_matches_sklearn_lloyd():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(9)
    X = rng.standard_normal((2048, D)).astype(np.float32)
    cb, _ = oracle.lloyd_train(X, iters=3, nstages=1)
    km = KMeans(n_clusters=K, init=X[:K].astype(np.float64), n_init=1, max_iter=3, tol=0.0,
                algorithm="lloyd").fit(X.astype(np.float64))
    close = np.all(np.abs(km.cluster_centers_ - cb[0]) < 1e-5, axis=1)
    assert close.mean() > 0.95


def test_lloyd_distortion_non_increasing_and_stages_reduce_error():
    rng = np.random.default_rng(10)
    X = rng.standard_normal((8192, D)).astype(np.float32)
    cb, tr = oracle.lloyd_train(X, iters=6)
    for s in range(3):
        assert np.all(np.diff(tr[s]) <= 1e-6 * tr[s][0])
    # on the training set each stage lowers total distortion (cluster means
    # minimise squared error; zero is always a worse candidate centre)
    e = []
    for ns in (1, 2, 3):
        _, res = oracle.encode_vectors(X, cb[:ns], nstages=ns)
        e.append(float((res.astype(np.float64) ** 2).sum()))
    assert e[0] > e[1] > e[2]
    assert e[0] < float((X.astype(np.float64) ** 2).sum())
    # stage s training distortion equals the encoder's residual energy
    np.testing.assert_allclose(tr[2, -1], e[2], rtol=1e-6)


# ---------------------------------------------------------------- metric, GEMV, rtn4-row (§3.1)

def test_rel_frobenius_closed_forms():
    rng = np.random.default_rng(11)
    Wf = rng.standard_normal((8, 64)).astype(np.float32)
    W = (Wf.view(np.uint32) >> 16).astype(np.uint16)
    Wx = synth.bf16_bits_to_f32(W)
    assert oracle.rel_frobenius(W, "bf16", Wx) == 0.0
    assert oracle.rel_frobenius(W, "bf16", np.zeros_like(Wx)) == 1.0
    assert oracle.rel_frobenius(W, "bf16", Wx * np.float32(0.875)) == 0.125


def test_gemv_matches_float64_matmul():
    rng = np.random.default_rng(12)
    What = rng.standard_normal((33, 520)).astype(np.float32)
    x = rng.standard_normal((5, 520)).astype(np.float32)
    y = oracle.gemv(What, x, "f32")
    ref = x.astype(np.float64) @ What.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_bf16_rounding_matches_torch():
    """binary32 -> bfloat16 (RNE) against torch's CPU conversion: random values, exact ties either way,
    signed zeros, infinities, the largest finite values (overflow to inf) and subnormals."""
    import torch
    rng = np.random.default_rng(14)
    vals = [rng.standard_normal(3000) * 10.0 ** rng.integers(-38, 38, 3000)]
    ties = (np.arange(1, 200, dtype=np.uint32) << 16) | 0x8000  # exactly half-way, even and odd kept parts
    vals.append(ties.view(np.float32))
    vals.append(np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38, 1e-40, -1e-45], np.float64))
    xs = np.concatenate([v.astype(np.float32) for v in vals])
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.lib().orc_bf16_from_float(float(x)) for x in xs], dtype=np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_gemm_is_bf16_decoded_weights_times_x():
    """The prefill oracle: decode to bf16 equals torch's RNE of the binary32 decode, and the product equals
    numpy's float64 matmul of those weights with x."""
    import torch
    rng = np.random.default_rng(15)
    cb = rng.standard_normal((3, K, D)).astype(np.float32)
    idx = rng.integers(0, K, size=(3, 40, 24), dtype=np.uint8)
    sc = np.array([oracle.fp16_from_double_sat(v) for v in np.exp(rng.standard_normal(40))], np.uint16)
    w32 = oracle.decode(idx, sc, cb)
    wb = oracle.decode(idx, sc, cb, out="bf16")
    np.testing.assert_array_equal(wb, torch.from_numpy(w32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    xb = (rng.standard_normal((7, 192)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    y = oracle.gemm(idx, sc, cb, xb)
    W = (wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    x = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    np.testing.assert_allclose(y, x @ W.T, rtol=1e-12, atol=1e-12)


def test_rtn4_row_exact_grid_and_clamp():
    rng = np.random.default_rng(13)
    s = np.float32(0.375)
    q = rng.integers(-7, 8, size=(4, 64)).astype(np.float32)
    q[:, 0] = 7
    W = q * s
    What, sc = oracle.rtn4_row(W, "f32")
    assert all(oracle.fp16_to_double(h) == 0.375 for h in sc)
    np.testing.assert_array_equal(What, W)
    # a value of -7.6 scales rounds to -8 (inside the int4 range); with max |w| = 7.6 s the
    # scale is fp16(7.6 s / 7) and the extreme maps to +-7
    W2 = np.array([[7.0, -3.0, 1.0, 0.0] * 2], np.float32)
    W2[0, 1] = -7.6
    What2, sc2 = oracle.rtn4_row(W2, "f32")
    s2 = oracle.fp16_to_double(sc2[0])
    assert s2 == float(np.float16(7.6 / 7))
    assert What2[0, 1] == np.float32(-7 * s2)


# ---------------------------------------------------------------- sanity bands (not pins)

def test_tiny_pipeline_sanity_bands():
    """The tiny N(0,1) 256 x 512 case: errors in the expected bands and ordered
    rtn4-row < vq3 < vq2, the pattern of the Gate 3 table (§3.1)."""
    W = synth.fill_rows(512, 0, 256, 0, 0, synth.normal(), dtype="f32")
    sc = oracle.row_scales(W, "f32")
    vecs = oracle.normalize_rows(W, "f32", sc)
    cb, _ = oracle.lloyd_train(vecs, iters=10)
    idx3, sc3 = oracle.encode(W, "f32", cb)
    e3 = oracle.rel_frobenius(W, "f32", oracle.decode(idx3, sc3, cb))
    idx2, sc2 = oracle.encode(W, "f32", cb[:2], nstages=2)
    e2 = oracle.rel_frobenius(W, "f32", oracle.decode(idx2, sc2, cb[:2]))
    rt, _ = oracle.rtn4_row(W, "f32")
    e4 = oracle.rel_frobenius(W, "f32", rt)
    assert 0.10 < e3 < 0.26 and e2 > e3 and 0.10 < e4 < 0.18, (e4, e3, e2)


# ---------------------------------------------------------------- VQ4P, VQ3R's sibling (§5)

K4 = 64


def test_vq4p_packing_layout():
    """Four 6-bit indices per vector in the 24-bit word i1 | i2 << 6 | i3 << 12 | i4 << 18, stored as three
    byte planes: exactly the bytes of VQ3R's three index planes (3.00 bits/weight)."""
    idx = np.array([[1], [2], [4], [8]], dtype=np.uint8)  # word 0x204081
    np.testing.assert_array_equal(oracle.vq4p_pack(idx)[:, 0], [0x81, 0x40, 0x20])
    np.testing.assert_array_equal(oracle.vq4p_pack(np.full((4, 1), 63, np.uint8))[:, 0], [0xFF, 0xFF, 0xFF])
    np.testing.assert_array_equal(oracle.vq4p_pack(np.array([[0], [0], [0], [63]], np.uint8))[:, 0], [0, 0, 0xFC])
    rng = np.random.default_rng(40)
    idx = rng.integers(0, K4, size=(4, 7, 33), dtype=np.uint8)
    planes = oracle.vq4p_pack(idx)
    assert planes.shape == (3, 7, 33)
    np.testing.assert_array_equal(oracle.vq4p_unpack(planes), idx)


def _vq4p_sign_codebooks():
    """Stage s codeword j: dims 0..5 = -step if bit k of j is set else +step (step = 1, 1/2, 1/4, 1/8),
    dims 6 and 7 zero."""
    cb = np.zeros((4, K4, D), np.float32)
    for s, step in enumerate([1.0, 0.5, 0.25, 0.125]):
        for j in range(K4):
            for k in range(6):
                cb[s, j, k] = -step if (j >> k) & 1 else step
    return cb


def test_vq4p_sign_codebooks_equal_16_level_scalar_quantizer():
    """With those codebooks greedy VQ4P quantises dims 0..5 independently by sign at each stage (the 16-level
    uniform scalar quantizer), a zero residual taking the positive codeword (the lower index); inputs on a
    1/64 grid keep all binary32 arithmetic exact, so the expected indices follow in rationals."""
    rng = np.random.default_rng(41)
    cb = _vq4p_sign_codebooks()
    r = np.zeros((300, D), np.float32)
    r[:, :6] = rng.integers(-128, 129, size=(300, 6)) / 64.0
    r[:5, :6] = 0.0  # ties everywhere at stage 1
    idx, res = oracle.vq4p_encode_vectors(r, cb)
    for i in range(300):
        e = [Fraction(float(v)) for v in r[i, :6]]
        for s, step in enumerate([Fraction(1), Fraction(1, 2), Fraction(1, 4), Fraction(1, 8)]):
            bits = [1 if ek < 0 else 0 for ek in e]
            assert idx[i, s] == sum(b << k for k, b in enumerate(bits)), (i, s)
            e = [ek + step if b else ek - step for ek, b in zip(e, bits)]
        np.testing.assert_array_equal(res[i, :6], np.array([float(v) for v in e], np.float32))
        assert not res[i, 6:].any()


def test_vq4p_planted_exact_reconstruction():
    """Rows s * C1[pi(v)] with 64 distinct +-1 patterns as C1 and a zero codeword 0 in C2..C4: scale s exactly,
    indices (pi(v), 0, 0, 0), decode exact, error 0."""
    rng = np.random.default_rng(42)
    cb = (rng.standard_normal((4, K4, D)) * np.array([1.0, 0.3, 0.1, 0.03])[:, None, None]).astype(np.float32)
    for j in range(K4):
        cb[0, j] = [-1.0 if (j >> k) & 1 else 1.0 for k in range(6)] + [-1.0 if bin(j).count("1") & 1 else 1.0, 1.0]
    cb[0] = cb[0][rng.permutation(K4)]
    cb[1:, 0] = 0.0
    rows, V = 6, 16
    pi = rng.integers(0, K4, size=(rows, V))
    svals = np.array([0.75, 3.0, 2.0 ** -6, 1.5, 40.0, 0.125], dtype=np.float32)
    W = (cb[0][pi].reshape(rows, V * D) * svals[:, None]).astype(np.float32)
    planes, sc = oracle.vq4p_encode(W, "f32", cb)
    np.testing.assert_array_equal([oracle.fp16_to_double(s) for s in sc], svals.astype(np.float64))
    idx = oracle.vq4p_unpack(planes)
    np.testing.assert_array_equal(idx[0], pi)
    assert not idx[1:].any()
    What = oracle.vq4p_decode(planes, sc, cb)
    np.testing.assert_array_equal(What, W)
    assert oracle.rel_frobenius(W, "f32", What) == 0.0


def test_vq4p_exhaustive_joint_search_lower_bounds_greedy():
    rng = np.random.default_rng(43)
    cb = (rng.standard_normal((4, K4, D)) * np.array([1.0, 0.5, 0.25, 0.125])[:, None, None]).astype(np.float32)
    r = rng.standard_normal((2, D)).astype(np.float32)
    idx, _ = oracle.vq4p_encode_vectors(r, cb)
    g = sum(cb[s][idx[:, s]].astype(np.float64) for s in range(4))
    greedy_err = ((r.astype(np.float64) - g) ** 2).sum(1)
    bidx, berr = oracle.vq4p_bruteforce(r, cb)
    assert np.all(berr <= greedy_err + 1e-12)
    bj = sum(cb[s][bidx[:, s]].astype(np.float64) for s in range(4))
    np.testing.assert_allclose(((r.astype(np.float64) - bj) ** 2).sum(1), berr, rtol=1e-12)


def test_vq4p_lloyd_matches_sklearn_and_stages_reduce_error():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(44)
    X = rng.standard_normal((4096, D)).astype(np.float32)
    cb, tr = oracle.vq4p_train(X, 4)
    km = KMeans(n_clusters=K4, init=X[:K4].astype(np.float64), n_init=1, max_iter=4, tol=0.0,
                algorithm="lloyd").fit(X.astype(np.float64))
    close = np.all(np.abs(km.cluster_centers_ - cb[0]) < 1e-5, axis=1)
    assert close.mean() > 0.95
    for s in range(4):
        assert np.all(np.diff(tr[s]) <= 1e-6 * tr[s][0])
    idx, res = oracle.vq4p_encode_vectors(X, cb)
    np.testing.assert_allclose(tr[3, -1], float((res.astype(np.float64) ** 2).sum()), rtol=1e-6)
    # each added stage lowers the training error
    errs = []
    for ns in range(1, 5):
        g = sum(cb[s][idx[:, s]].astype(np.float64) for s in range(ns))
        errs.append(float(((X.astype(np.float64) - g) ** 2).sum()))
    assert errs[0] > errs[1] > errs[2] > errs[3]


# ---------------------------------------------------------------- outlier-aware variant (page "XFP", 权重分解)

def _vq3r_roundtrip(W, dtype, cb):
    idx, sc = oracle.encode(W, dtype, cb)
    return oracle.decode(idx, sc, cb)


def _widened(W, dtype):
    if dtype == "f32":
        return np.asarray(W, dtype=np.float64)
    if dtype == "bf16":
        return (np.asarray(W, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(W, dtype=np.uint16).view(np.float16).astype(np.float64)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_outliers_are_the_k_largest_errors_ties_to_lower_columns(dtype):
    """The stored set is the k largest |w - w_hat| of each row, lower columns first on ties, stored in column
    order with fp16(e) values: checked against numpy's own sort and float16 conversion."""
    from vq3r_cases import f32_to_bf16_bits, random_codebooks
    rng = np.random.default_rng(5)
    Wf = rng.standard_normal((24, 256)).astype(np.float32)
    Wf[:4] = rng.choice([-2.0, -1.0, 1.0, 2.0], size=(4, 256))  # many exact ties among the |e| of these rows
    W = Wf if dtype == "f32" else f32_to_bf16_bits(Wf)
    cb = random_codebooks(3)
    What = _vq3r_roundtrip(W, dtype, cb)
    What[:4] = 0.0  # so e = w exactly on the tie rows
    for k in (1, 7, 40, 256):
        oc, ov = oracle.outliers_select(W, dtype, What, k)
        e = _widened(W, dtype) - What.astype(np.float64)
        for i in range(W.shape[0]):
            order = np.lexsort((np.arange(256), -np.abs(e[i])))[:k]
            sel = np.sort(order)
            np.testing.assert_array_equal(oc[i], sel)
            np.testing.assert_array_equal(ov[i], e[i][sel].astype(np.float16).view(np.uint16))


def test_outliers_with_zero_codebooks_and_full_budget_reconstruct_exactly():
    """Zero codebooks decode to 0, so e = w; with every position an outlier and fp16-representable weights the
    decode plus outliers is W itself and the relative Frobenius error is exactly 0."""
    rng = np.random.default_rng(6)
    W = (rng.integers(-2048, 2048, size=(16, 128)) / 64.0).astype(np.float32)
    cb = np.zeros((3, 256, 8), dtype=np.float32)
    What = _vq3r_roundtrip(W, "f32", cb)
    assert not What.any()
    oc, ov = oracle.outliers_select(W, "f32", What, 128)
    W2 = oracle.outliers_apply(What, oc, ov)
    np.testing.assert_array_equal(W2, W)
    assert oracle.rel_frobenius(W, "f32", W2) == 0.0


def test_outlier_budget_never_increases_the_error():
    """Each added outlier replaces |e| by |e - fp16(e)| (plus one binary32 rounding), so the error is
    non-increasing in k; with every position an outlier it falls by about 2^-11."""
    cfg = wl.TINY
    W = synth.fill_rows(cfg["cols"], 0, cfg["rows"], cfg["seed"], wl.tag(0, wl.W1), synth.normal(), dtype="f32")
    cb, _ = oracle.lloyd_train(oracle.normalize_rows(W, "f32", oracle.row_scales(W, "f32")), 3)
    What = _vq3r_roundtrip(W, "f32", cb)
    errs = []
    for k in (0, 1, 2, 4, 8, 32, 128, 512):
        oc, ov = oracle.outliers_select(W, "f32", What, k)
        errs.append(oracle.rel_frobenius(W, "f32", oracle.outliers_apply(What, oc, ov)))
    assert all(b <= a for a, b in zip(errs, errs[1:])), errs
    assert errs[-1] < 1e-3 * errs[0]


def test_outliers_pick_planted_spikes():
    """Rows of N(0,1) weights with three 20-sigma spikes: the codebooks cannot follow a spike, so with k = 3 the
    spikes are exactly the stored outliers, and the error falls well below the plain VQ3R error."""
    from vq3r_cases import random_codebooks
    rng = np.random.default_rng(7)
    W = rng.standard_normal((32, 512)).astype(np.float32)
    spikes = np.stack([np.sort(rng.choice(512, 3, replace=False)) for _ in range(32)])
    for i in range(32):
        W[i, spikes[i]] = 20.0 * rng.choice([-1.0, 1.0], size=3)
    cb = random_codebooks(8)
    What = _vq3r_roundtrip(W, "f32", cb)
    oc, ov = oracle.outliers_select(W, "f32", What, 3)
    np.testing.assert_array_equal(oc, spikes)
    e0 = oracle.rel_frobenius(W, "f32", What)
    e3 = oracle.rel_frobenius(W, "f32", oracle.outliers_apply(What, oc, ov))
    assert e3 < 0.9 * e0
