"""The encoder's screening certificate, checked on the CPU against the distance definition.

The GPU encoder screens every codeword with a fused form
    L(c) = fl32((1/2 - 16u) |c|^2), then acc = fma(r_k, -c_k, acc), k = 0..7   (u = 2^-24)
and accepts the smallest L without the definition's scan when the second smallest exceeds it by
    M = fma(fl(fl(|c_best|^2 + R2) + |L_best|), 2^-19, 2^-126),   R2 = sum_k r_k^2 by fused multiply-adds.
These tests emulate that arithmetic in numpy and assert that whenever the test accepts, the screened winner is the
definition's winner: d_j = sum_k (r_k - c_jk)^2 with every binary32 operation rounded, lowest index on ties.
They also check that the test accepts nearly every vector of ordinary data.

The fused multiply-add is emulated exactly.  A binary32 product is exact in binary64, but the binary64 sum p + c
may round, and rounding that sum again to binary32 can differ from one rounding of the exact value: this happens
exactly when the binary64 sum lands on a binary32 rounding midpoint while the exact sum does not.  TwoSum gives
the rounding error of the binary64 sum, and its sign settles those midpoints.
"""
from fractions import Fraction

import numpy as np

F32 = np.float32


def fma32(a, b, c):
    """binary32 fused multiply-add fl32(a*b + c) with a single rounding (round to nearest even), elementwise."""
    a, b, c = np.broadcast_arrays(np.asarray(a, F32), np.asarray(b, F32), np.asarray(c, F32))
    p = a.astype(np.float64) * b.astype(np.float64)  # exact: 24 + 24 bits fit in 53
    c64 = c.astype(np.float64)
    s = p + c64
    bb = s - p
    err = (p - (s - bb)) + (c64 - bb)  # TwoSum: p + c = s + err exactly
    out = s.astype(F32)
    # binary32 neighbours around s, and the midpoint between them (exact in binary64)
    lo = np.where(out.astype(np.float64) <= s, out, np.nextafter(out, F32(-np.inf)))
    hi = np.nextafter(lo, F32(np.inf))
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) * 0.5
    on_mid = np.isfinite(mid) & (s == mid) & (err != 0)
    return np.where(on_mid, np.where(err > 0, hi, lo), out).astype(F32)


def _fma32_exact(a, b, c):
    """Reference for fma32: the exact rational a*b + c rounded once to binary32 (nearest, ties to even)."""
    v = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    x = F32(float(v))  # float(v) rounds once to binary64; correct it below when that lands on a midpoint
    lo = x if Fraction(float(x)) <= v else np.nextafter(x, F32(-np.inf))
    hi = np.nextafter(lo, F32(np.inf))
    dl, dh = v - Fraction(float(lo)), Fraction(float(hi)) - v
    if dl < dh:
        return lo
    if dh < dl:
        return hi
    return lo if (int(lo.view(np.uint32)) & 1) == 0 else hi


def test_fma32_rounds_once():
    """The emulation against exact rational arithmetic, on a constructed double-rounding case and on random and
    cancelling inputs.  The constructed case: c = 1 + 2^-23 (odd last bit), a*b = 2^-24 - 2^-70; the exact sum
    lies just below the midpoint 1 + 3 * 2^-24 and rounds down to c, while its binary64 rounding is the midpoint
    itself, which rounds to even, up to 1 + 2^-22."""
    a = np.array([2.0 ** -24 * (1 + 2.0 ** -23)], F32)
    b = np.array([1 - 2.0 ** -23], F32)
    c = np.array([1 + 2.0 ** -23], F32)
    naive = (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(F32)
    assert naive[0] == F32(1 + 2.0 ** -22)
    assert fma32(a, b, c)[0] == F32(1 + 2.0 ** -23) == _fma32_exact(a[0], b[0], c[0])
    rng = np.random.default_rng(11)
    n = 4000
    a = (rng.standard_normal(n) * 2.0 ** rng.integers(-30, 30, n)).astype(F32)
    b = (rng.standard_normal(n) * 2.0 ** rng.integers(-30, 30, n)).astype(F32)
    c = (rng.standard_normal(n) * 2.0 ** rng.integers(-60, 60, n)).astype(F32)
    c[: n // 4] = (-(a[: n // 4].astype(np.float64) * b[: n // 4])).astype(F32)  # near-total cancellation
    got = fma32(a, b, c)
    for i in range(n):
        assert got[i] == _fma32_exact(a[i], b[i], c[i]), (a[i], b[i], c[i])


def definition_argmin(r, C):
    """d_j in binary32 with every operation rounded, k ascending; argmin with the lowest index on ties."""
    e = (r[:, None, 0] - C[None, :, 0]).astype(F32)
    d = (e * e).astype(F32)
    for k in range(1, 8):
        e = (r[:, None, k] - C[None, :, k]).astype(F32)
        d = (d + (e * e).astype(F32)).astype(F32)
    return np.argmin(d, axis=1)  # first minimum = lowest index


def screen(r, C):
    """(index of the smallest L, accepted?) per vector, as the kernel computes them."""
    n = (C.astype(np.float64) ** 2).sum(axis=1)
    start = ((0.5 - 2.0 ** -20) * n).astype(F32)
    c2 = n.astype(F32)
    c2 = np.where(c2.astype(np.float64) < n, np.nextafter(c2, F32(np.inf)), c2)  # rounded up
    acc = np.broadcast_to(start, (r.shape[0], C.shape[0])).astype(F32)
    for k in range(8):
        acc = fma32(np.broadcast_to(r[:, None, k], acc.shape), np.broadcast_to(-C[None, :, k], acc.shape), acc)
    bi = np.argmin(acc, axis=1)  # strict < tracking keeps the first minimum
    best = acc[np.arange(len(r)), bi]
    part = np.partition(acc, 1, axis=1)
    second = part[:, 1]
    r2 = fma32(r[:, 0], r[:, 0], np.zeros(len(r), F32))
    for k in range(1, 8):
        r2 = fma32(r[:, k], r[:, k], r2)
    s = ((c2[bi] + r2).astype(F32) + np.abs(best)).astype(F32)
    m = fma32(s, np.full_like(s, F32(2.0 ** -19)), np.full_like(s, F32(2.0 ** -126)))
    ok = ((second - best).astype(F32) > m) & (m < F32(2.0 ** 100))
    return bi, ok


def near_twin_codebook(rng, K=256, scale=1.0):
    C = (rng.standard_normal((K, 8)) * scale).astype(F32)
    half = K // 2
    for j in range(half):
        c = C[j].copy()
        k = j % 8
        kind = j % 4
        if kind == 1:
            c[k] = np.nextafter(c[k], F32(np.inf))
        elif kind >= 2:
            c[k] = F32(c[k] * (1 + 2.0 ** -int(rng.integers(10, 24))))
        C[half + j] = c
    return C


def test_no_false_accept_on_near_twins_and_near_codeword_vectors():
    rng = np.random.default_rng(2024)
    for trial in range(6):
        C = near_twin_codebook(rng, scale=float(0.25 * (trial + 1)))
        # residuals close to codewords (tiny gaps between a codeword and its twin), plus plain random ones
        j = rng.integers(0, 256, 6000)
        near = (C[j] + rng.standard_normal((6000, 8)).astype(F32) * F32(10.0 ** -rng.integers(1, 7))).astype(F32)
        plain = (rng.standard_normal((6000, 8)) * rng.uniform(0.1, 4.0)).astype(F32)
        r = np.concatenate([near, plain]).astype(F32)
        bi, ok = screen(r, C)
        want = definition_argmin(r, C)
        assert np.array_equal(bi[ok], want[ok]), "certificate accepted a wrong winner"
        assert ok.sum() > 0


def test_certificate_accepts_almost_all_ordinary_vectors():
    rng = np.random.default_rng(7)
    C = (rng.standard_normal((256, 8)) * 0.8).astype(F32)
    r = (rng.standard_normal((20000, 8))).astype(F32)
    bi, ok = screen(r, C)
    assert np.array_equal(bi[ok], definition_argmin(r, C)[ok])
    assert ok.mean() > 0.995, ok.mean()


def test_exact_ties_are_never_accepted():
    rng = np.random.default_rng(9)
    C = (rng.standard_normal((128, 8))).astype(F32)
    C = np.concatenate([C, C]).astype(F32)  # every codeword twice: every screen has a tie
    r = (rng.standard_normal((4000, 8))).astype(F32)
    _, ok = screen(r, C)
    assert not ok.any()


def test_vq4p_sized_codebooks_near_twins():
    rng = np.random.default_rng(64)
    for trial in range(4):
        C = near_twin_codebook(rng, K=64, scale=float(0.5 * (trial + 1)))
        j = rng.integers(0, 64, 8000)
        r = (C[j] + rng.standard_normal((8000, 8)).astype(F32) * F32(10.0 ** -rng.integers(1, 7))).astype(F32)
        bi, ok = screen(r, C)
        assert np.array_equal(bi[ok], definition_argmin(r, C)[ok])


def test_mixed_norm_codebooks():
    """A few codewords of norm ~1e3 among ordinary ones: the margin uses the chosen codeword's own norm."""
    rng = np.random.default_rng(65)
    C = (rng.standard_normal((256, 8)) * 0.7).astype(F32)
    C[rng.choice(256, 8, replace=False)] *= F32(1500.0)
    r = np.concatenate([(rng.standard_normal((8000, 8))).astype(F32),
                        (C[rng.integers(0, 256, 2000)] * F32(1.0001)).astype(F32)])
    bi, ok = screen(r, C)
    assert np.array_equal(bi[ok], definition_argmin(r, C)[ok])
    assert ok[:8000].mean() > 0.99


def test_tiny_and_subnormal_scale_residuals():
    """Residuals and codewords around 1e-20 (squares near the binary32 subnormal range)."""
    rng = np.random.default_rng(66)
    for s in (1e-12, 1e-18, 1e-20):
        C = (rng.standard_normal((256, 8)) * s).astype(F32)
        r = (rng.standard_normal((6000, 8)) * s).astype(F32)
        bi, ok = screen(r, C)
        assert np.array_equal(bi[ok], definition_argmin(r, C)[ok])


def test_large_values_and_overflow():
    """Large values whose squares stay finite (1e17): accepted winners are right.  Values whose squares overflow
    binary32 (1e19 and up): the margin is infinite or at least 2^100 and the test refuses, so those vectors go to
    the definition's scan."""
    rng = np.random.default_rng(67)
    with np.errstate(over="ignore", invalid="ignore"):
        C = (rng.standard_normal((256, 8)) * 1e17).astype(F32)
        r = (rng.standard_normal((2000, 8)) * 1e17).astype(F32)
        bi, ok = screen(r, C)
        assert np.array_equal(bi[ok], definition_argmin(r, C)[ok])
        for s in (1e19, 1e30):
            C = (rng.standard_normal((256, 8)) * s).astype(F32)
            r = (rng.standard_normal((2000, 8)) * s).astype(F32)
            _, ok = screen(r, C)
            assert not ok.any()
