"""Shared test inputs: closed-form codebooks, exact-energy vectors, random
codebooks, and the GEMV tolerance rule."""
import itertools

import numpy as np

K, D = 256, 8


def sign_pattern_codebooks(a=1.0):
    """C1 = all 256 sign patterns of +-a (bit k of j set <=> dim k negative),
    C2 = same with a/2, C3 = same with a/4."""
    j = np.arange(K)[:, None]
    k = np.arange(D)[None, :]
    sgn = np.where((j >> k) & 1, -1.0, 1.0)
    return np.stack([sgn * a, sgn * a / 2, sgn * a / 4]).astype(np.float32)


_TUPLES = None


def energy8_vectors(rng, n):
    """n vectors with entries k/4 (k integer in [-8, 8], zeros included) whose
    8 squares sum to exactly 8, so a row made of them has RMS exactly 1."""
    global _TUPLES
    if _TUPLES is None:
        _TUPLES = [c for c in itertools.combinations_with_replacement(range(0, 9), D)
                   if sum(x * x for x in c) == 128 and len(set(c)) >= 3]
    out = np.empty((n, D), dtype=np.float32)
    for i in range(n):
        t = np.array(_TUPLES[rng.integers(len(_TUPLES))], dtype=np.float64)
        rng.shuffle(t)
        t *= rng.choice([-1.0, 1.0], size=D)
        out[i] = t / 4.0
    return out


def random_codebooks(seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((3, K, D)) * np.array([1.0, 0.45, 0.2])[:, None, None]).astype(np.float32)


def f32_to_bf16_bits(a):
    """Round float32 to bfloat16 bits (RNE), for building exact test inputs."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def gemv_rel_err(y, y_ref):
    """max_i |y_i - y_ref_i| / max(|y_ref_i|, rms(y_ref[b])) over each token b."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    y_ref = np.atleast_2d(np.asarray(y_ref, dtype=np.float64))
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    den = np.maximum(np.abs(y_ref), rms)
    den[den == 0] = 1.0
    return float(np.max(np.abs(y - y_ref) / den)) if y.size else 0.0


GEMV_TOL = 2e-3       # max relative error of the GEMV (fp32 accumulation vs binary64)
RELFRO_TOL = 1e-9     # relative agreement of the binary64 error sums
# The prefill product multiplies bf16 weights by bf16 x: each product is exact in fp32, so only the fp32
# additions round.  Adding K terms of random sign, each addition errs by at most 2^-24 of a partial sum of
# size ~ sqrt(k) rms(term), so the error is at most ~ (2/3) 2^-24 K^1.5 rms(term) against |y| ~ sqrt(K)
# rms(term): (2/3) 2^-24 K = 3e-4 relative to rms(y) at K = 7168 in the worst case, about 1e-6 typically.
GEMM_TOL = 3e-4
