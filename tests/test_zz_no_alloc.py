"""vq3r_gemv_noalloc: the GEMV entry point for callers that cannot allocate
device memory (it uses the library's own static device scratch).

Kept in a file of its own that pytest collects last, so that a failure here
comes after every other test has run.  It passes alone in a fresh process
and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

from vq3r_cases import GEMV_TOL, gemv_rel_err

pytestmark = pytest.mark.gpu

vq = pytest.importorskip("residual_vector_quantization_b200")
DEV = "cuda"


def _matrices(B, seed):
    """Encoded-format inputs (indices, binary16 scales, codebooks) and activations
    for a grouped call: two matrices sharing x, one with its own x."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    cb = (torch.randn((3, 256, 8), generator=g) * torch.tensor([1.0, 0.45, 0.2])[:, None, None]).to(DEV)
    shapes = [(512, 1024, 0), (300, 1024, 0), (1000, 2048, 1)]
    xs = {0: torch.randn((B, 1024), generator=g).to(torch.bfloat16).to(DEV),
          1: torch.randn((B, 2048), generator=g).to(torch.bfloat16).to(DEV)}
    mats = []
    for rows, cols, xk in shapes:
        idx = torch.randint(0, 256, (3, rows, cols // 8), generator=g, dtype=torch.uint8).to(DEV)
        sc = torch.from_numpy(np.float16(np.exp(np.random.default_rng(seed + rows).standard_normal(rows)))
                              .view(np.int16)).to(DEV)
        mats.append(dict(idx=idx, scales=sc, codebooks=cb, x=xs[xk]))
    return mats


def _outs(mats, B):
    return [dict(m, y=torch.full((B, m["idx"].shape[1]), float("nan"), device=DEV)) for m in mats]


@pytest.mark.parametrize("B", [1, 3])
def test_noalloc_matches_gemv_on_two_calls_in_a_row(B):
    mats = _matrices(B, 7 + B)
    ref = _outs(mats, B)
    vq.vq3r_gemv(ref, B)  # the existing entry point, with a caller-allocated workspace
    L = vq.lib()
    s = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        got = _outs(mats, B)
        descs = vq._descs(got)
        assert L.vq3r_gemv_noalloc(descs, len(got), B, vq.VQ3R_BF16, s) == 0
        torch.cuda.synchronize()
        for r, o in zip(ref, got):
            y_ref = r["y"].cpu().numpy().astype(np.float64)
            y = o["y"].cpu().numpy()
            assert np.all(np.isfinite(y))
            assert gemv_rel_err(y, y_ref) <= GEMV_TOL


def test_noalloc_rejects_calls_that_need_more_scratch():
    B = 32
    cb = torch.zeros((3, 256, 8), device=DEV)
    x = torch.zeros((B, 4096), dtype=torch.bfloat16, device=DEV)
    mats = []
    for _ in range(2):
        rows, cols = 8192, 4096
        mats.append(dict(idx=torch.zeros((3, rows, cols // 8), dtype=torch.uint8, device=DEV),
                         scales=torch.zeros(rows, dtype=torch.int16, device=DEV), codebooks=cb, x=x,
                         y=torch.empty((B, rows), device=DEV)))
    descs = vq._descs(mats)
    L = vq.lib()
    assert L.vq3r_gemv_workspace_size(descs, len(mats), B) > (16 << 20)
    assert L.vq3r_gemv_noalloc(descs, len(mats), B, vq.VQ3R_BF16, torch.cuda.current_stream().cuda_stream) == 7
