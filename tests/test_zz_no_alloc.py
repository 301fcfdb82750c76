"""vq3r_gemv_noalloc: the GEMV entry point for callers that cannot allocate
device memory (it uses the library's own static device scratch).

Kept in a file of its own that pytest collects last, so that a failure here
comes after every other test has run.  It passes alone in a fresh process
and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import oracle
from vq3r_cases import GEMV_TOL, gemv_rel_err

pytestmark = pytest.mark.gpu

vq = pytest.importorskip("residual_vector_quantization_b200")
DEV = "cuda"


def _matrices(B, seed):
    """Encoded-format inputs (indices, binary16 scales, codebooks) and activations
    for a grouped call: two matrices sharing x, one with its own x.  Host copies
    are kept for the oracle."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    cb = (torch.randn((3, 256, 8), generator=g) * torch.tensor([1.0, 0.45, 0.2])[:, None, None])
    shapes = [(512, 1024, 0), (300, 1024, 0), (1000, 2048, 1)]
    xs = {0: torch.randn((B, 1024), generator=g).to(torch.bfloat16),
          1: torch.randn((B, 2048), generator=g).to(torch.bfloat16)}
    mats = []
    for rows, cols, xk in shapes:
        idx = torch.randint(0, 256, (3, rows, cols // 8), generator=g, dtype=torch.uint8)
        sc = np.float16(np.exp(np.random.default_rng(seed + rows).standard_normal(rows))).view(np.uint16)
        x_bits = xs[xk].view(torch.int16).numpy().view(np.uint16)
        y_ref = oracle.gemv(oracle.decode(idx.numpy(), sc, cb.numpy()), x_bits, "bf16")
        mats.append(dict(idx=idx.to(DEV), scales=torch.from_numpy(sc.view(np.int16)).to(DEV), codebooks=cb.to(DEV),
                         x=xs[xk].to(DEV), y_ref=y_ref))
    return mats


def _descs(mats, B, layout):
    """Output buffers (filled with NaN) and the C descriptors of one call in the given index layout."""
    outs = []
    for m in mats:
        d = dict(idx=m["idx"], scales=m["scales"], codebooks=m["codebooks"], x=m["x"],
                 y=torch.full((B, m["idx"].shape[1]), float("nan"), device=DEV))
        if layout == "tiles":
            d.update(idx=m["tiles"], layout="tiles", cols=m["idx"].shape[2] * 8)
        outs.append(d)
    return outs, vq._descs(outs)


def _check(mats, outs):
    for m, o in zip(mats, outs):
        y = o["y"].cpu().numpy()
        assert np.all(np.isfinite(y))
        assert gemv_rel_err(y, m["y_ref"]) <= GEMV_TOL


@pytest.mark.parametrize("B", [1, 3])
def test_noalloc_matches_oracle_and_gemv_on_two_calls_in_a_row(B):
    mats = _matrices(B, 7 + B)
    ref, _ = _descs(mats, B, "planes")
    vq.vq3r_gemv(ref, B)  # the existing entry point, with a caller-allocated workspace
    torch.cuda.synchronize()
    _check(mats, ref)
    L = vq.lib()
    s = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        got, descs = _descs(mats, B, "planes")
        assert L.vq3r_gemv_noalloc(descs, len(got), B, vq.VQ3R_BF16, s) == 0
        torch.cuda.synchronize()
        _check(mats, got)
        for r, o in zip(ref, got):
            assert gemv_rel_err(o["y"].cpu().numpy(), r["y"].cpu().numpy().astype(np.float64)) <= GEMV_TOL


def test_noalloc_alternating_layouts_share_the_array_and_allocate_nothing():
    """Tiled calls (B = 1 on the lookup-table kernel, B = 8 on the tensor-core kernel) alternate with plane-layout
    calls (which keep partial sums in the array) on the one static array.  Every result matches the oracle, and
    the device's free memory is the same before and after the calls."""
    L = vq.lib()
    s = torch.cuda.current_stream().cuda_stream
    cases = []
    for B in (1, 8):
        mats = _matrices(B, 40 + B)
        for m in mats:
            m["tiles"] = vq.vq3r_pack_tiles(m["idx"])
        for layout in ("tiles", "planes"):
            outs, descs = _descs(mats, B, layout)
            cases.append((B, layout, mats, outs, descs))
    # one call of each kind first: any lazily loaded kernel code is in place before free memory is measured
    for B, layout, mats, outs, descs in cases:
        assert L.vq3r_gemv_noalloc(descs, len(outs), B, vq.VQ3R_BF16, s) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        for B, layout, mats, outs, descs in cases:
            for o in outs:
                o["y"].fill_(float("nan"))
            assert L.vq3r_gemv_noalloc(descs, len(outs), B, vq.VQ3R_BF16, s) == 0, (B, layout)
            torch.cuda.synchronize()
            _check(mats, outs)
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


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
