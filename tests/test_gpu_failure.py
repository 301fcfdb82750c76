"""Failure detection without a GPU fault: a bounded wait that nothing completes runs out after about one second,
the kernel records the device error word and returns, the host reads (and clears) it, and the context is still
usable afterwards."""
import time

import numpy as np
import pytest
import torch

import oracle
from vq3r_cases import random_codebooks

pytestmark = pytest.mark.gpu

vq = pytest.importorskip("residual_vector_quantization_b200")


def test_bounded_wait_runs_out_and_is_reported():
    assert vq.vq3r_device_error() in (0, 1)  # clear anything earlier
    assert vq.vq3r_device_error() == 0
    t0 = time.perf_counter()
    vq.vq3r_selftest_wait_timeout()
    code = vq.vq3r_device_error()  # synchronises, reads and clears
    dt = time.perf_counter() - t0
    assert code == 1, code
    assert 0.9 < dt < 60.0, dt
    assert vq.vq3r_device_error() == 0
    # the context is still usable: a small encode is bit-exact against the oracle
    rng = np.random.default_rng(3)
    W = rng.standard_normal((64, 256)).astype(np.float32)
    cb = random_codebooks(3)
    idx_t, sc_t = vq.vq3r_encode(torch.from_numpy(W).cuda(), torch.from_numpy(cb).cuda())
    idx_o, sc_o = oracle.encode(W, "f32", cb)
    np.testing.assert_array_equal(idx_t.cpu().numpy(), idx_o)
    np.testing.assert_array_equal(sc_t.cpu().numpy().view(np.uint16), sc_o)
    assert vq.vq3r_device_error() == 0
