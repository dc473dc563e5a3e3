"""Failure detection on the GPU without a GPU fault: a bounded wait on a barrier that nothing
completes gives up after its wall-clock limit, the device error flag reports
MOBA_ERR_DEVICE_TIMEOUT to the host, and the context stays usable for the next forward."""
import time

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

MOBA_ERR_DEVICE_TIMEOUT = 7


def test_bounded_wait_times_out_and_context_survives(moba, cuda_dev):
    assert moba.sync_status() == 0
    t0 = time.perf_counter()
    moba.selftest_wait_timeout(50_000_000)  # 50 ms
    status = moba.sync_status()
    dt = time.perf_counter() - t0
    assert status == MOBA_ERR_DEVICE_TIMEOUT
    assert 0.04 < dt < 10.0, dt
    assert moba.sync_status() == 0  # the flag was cleared by the read
    q, k, v = (t.to(cuda_dev) for t in synth.inputs(1, 1024, 2, 1, 128, 256, 11))
    out, lse = moba.forward(q, k, v, 256, 3)
    assert moba.sync_status() == 0
    assert bool(torch.isfinite(out.float()).all()) and bool(torch.isfinite(lse).all())
