"""moba_gate_noalloc: the gate for callers that cannot allocate device memory during a call
(serving engines that pre-plan all of HBM, fixed-budget embedders). Its scratch is a fixed array
inside the library, so this test checks, through the C ABI, that two calls in a row give the same
selection as moba_gate (selections are integers: exact equality), and that sizes over the array's
limit are refused. The file sorts last so a failure here cannot hide the other tests."""
import ctypes

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _call(L, fn, q, k, idx, bs, topk):
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    st = torch.cuda.current_stream().cuda_stream
    return getattr(L, fn)(q.data_ptr(), k.data_ptr(), idx.data_ptr(), B, Hq, Hkv, N, d, bs, topk, st)


@pytest.mark.parametrize("first,second", [((2, 8192, 8, 2, 512, 4, 41), (1, 20000, 4, 4, 1000, 6, 42))])
def test_noalloc_gate_matches_gate_on_two_calls(moba, cuda_dev, first, second):
    L = moba.lib()
    for B, N, Hq, Hkv, bs, topk, seed in (first, second):
        q, k, _ = synth.inputs(B, N, Hq, Hkv, 128, bs, seed)
        q, k = q.to(cuda_dev), k.to(cuda_dev)
        want = torch.full((B, Hq, N, topk), -7, dtype=torch.int32, device=cuda_dev)
        got = torch.full_like(want, -7)
        assert _call(L, "moba_gate", q, k, want, bs, topk) == 0
        assert _call(L, "moba_gate_noalloc", q, k, got, bs, topk) == 0
        assert moba.sync_status() == 0
        assert torch.equal(got, want)


def test_noalloc_gate_refuses_sizes_over_its_array(moba, cuda_dev):
    L = moba.lib()
    q = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16, device=cuda_dev)
    idx = torch.zeros(1, 1, 8, 2, dtype=torch.int32, device=cuda_dev)
    # B * Hkv * floor(N / block_size) = 9000 > 8192: refused on the host before any device work
    st = torch.cuda.current_stream().cuda_stream
    assert L.moba_gate_noalloc(q.data_ptr(), q.data_ptr(), idx.data_ptr(), 1, 1, 1, 9000, 128, 1, 2, st) == 2
