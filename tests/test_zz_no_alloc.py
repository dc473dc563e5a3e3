"""moba_gate_noalloc: the gate for callers that cannot allocate device memory during a call
(serving engines that pre-plan all of HBM, fixed-budget embedders). Its scratch is a fixed array
inside the library, so this test checks, through the C ABI:
  - two calls in a row give the same selection as moba_gate (selections are integers: exact
    equality), also at the array's exact limit with a ragged last block;
  - a call takes nothing from the device's stream-ordered memory pool (the pool moba_gate's
    own scratch comes from, used here as the positive control) and leaves free memory unchanged;
  - sizes one row over the array's limit are refused on the host.
The file sorts last so a failure here cannot hide the other tests."""
import ctypes

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

LIMIT_ROWS = 8192  # B * Hkv * floor(N / block_size) the library's fixed array holds


def _call(L, fn, q, k, idx, bs, topk):
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    st = torch.cuda.current_stream().cuda_stream
    return getattr(L, fn)(q.data_ptr(), k.data_ptr(), idx.data_ptr(), B, Hq, Hkv, N, d, bs, topk, st)


class _DefaultPool:
    """Used-bytes counters of the device's default stream-ordered memory pool (driver API)."""

    USED_MEM_CURRENT, USED_MEM_HIGH = 7, 8  # CUmemPool_attribute values

    def __init__(self, device_index):
        self.cu = ctypes.CDLL("libcuda.so.1")
        assert self.cu.cuInit(0) == 0
        dev = ctypes.c_int(0)
        assert self.cu.cuDeviceGet(ctypes.byref(dev), device_index) == 0
        self.pool = ctypes.c_void_p(0)
        assert self.cu.cuDeviceGetDefaultMemPool(ctypes.byref(self.pool), dev) == 0

    def get(self, attr):
        v = ctypes.c_uint64(0)
        assert self.cu.cuMemPoolGetAttribute(self.pool, attr, ctypes.byref(v)) == 0
        return int(v.value)

    def reset_high(self):
        z = ctypes.c_uint64(0)
        assert self.cu.cuMemPoolSetAttribute(self.pool, self.USED_MEM_HIGH, ctypes.byref(z)) == 0


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


def test_noalloc_gate_at_its_limit_with_a_ragged_last_block(moba, cuda_dev):
    """B * Hkv * floor(N / bs) == 8192 exactly, N % bs != 0 (the last block is never pooled)."""
    L = moba.lib()
    B, Hq, Hkv, bs, topk = 1, 4, 2, 64, 5
    N = (LIMIT_ROWS // Hkv) * bs + 37
    assert B * Hkv * (N // bs) == LIMIT_ROWS
    q, k, _ = synth.inputs(B, N, Hq, Hkv, 128, bs, 43)
    q, k = q.to(cuda_dev), k.to(cuda_dev)
    want = torch.full((B, Hq, N, topk), -7, dtype=torch.int32, device=cuda_dev)
    assert _call(L, "moba_gate", q, k, want, bs, topk) == 0
    for _ in range(2):
        got = torch.full_like(want, -7)
        assert _call(L, "moba_gate_noalloc", q, k, got, bs, topk) == 0
        assert moba.sync_status() == 0
        assert torch.equal(got, want)


def test_noalloc_gate_allocates_nothing(moba, cuda_dev):
    L = moba.lib()
    B, N, Hq, Hkv, bs, topk = 1, 16384, 4, 2, 256, 6
    q, k, _ = synth.inputs(B, N, Hq, Hkv, 128, bs, 44)
    q, k = q.to(cuda_dev), k.to(cuda_dev)
    idx = torch.empty((B, Hq, N, topk), dtype=torch.int32, device=cuda_dev)
    # first call: the one-time address lookup happens here, outside the measured calls
    assert _call(L, "moba_gate_noalloc", q, k, idx, bs, topk) == 0
    assert moba.sync_status() == 0
    pool = _DefaultPool(cuda_dev.index or 0)

    # positive control: moba_gate takes its scratch from this pool
    torch.cuda.synchronize()
    pool.reset_high()
    base = pool.get(pool.USED_MEM_CURRENT)
    assert _call(L, "moba_gate", q, k, idx, bs, topk) == 0
    assert moba.sync_status() == 0
    assert pool.get(pool.USED_MEM_HIGH) > base

    torch.cuda.synchronize()
    pool.reset_high()
    base = pool.get(pool.USED_MEM_CURRENT)
    free0, _ = torch.cuda.mem_get_info(cuda_dev)
    torch_bytes0 = torch.cuda.memory_allocated(cuda_dev)
    for _ in range(2):
        assert _call(L, "moba_gate_noalloc", q, k, idx, bs, topk) == 0
    assert moba.sync_status() == 0
    assert pool.get(pool.USED_MEM_HIGH) == base
    assert pool.get(pool.USED_MEM_CURRENT) == base
    free1, _ = torch.cuda.mem_get_info(cuda_dev)
    assert free1 == free0
    assert torch.cuda.memory_allocated(cuda_dev) == torch_bytes0


def test_noalloc_gate_refuses_sizes_over_its_array(moba, cuda_dev):
    L = moba.lib()
    q = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16, device=cuda_dev)
    idx = torch.zeros(1, 1, 8, 2, dtype=torch.int32, device=cuda_dev)
    st = torch.cuda.current_stream().cuda_stream
    # B * Hkv * floor(N / block_size): 8193 and 9000 > 8192 are refused on the host before any
    # device work (the pointers are never read)
    assert L.moba_gate_noalloc(q.data_ptr(), q.data_ptr(), idx.data_ptr(), 1, 1, 1, 8193, 128, 1, 2, st) == 2
    assert L.moba_gate_noalloc(q.data_ptr(), q.data_ptr(), idx.data_ptr(), 1, 1, 1, 9000, 128, 1, 2, st) == 2
    assert L.moba_gate_noalloc(q.data_ptr(), q.data_ptr(), idx.data_ptr(), 1, 3, 3, 2732 * 64, 128, 64, 2,
                               st) == 2  # Hkv = 3: 3 * 2732 = 8196
