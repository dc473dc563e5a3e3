"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects invalid arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moba_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(moba):
    names = _declared()
    assert "moba_forward" in names and "moba_gate" in names
    L = moba.lib()
    for n in names:
        assert hasattr(L, n), n
    assert sorted(moba.EXPORTED) == names


def test_status_strings(moba):
    L = moba.lib()
    for s in range(11):
        assert L.moba_status_string(s).decode() not in ("", "unknown status")
    assert L.moba_status_string(99).decode() == "unknown status"


@pytest.mark.parametrize("args,status", [
    ((1, 1, 1, 4096, 64, 512, 3), 2),     # d != 128
    ((1, 3, 2, 4096, 128, 512, 3), 2),    # Hq not a multiple of Hkv
    ((1, 1, 1, 4096, 128, 512, 0), 2),    # topk < 1
    ((1, 1, 1, 4096, 128, 512, 65), 2),   # topk > 64
    ((1, 1, 1, 0, 128, 512, 3), 2),       # N < 1
    ((1, 1, 1, 1 << 31, 128, 1 << 20, 3), 2),  # N >= 2^31
    ((1, 1, 1, 20000, 128, 1, 3), 2),     # more than 16384 blocks
    ((0, 1, 1, 4096, 128, 512, 3), 2),    # B < 1
])
def test_workspace_size_rejects_bad_shapes(moba, args, status):
    n = ctypes.c_size_t(0)
    assert moba.lib().moba_workspace_size(*args, ctypes.byref(n)) == status


def test_workspace_size_accounts_for_partials(moba):
    n = ctypes.c_size_t(0)
    assert moba.lib().moba_workspace_size(1, 32, 8, 1 << 20, 128, 4096, 12, ctypes.byref(n)) == 0
    partials = 32 * (1 << 20) * 11 * (128 * 2 + 4)
    assert partials < n.value < partials * 1.2


def test_null_and_misaligned_pointers_rejected_on_host(moba):
    L = moba.lib()
    ok = 0x10000
    assert L.moba_forward(None, ok, ok, ok, ok, 1, 1, 1, 4096, 128, 512, 3, None) == 1
    assert L.moba_forward(ok, ok, ok + 8, ok, ok, 1, 1, 1, 4096, 128, 512, 3, None) == 3
    assert L.moba_gate(ok, ok, None, 1, 1, 1, 4096, 128, 512, 3, None) == 1
    assert L.moba_forward_selected(ok, ok, ok, None, ok, ok, 1, 1, 1, 4096, 128, 512, 3, None) == 1
    assert L.moba_forward_ws(ok, ok, ok, ok, ok, 1, 1, 1, 4096, 128, 512, 3, None, 0, None) == 8
    assert L.moba_dense_causal(ok, ok, ok, ok, ok, 1, 1, 1, 4096, 96, None) == 2


def test_no_device_is_an_error_not_a_fallback(moba):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    ok = 0x10000
    st = moba.lib().moba_forward(ok, ok, ok, ok, ok, 1, 1, 1, 4096, 128, 512, 3, None)
    assert st in (4, 5)  # unsupported device / CUDA error: nothing runs on the CPU


def test_binding_refuses_cpu_tensors(moba):
    import torch
    q = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moba.forward(q, q, q, 64, 2)


def test_selftest_wait_timeout_checks_its_limit_on_host(moba):
    L = moba.lib()
    assert L.moba_selftest_wait_timeout(10, None) == 2            # below 1 us
    assert L.moba_selftest_wait_timeout(10 ** 11, None) == 2      # above 10 s
    import torch
    if not torch.cuda.is_available():
        assert L.moba_selftest_wait_timeout(10 ** 6, None) in (4, 5)  # no device: nothing runs


def test_test_hooks_refuse_unknown_values(moba):
    L = moba.lib()
    assert L.moba_set_attention_impl(7) == 2 and L.moba_set_gate_impl(-1) == 2
    assert L.moba_set_attention_impl(0) == 0 and L.moba_set_gate_impl(0) == 0  # previous values
