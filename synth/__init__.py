"""Seeded synthetic inputs shared by the oracle tests and the GPU harness.

Only random numbers live here (splitmix64 counters, Box-Muller normals, one
round-to-nearest-even to bfloat16); none of the attention method's arithmetic.
The C source `synth.c` states the exact definition. Shapes follow the MoBA
pages' workloads: Q, V ~ N(0,1) and K = N(0,1) + c[b, h, j] with a per key
block offset c ~ N(0, 0.5^2), all bf16 in the [B, N, H, d] layout.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

Q_ID, K_ID, V_ID, KOFF_ID = 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.synth_stream_key.restype = ctypes.c_uint64
            lib.synth_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
            lib.synth_normal_at.restype = ctypes.c_double
            lib.synth_normal_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
            lib.synth_bf16_rne.restype = ctypes.c_uint16
            lib.synth_bf16_rne.argtypes = [ctypes.c_double]
            lib.synth_fill_normal.restype = None
            lib.synth_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                              ctypes.c_int64]
            lib.synth_key_offset.restype = ctypes.c_double
            lib.synth_key_offset.argtypes = [ctypes.c_uint64] + [ctypes.c_int64] * 5
            lib.synth_fill_keys.restype = None
            lib.synth_fill_keys.argtypes = [ctypes.c_void_p, ctypes.c_uint64] + [ctypes.c_int64] * 5
            lib.synth_fill_normal_heads.restype = None
            lib.synth_fill_normal_heads.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32] + \
                [ctypes.c_int64] * 6
            lib.synth_fill_keys_heads.restype = None
            lib.synth_fill_keys_heads.argtypes = [ctypes.c_void_p, ctypes.c_uint64] + [ctypes.c_int64] * 7
            _lib = lib
    return _lib


def lib():
    return _load()


def _empty(shape, pin: bool) -> torch.Tensor:
    return torch.empty(shape, dtype=torch.bfloat16, pin_memory=pin)


def normal(seed: int, tensor_id: int, shape, pin: bool = False) -> torch.Tensor:
    """bf16 tensor of N(0,1) numbers of stream (seed, tensor_id), element i = flat index i."""
    t = _empty(shape, pin)
    _load().synth_fill_normal(t.data_ptr(), seed, tensor_id, t.numel())
    return t


def keys(seed: int, B: int, N: int, Hkv: int, d: int, block_size: int, pin: bool = False) -> torch.Tensor:
    """bf16 K [B, N, Hkv, d] = N(0,1) + per (b, h, key block) offset N(0, 0.5^2)."""
    t = _empty((B, N, Hkv, d), pin)
    _load().synth_fill_keys(t.data_ptr(), seed, B, N, Hkv, d, block_size)
    return t


def inputs(B: int, N: int, Hq: int, Hkv: int, d: int, block_size: int, seed: int, pin: bool = False):
    """(q, k, v) on the host, bf16, layout [B, N, H, d]."""
    q = normal(seed, Q_ID, (B, N, Hq, d), pin)
    k = keys(seed, B, N, Hkv, d, block_size, pin)
    v = normal(seed, V_ID, (B, N, Hkv, d), pin)
    return q, k, v


def inputs_heads(B: int, N: int, Hq: int, Hkv: int, d: int, block_size: int, seed: int, hkv0: int, hkv1: int,
                 pin: bool = False):
    """The slice of `inputs(...)` a rank owning kv heads [hkv0, hkv1) needs: q of query heads
    [hkv0 * G, hkv1 * G) (G = Hq / Hkv) and k, v of kv heads [hkv0, hkv1), each contiguous and
    equal element for element to that slice of the whole tensors."""
    G = Hq // Hkv
    L = _load()
    q = _empty((B, N, (hkv1 - hkv0) * G, d), pin)
    L.synth_fill_normal_heads(q.data_ptr(), seed, Q_ID, B, N, Hq, d, hkv0 * G, hkv1 * G)
    k = _empty((B, N, hkv1 - hkv0, d), pin)
    L.synth_fill_keys_heads(k.data_ptr(), seed, B, N, Hkv, d, block_size, hkv0, hkv1)
    v = _empty((B, N, hkv1 - hkv0, d), pin)
    L.synth_fill_normal_heads(v.data_ptr(), seed, V_ID, B, N, Hkv, d, hkv0, hkv1)
    return q, k, v


def bf16_rne(x: float) -> int:
    """bf16 bit pattern of x rounded to nearest even (the module's one rounding step)."""
    return int(_load().synth_bf16_rne(float(x)))


def normal_at(seed: int, tensor_id: int, i: int) -> float:
    """Number i of stream (seed, tensor_id) in double precision, before rounding."""
    L = _load()
    return float(L.synth_normal_at(L.synth_stream_key(seed, tensor_id), i))


def key_offset(seed: int, b: int, h: int, j: int, Hkv: int, nblk: int) -> float:
    return float(_load().synth_key_offset(seed, b, h, j, Hkv, nblk))
