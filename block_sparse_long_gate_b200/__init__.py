"""MoBA (Mixture of Block Attention) causal prefill forward on B200 (sm_100a).

A thin Python binding over the C ABI of `libmoba.so` (declared in
`include/moba.h`). This module only marshals arguments: it checks tensor
dtypes, shapes and devices, takes device pointers and the current CUDA stream
from PyTorch, and calls the library, where every step of the method runs in
hand-written CUDA kernels. There is no CPU path: without the built library or a
sm_100 device every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import flops  # noqa: F401  (work accounting helpers)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoba.so")

MOBA_OK = 0
STATUS_NAMES = {
    0: "MOBA_OK", 1: "MOBA_ERR_NULL", 2: "MOBA_ERR_SHAPE", 3: "MOBA_ERR_ALIGN", 4: "MOBA_ERR_UNSUPPORTED",
    5: "MOBA_ERR_CUDA", 6: "MOBA_ERR_OOM", 7: "MOBA_ERR_DEVICE_TIMEOUT", 8: "MOBA_ERR_WORKSPACE",
    9: "MOBA_ERR_SELECTION", 10: "MOBA_ERR_VALUE",
}
POOLINGS = {"mean": 0, "max": 1, "weighted": 2}


class Options(ctypes.Structure):
    """moba_options of include/moba.h."""
    _fields_ = [("struct_size", ctypes.c_uint32), ("pooling", ctypes.c_int32), ("pool_weights", ctypes.c_void_p),
                ("full_attention", ctypes.c_int32), ("reserved", ctypes.c_int32)]

EXPORTED = [
    "moba_status_string", "moba_workspace_size", "moba_forward", "moba_forward_ws", "moba_gate",
    "moba_forward_selected", "moba_forward_selected_ws", "moba_dense_causal", "moba_sync_status",
    "moba_set_attention_impl", "moba_set_gate_impl", "moba_stage_timing", "moba_stage_times",
    "moba_launch_count", "moba_gate_noalloc", "moba_last_error_string", "moba_selftest_wait_timeout",
    "moba_forward_ex", "moba_gate_ex", "moba_decode_workspace_size", "moba_pool_cache", "moba_decode",
    "moba_varlen_workspace_size", "moba_forward_varlen", "moba_gate_varlen", "moba_backward_workspace_size",
    "moba_backward",
]
STAGES = ("pool", "gate", "invert", "attention", "merge")


class MobaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = _status_string(status)
        if status == 5:  # MOBA_ERR_CUDA: add the runtime's own message
            try:
                detail += ": " + lib().moba_last_error_string().decode()
            except Exception:
                pass
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({detail})")


_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64


def lib():
    """The loaded libmoba.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libmoba.so is missing at {LIB_PATH}; build it with "
                                   "block_sparse_long_gate_b200.build.build_library()")
            L = ctypes.CDLL(LIB_PATH)
            L.moba_status_string.restype = ctypes.c_char_p
            L.moba_status_string.argtypes = [_I]
            L.moba_workspace_size.restype = _I
            L.moba_workspace_size.argtypes = [_I, _I, _I, _L, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]
            L.moba_forward.restype = _I
            L.moba_forward.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _L, _I, _I, _I, _P]
            L.moba_forward_ws.restype = _I
            L.moba_forward_ws.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _L, _I, _I, _I, _P, ctypes.c_size_t, _P]
            L.moba_gate.restype = _I
            L.moba_gate.argtypes = [_P, _P, _P, _I, _I, _I, _L, _I, _I, _I, _P]
            L.moba_forward_selected.restype = _I
            L.moba_forward_selected.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _L, _I, _I, _I, _P]
            L.moba_forward_selected_ws.restype = _I
            L.moba_forward_selected_ws.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _L, _I, _I, _I, _P,
                                                   ctypes.c_size_t, _P]
            L.moba_dense_causal.restype = _I
            L.moba_dense_causal.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _L, _I, _P]
            L.moba_sync_status.restype = _I
            L.moba_sync_status.argtypes = [_P]
            L.moba_set_attention_impl.restype = _I
            L.moba_set_attention_impl.argtypes = [_I]
            L.moba_set_gate_impl.restype = _I
            L.moba_set_gate_impl.argtypes = [_I]
            L.moba_stage_timing.restype = _I
            L.moba_stage_timing.argtypes = [_I]
            L.moba_stage_times.restype = _I
            L.moba_stage_times.argtypes = [ctypes.POINTER(ctypes.c_float), _I, ctypes.POINTER(ctypes.c_int)]
            L.moba_launch_count.restype = ctypes.c_uint64
            L.moba_launch_count.argtypes = []
            L.moba_last_error_string.restype = ctypes.c_char_p
            L.moba_last_error_string.argtypes = []
            L.moba_selftest_wait_timeout.restype = _I
            L.moba_selftest_wait_timeout.argtypes = [_L, _P]
            L.moba_forward_ex.restype = _I
            L.moba_forward_ex.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _L, _I, _I, _I, ctypes.POINTER(Options), _P,
                                          ctypes.c_size_t, _P]
            L.moba_gate_ex.restype = _I
            L.moba_gate_ex.argtypes = [_P, _P, _P, _I, _I, _I, _L, _I, _I, _I, ctypes.POINTER(Options), _P]
            L.moba_decode_workspace_size.restype = _I
            L.moba_decode_workspace_size.argtypes = [_I, _I, _I, _L, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]
            L.moba_pool_cache.restype = _I
            L.moba_pool_cache.argtypes = [_P, _P, _I, _I, _L, _L, _I, _I, _L, _L, ctypes.POINTER(Options), _P]
            L.moba_decode.restype = _I
            L.moba_decode.argtypes = [_P, _P, _P, _P, _L, _P, _P, _P, _I, _I, _I, _L, _L, _I, _I, _I, _I, _P,
                                      ctypes.c_size_t, _P]
            _LP = ctypes.POINTER(ctypes.c_int64)
            L.moba_varlen_workspace_size.restype = _I
            L.moba_varlen_workspace_size.argtypes = [_LP, _I, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]
            L.moba_forward_varlen.restype = _I
            L.moba_forward_varlen.argtypes = [_P, _P, _P, _P, _P, _LP, _I, _I, _I, _I, _I, _I, ctypes.POINTER(Options),
                                              _P, ctypes.c_size_t, _P]
            L.moba_gate_varlen.restype = _I
            L.moba_gate_varlen.argtypes = [_P, _P, _P, _LP, _I, _I, _I, _I, _I, _I, ctypes.POINTER(Options), _P,
                                           ctypes.c_size_t, _P]
            L.moba_backward_workspace_size.restype = _I
            L.moba_backward_workspace_size.argtypes = [_I, _I, _I, _L, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]
            L.moba_backward.restype = _I
            L.moba_backward.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _L, _I, _I, _I, _P,
                                        ctypes.c_size_t, _P]
            L.moba_gate_noalloc.restype = _I
            L.moba_gate_noalloc.argtypes = [_P, _P, _P, _I, _I, _I, _L, _I, _I, _I, _P]
            _lib = L
    return _lib


def _status_string(status: int) -> str:
    try:
        return lib().moba_status_string(status).decode()
    except Exception:  # library not loadable: fall back to the name table
        return STATUS_NAMES.get(status, "unknown")


def _check(status: int, where: str):
    if status != MOBA_OK:
        raise MobaError(status, where)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _check_qkv(q, k, v=None):
    ts = [q, k] + ([v] if v is not None else [])
    for t in ts:
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
        if t.dim() != 4:
            raise ValueError("q, k, v must have the layout [B, N, H, d]")
    B, N, Hq, d = q.shape
    if k.shape[0] != B or k.shape[1] != N or k.shape[3] != d:
        raise ValueError("k must be [B, N, Hkv, d] matching q")
    if v is not None and v.shape != k.shape:
        raise ValueError("v must have the shape of k")
    return B, N, Hq, k.shape[2], d


def workspace_size(B, Hq, Hkv, N, d, block_size, topk) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moba_workspace_size(B, Hq, Hkv, N, d, block_size, topk, ctypes.byref(n)), "moba_workspace_size")
    return int(n.value)


def options(pooling: str = "mean", pool_weights=None, full_attention: bool = False) -> Options:
    """moba_options for the extended entry points. pool_weights: fp32 CUDA tensor [block_size]."""
    if pooling not in POOLINGS:
        raise ValueError(f"pooling must be one of {sorted(POOLINGS)}")
    if pool_weights is not None and (pool_weights.dtype != torch.float32 or not pool_weights.is_cuda
                                     or not pool_weights.is_contiguous()):
        raise ValueError("pool_weights must be a contiguous fp32 CUDA tensor")
    o = Options()
    o.struct_size = ctypes.sizeof(Options)
    o.pooling = POOLINGS[pooling]
    o.pool_weights = _ptr(pool_weights)
    o.full_attention = 1 if full_attention else 0
    o.reserved = 0
    return o


def forward(q, k, v, block_size: int, topk: int, out=None, lse=None, workspace=None, stream=None,
            pooling: str = "mean", pool_weights=None, full_attention: bool = False):
    """MoBA causal prefill forward. Returns (out bf16 [B, N, Hq, d], lse fp32 [B, Hq, N]).

    pooling / pool_weights choose the gate's block summary ("mean", "max", "weighted"), and
    full_attention=True makes this a full-attention layer of a hybrid model (dense causal)."""
    B, N, Hq, Hkv, d = _check_qkv(q, k, v)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    if pooling != "mean" or full_attention:
        opt = options(pooling, pool_weights, full_attention)
        if workspace is None and not full_attention:
            workspace = torch.empty(workspace_size(B, Hq, Hkv, N, d, block_size, topk), dtype=torch.uint8,
                                    device=q.device)
        _check(lib().moba_forward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d, block_size,
                                     topk, ctypes.byref(opt), _ptr(workspace),
                                     0 if workspace is None else workspace.numel(), _stream(stream)),
               "moba_forward_ex")
        return out, lse
    if workspace is None:
        workspace = torch.empty(workspace_size(B, Hq, Hkv, N, d, block_size, topk), dtype=torch.uint8,
                                device=q.device)
    _check(lib().moba_forward_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d, block_size,
                                 topk, _ptr(workspace), workspace.numel(), _stream(stream)), "moba_forward_ws")
    return out, lse


def gate(q, k, block_size: int, topk: int, idx=None, stream=None, pooling: str = "mean", pool_weights=None):
    """Selected blocks per query: int32 [B, Hq, N, topk], ascending, own block last, -1 padded."""
    B, N, Hq, Hkv, d = _check_qkv(q, k)
    idx = torch.empty((B, Hq, N, topk), dtype=torch.int32, device=q.device) if idx is None else idx
    if pooling != "mean":
        opt = options(pooling, pool_weights)
        _check(lib().moba_gate_ex(_ptr(q), _ptr(k), _ptr(idx), B, Hq, Hkv, N, d, block_size, topk, ctypes.byref(opt),
                                  _stream(stream)), "moba_gate_ex")
        return idx
    _check(lib().moba_gate(_ptr(q), _ptr(k), _ptr(idx), B, Hq, Hkv, N, d, block_size, topk, _stream(stream)),
           "moba_gate")
    return idx


def gate_noalloc(q, k, block_size: int, topk: int, idx=None, stream=None):
    """gate() for callers that cannot allocate device memory during the call: the block means
    live in a fixed 8 MiB array inside the library (B * Hkv * floor(N / block_size) <= 8192).
    Calls that overlap on the GPU race on that array. (The output tensor, when not given, is
    still allocated here by PyTorch; pass `idx` to avoid that too.)"""
    B, N, Hq, Hkv, d = _check_qkv(q, k)
    idx = torch.empty((B, Hq, N, topk), dtype=torch.int32, device=q.device) if idx is None else idx
    _check(lib().moba_gate_noalloc(_ptr(q), _ptr(k), _ptr(idx), B, Hq, Hkv, N, d, block_size, topk,
                                   _stream(stream)), "moba_gate_noalloc")
    return idx


def forward_selected(q, k, v, idx, block_size: int, topk: int, out=None, lse=None, workspace=None, stream=None):
    """Attention with a given selection (same layout as gate()). Returns (out, lse)."""
    B, N, Hq, Hkv, d = _check_qkv(q, k, v)
    if idx.dtype != torch.int32 or not idx.is_cuda or not idx.is_contiguous() or tuple(idx.shape) != (B, Hq, N, topk):
        raise ValueError("idx must be a contiguous int32 CUDA tensor [B, Hq, N, topk]")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    if workspace is None:
        workspace = torch.empty(workspace_size(B, Hq, Hkv, N, d, block_size, topk), dtype=torch.uint8,
                                device=q.device)
    _check(lib().moba_forward_selected_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(out), _ptr(lse), B, Hq, Hkv,
                                          N, d, block_size, topk, _ptr(workspace), workspace.numel(),
                                          _stream(stream)), "moba_forward_selected_ws")
    return out, lse


def _cu_array(cu_seqlens):
    vals = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    return (ctypes.c_int64 * len(vals))(*vals), len(vals) - 1


def varlen_workspace_size(cu_seqlens, Hq, Hkv, d, block_size, topk) -> int:
    arr, nseq = _cu_array(cu_seqlens)
    n = ctypes.c_size_t(0)
    _check(lib().moba_varlen_workspace_size(arr, nseq, Hq, Hkv, d, block_size, topk, ctypes.byref(n)),
           "moba_varlen_workspace_size")
    return int(n.value)


def _check_packed(q, k, v=None):
    for t in [q, k] + ([v] if v is not None else []):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
        if t.dim() != 3:
            raise ValueError("packed q, k, v have the layout [total, H, d]")
    return q.shape[0], q.shape[1], k.shape[1], q.shape[2]


def forward_varlen(q, k, v, cu_seqlens, block_size: int, topk: int, out=None, lse=None, workspace=None,
                   stream=None, pooling: str = "mean", pool_weights=None, full_attention: bool = False):
    """Packed sequences (q [total, Hq, d], k, v [total, Hkv, d], host cu_seqlens). Returns
    (out [total, Hq, d], lse [Hq, total])."""
    total, Hq, Hkv, d = _check_packed(q, k, v)
    arr, nseq = _cu_array(cu_seqlens)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((Hq, total), dtype=torch.float32, device=q.device) if lse is None else lse
    if workspace is None:
        workspace = torch.empty(varlen_workspace_size(cu_seqlens, Hq, Hkv, d, block_size, topk), dtype=torch.uint8,
                                device=q.device)
    opt = options(pooling, pool_weights, full_attention)
    _check(lib().moba_forward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), arr, nseq, Hq, Hkv, d,
                                     block_size, topk, ctypes.byref(opt), _ptr(workspace), workspace.numel(),
                                     _stream(stream)), "moba_forward_varlen")
    return out, lse


def gate_varlen(q, k, cu_seqlens, block_size: int, topk: int, idx=None, workspace=None, stream=None,
                pooling: str = "mean", pool_weights=None):
    """Selected blocks of every packed token: int32 [Hq, total, topk]."""
    total, Hq, Hkv, d = _check_packed(q, k)
    arr, nseq = _cu_array(cu_seqlens)
    idx = torch.empty((Hq, total, topk), dtype=torch.int32, device=q.device) if idx is None else idx
    if workspace is None:
        workspace = torch.empty(varlen_workspace_size(cu_seqlens, Hq, Hkv, d, block_size, topk), dtype=torch.uint8,
                                device=q.device)
    opt = options(pooling, pool_weights)
    _check(lib().moba_gate_varlen(_ptr(q), _ptr(k), _ptr(idx), arr, nseq, Hq, Hkv, d, block_size, topk,
                                  ctypes.byref(opt), _ptr(workspace), workspace.numel(), _stream(stream)),
           "moba_gate_varlen")
    return idx


def decode_workspace_size(B, Hq, Hkv, L, d, block_size, topk, full_attention=False) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moba_decode_workspace_size(B, Hq, Hkv, L, d, block_size, topk, 1 if full_attention else 0,
                                            ctypes.byref(n)), "moba_decode_workspace_size")
    return int(n.value)


def pool_cache(k, block_size: int, length: int, kbar=None, first_block: int = 0, pooling: str = "mean",
               pool_weights=None, stream=None):
    """Block summaries (fp64 [B, Hkv, rows, d]) of the full blocks of a KV cache k [B, Lmax, Hkv, d]
    holding `length` tokens; blocks before first_block are left as they are in `kbar`."""
    if k.dtype != torch.bfloat16 or not k.is_cuda or not k.is_contiguous() or k.dim() != 4:
        raise ValueError("k must be a contiguous bf16 CUDA tensor [B, Lmax, Hkv, d]")
    B, Lmax, Hkv, d = k.shape
    rows = max(length // block_size, 1)
    if kbar is None:
        kbar = torch.zeros((B, Hkv, rows, d), dtype=torch.float64, device=k.device)
    opt = options(pooling, pool_weights)
    _check(lib().moba_pool_cache(_ptr(k), _ptr(kbar), B, Hkv, length, Lmax, d, block_size, kbar.shape[2],
                                 first_block, ctypes.byref(opt), _stream(stream)), "moba_pool_cache")
    return kbar


def decode(q, k, v, kbar, block_size: int, topk: int, length: int, full_attention: bool = False, out=None,
           lse=None, idx=None, workspace=None, stream=None):
    """One decode step: q [B, Hq, d] (the token at position length - 1) against the cache k, v
    [B, Lmax, Hkv, d]. Returns (out [B, Hq, d], lse [B, Hq], idx [B, Hq, topk] or None)."""
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    B, Hq, d = q.shape
    _, Lmax, Hkv, _ = k.shape
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    if idx is None and not full_attention:
        idx = torch.empty((B, Hq, topk), dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = torch.empty(decode_workspace_size(B, Hq, Hkv, length, d, block_size, topk, full_attention),
                                dtype=torch.uint8, device=q.device)
    rows = 0 if kbar is None else kbar.shape[2]
    _check(lib().moba_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(kbar), rows, _ptr(out), _ptr(lse), _ptr(idx), B, Hq,
                             Hkv, length, Lmax, d, block_size, topk, 1 if full_attention else 0, _ptr(workspace),
                             workspace.numel(), _stream(stream)), "moba_decode")
    return out, lse, idx


def backward_workspace_size(B, Hq, Hkv, N, d, block_size, topk) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moba_backward_workspace_size(B, Hq, Hkv, N, d, block_size, topk, ctypes.byref(n)),
           "moba_backward_workspace_size")
    return int(n.value)


def backward(q, k, v, out, lse, dout, block_size: int, topk: int, idx=None, dq=None, dk=None, dv=None,
             workspace=None, stream=None):
    """Gradients (dq, dk, dv) of sum(dout * out) through the forward with its selection held fixed.
    out, lse: the forward's results; idx: the forward's selection (None: the gate runs again)."""
    B, N, Hq, Hkv, d = _check_qkv(q, k, v)
    for t in (out, dout):
        if t.shape != q.shape or t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("out and dout must be contiguous bf16 CUDA tensors shaped like q")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(backward_workspace_size(B, Hq, Hkv, N, d, block_size, topk), dtype=torch.uint8,
                                device=q.device)
    _check(lib().moba_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(idx), _ptr(dq),
                               _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, block_size, topk, _ptr(workspace),
                               workspace.numel(), _stream(stream)), "moba_backward")
    return dq, dk, dv


def dense_causal(q, k, v, out=None, lse=None, stream=None):
    """Dense causal attention of the same shape. Returns (out, lse)."""
    B, N, Hq, Hkv, d = _check_qkv(q, k, v)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(lib().moba_dense_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d,
                                   _stream(stream)), "moba_dense_causal")
    return out, lse


def sync_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the library's device error flag."""
    return int(lib().moba_sync_status(_stream(stream)))


def selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Queue the bounded-wait self-test (a wait on a barrier nothing completes, given up
    after limit_ns); the timeout shows up in the next sync_status()."""
    _check(lib().moba_selftest_wait_timeout(int(limit_ns), _stream(stream)), "moba_selftest_wait_timeout")


def check_status(stream=None):
    _check(sync_status(stream), "device")


def set_attention_impl(impl: int) -> int:
    return int(lib().moba_set_attention_impl(impl))


def set_gate_impl(impl: int) -> int:
    return int(lib().moba_set_gate_impl(impl))


def stage_timing(enable: bool) -> bool:
    """Record CUDA events between the stages of every forward call (for measurement)."""
    return bool(lib().moba_stage_timing(1 if enable else 0))


def stage_times() -> tuple[dict, int]:
    """({stage: ms summed over the recorded calls}, number of calls); clears the records."""
    arr = (ctypes.c_float * len(STAGES))()
    calls = ctypes.c_int(0)
    _check(lib().moba_stage_times(arr, len(STAGES), ctypes.byref(calls)), "moba_stage_times")
    return {name: float(arr[i]) for i, name in enumerate(STAGES)}, int(calls.value)


def launch_count() -> int:
    """Kernels launched by libmoba so far in this process."""
    return int(lib().moba_launch_count())
