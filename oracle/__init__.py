"""fp64 CPU oracle of the MoBA causal prefill forward (ctypes wrapper of oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may use it; the product path never does. It shares no code with
the CUDA library. `oracle.c` lists each step with the page passage it follows.

Inputs are host bf16 torch tensors in the [B, N, H, d] layout; results are
float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, OpenMP, no FP contraction)."""
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
            lib.oracle_pool.restype = None
            lib.oracle_pool.argtypes = [_P, _I, _I, _I, _I, _I, _P]
            lib.oracle_pool_mode.restype = None
            lib.oracle_pool_mode.argtypes = [_P, _I, _I, _I, _I, _I, _I, _P, _P]
            lib.oracle_backward.restype = _I
            lib.oracle_backward.argtypes = [_P, _P, _P, _P] + [_I] * 7 + [_P, _P, _P, _P]
            lib.oracle_select.restype = None
            lib.oracle_select.argtypes = [_P, _P] + [_I] * 7 + [_P, _I, _P, _P, _P, _P, _I]
            lib.oracle_attend.restype = _I
            lib.oracle_attend.argtypes = [_P, _P, _P] + [_I] * 7 + [_P, _I, _P, _P, _P]
            lib.oracle_attend_blockwise.restype = _I
            lib.oracle_attend_blockwise.argtypes = [_P, _P, _P] + [_I] * 7 + [_P, _I, _P, _P, _P]
            _lib = lib
    return _lib


def _ptr(a):
    if isinstance(a, torch.Tensor):
        assert a.device.type == "cpu" and a.is_contiguous()
        return a.data_ptr()
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _check_bf16(*ts):
    for t in ts:
        assert isinstance(t, torch.Tensor) and t.dtype == torch.bfloat16 and t.device.type == "cpu"
        assert t.is_contiguous() and t.dim() == 4


def all_rows(B: int, Hq: int, N: int) -> np.ndarray:
    """Every (b, hq, t) triple, b-major then head then token."""
    b, h, t = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(N), indexing="ij")
    return np.ascontiguousarray(np.stack([b.ravel(), h.ravel(), t.ravel()], axis=1).astype(np.int64))


POOLINGS = {"mean": 0, "max": 1, "weighted": 2}


def pool(k: torch.Tensor, block_size: int, pooling: str = "mean", weights=None) -> np.ndarray:
    """Kbar [B, Hkv, N // block_size, d] in fp64: the mean of each full key block (default), the
    feature-wise maximum ("max"), or the weighted mean with one weight per position inside a
    block ("weighted", weights: block_size non-negative numbers with a positive sum)."""
    _check_bf16(k)
    B, N, Hkv, d = k.shape
    nfull = N // block_size
    kbar = np.zeros((B, Hkv, max(nfull, 1), d), dtype=np.float64)
    mode = POOLINGS[pooling]
    if mode == 0:
        _load().oracle_pool(_ptr(k), B, N, Hkv, d, block_size, _ptr(kbar))
    else:
        w = np.zeros(1) if weights is None else np.ascontiguousarray(weights, dtype=np.float64)
        if mode == 2:
            assert w.shape == (block_size,) and (w >= 0).all() and w.sum() > 0
        _load().oracle_pool_mode(_ptr(k), B, N, Hkv, d, block_size, mode, _ptr(w), _ptr(kbar))
    return kbar[:, :, :nfull]


def select(q: torch.Tensor, kbar: np.ndarray, Hkv: int, block_size: int, topk: int, rows: np.ndarray,
           want_scores: bool = False):
    """Selection of each row: (sel int32 [R, topk], s_last, s_next[, scores])."""
    _check_bf16(q)
    B, N, Hq, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    R = rows.shape[0]
    nfull = N // block_size
    kb = np.ascontiguousarray(kbar if kbar.shape[2] > 0 else np.zeros((B, Hkv, 1, d)), dtype=np.float64)
    sel = np.empty((R, topk), dtype=np.int32)
    s_last = np.empty(R, dtype=np.float64)
    s_next = np.empty(R, dtype=np.float64)
    max_past = max(nfull, 1)
    scores = np.empty((R, max_past), dtype=np.float64) if want_scores else None
    _load().oracle_select(_ptr(q), _ptr(kb), B, N, Hq, Hkv, d, block_size, topk, _ptr(rows), R,
                          _ptr(sel), _ptr(s_last), _ptr(s_next),
                          _ptr(scores) if want_scores else None, max_past)
    if want_scores:
        return sel, s_last, s_next, scores
    return sel, s_last, s_next


def attend(q, k, v, block_size: int, topk: int, rows: np.ndarray, sel: np.ndarray, blockwise: bool = False):
    """(out [R, d], lse [R]) in fp64 for the rows with the given selection."""
    _check_bf16(q, k, v)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    R = rows.shape[0]
    assert sel.shape == (R, topk)
    out = np.zeros((R, d), dtype=np.float64)
    lse = np.full(R, np.nan, dtype=np.float64)
    fn = _load().oracle_attend_blockwise if blockwise else _load().oracle_attend
    bad = fn(_ptr(q), _ptr(k), _ptr(v), B, N, Hq, Hkv, d, block_size, topk, _ptr(rows), R, _ptr(sel),
             _ptr(out), _ptr(lse))
    if bad:
        raise ValueError(f"{bad} rows name a future block, repeat a block or lack their own block")
    return out, lse


def forward(q, k, v, block_size: int, topk: int, rows: np.ndarray | None = None, pooling: str = "mean",
            weights=None):
    """The whole method for the given rows (all rows by default).

    Returns a dict with sel, s_last, s_next, out, lse (rows in the order given)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if rows is None:
        rows = all_rows(B, Hq, N)
    kbar = pool(k, block_size, pooling, weights)
    sel, s_last, s_next = select(q, kbar, Hkv, block_size, topk, rows)
    out, lse = attend(q, k, v, block_size, topk, rows, sel)
    return {"rows": rows, "sel": sel, "s_last": s_last, "s_next": s_next, "out": out, "lse": lse}


def backward(q, k, v, dout, block_size: int, topk: int, sel=None, pooling: str = "mean", weights=None):
    """Gradients of sum(dout * out) through the forward with its selection held fixed (the top-k
    choice is discrete: the block summaries get no gradient). sel: int32 [B, Hq, N, topk] for every
    row (computed by the oracle's gate when None). Returns (dq [B, N, Hq, d], dk, dv [B, N, Hkv, d])
    as float64 numpy arrays."""
    _check_bf16(q, k, v, dout)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if sel is None:
        rows = all_rows(B, Hq, N)
        s, _, _ = select(q, pool(k, block_size, pooling, weights), Hkv, block_size, topk, rows)
        sel = s.reshape(B, Hq, N, topk)
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    assert sel.shape == (B, Hq, N, topk)
    dq = np.zeros((B, N, Hq, d))
    dk = np.zeros((B, N, Hkv, d))
    dv = np.zeros((B, N, Hkv, d))
    bad = _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, N, Hq, Hkv, d, block_size, topk,
                                  _ptr(sel), _ptr(dq), _ptr(dk), _ptr(dv))
    if bad:
        raise ValueError(f"{bad} rows name a future block, repeat a block or lack their own block")
    return dq, dk, dv


def forward_varlen(q, k, v, cu_seqlens, block_size: int, topk: int, pooling: str = "mean", weights=None):
    """Packed sequences: q [total, Hq, d], k, v [total, Hkv, d], sequence s holding tokens
    cu_seqlens[s] .. cu_seqlens[s+1] - 1. Reading: each sequence is its own context (its blocks start
    at its first token; no query reads another sequence's keys), so the method is applied to each
    sequence on its own. Returns sel [Hq, total, topk], out [total, Hq, d], lse [Hq, total]."""
    _check_bf16(q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0))
    total, Hq, d = q.shape
    sel = np.full((Hq, total, topk), -1, dtype=np.int32)
    out = np.zeros((total, Hq, d))
    lse = np.zeros((Hq, total))
    cu = [int(x) for x in cu_seqlens]
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b <= a:
            continue
        r = forward(q[a:b].unsqueeze(0).contiguous(), k[a:b].unsqueeze(0).contiguous(),
                    v[a:b].unsqueeze(0).contiguous(), block_size, topk, pooling=pooling, weights=weights)
        rows = r["rows"]
        sel[rows[:, 1], a + rows[:, 2]] = r["sel"]
        out[a + rows[:, 2], rows[:, 1]] = r["out"]
        lse[rows[:, 1], a + rows[:, 2]] = r["lse"]
    return {"sel": sel, "out": out, "lse": lse}


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_size: int, topk: int, length: int,
           pooling: str = "mean", weights=None, full_attention: bool = False):
    """One decode step: the query q [B, Hq, d] is the token at position length - 1 of each sequence,
    attending its KV cache k, v [B, >= length, Hkv, d] (keys 0 .. length - 1). It is the prefill
    definition at that row (the gate, its causal rules and the attention of the pages), so the oracle
    evaluates row length - 1 of a prefill whose query tensor holds q there. full_attention: every
    earlier block is kept (the full-attention decode of a hybrid model).

    Returns a dict with sel [B * Hq, topk], s_last, s_next, out [B * Hq, d], lse [B * Hq]
    (rows b-major, then head)."""
    _check_bf16(k, v)
    B, Hq, d = q.shape
    Hkv = k.shape[2]
    L = int(length)
    kk = k[:, :L].contiguous()
    vv = v[:, :L].contiguous()
    qf = torch.zeros((B, L, Hq, d), dtype=torch.bfloat16)
    qf[:, L - 1] = q
    rows = np.ascontiguousarray(np.stack(np.meshgrid(np.arange(B), np.arange(Hq), indexing="ij"), -1)
                                .reshape(-1, 2))
    rows = np.ascontiguousarray(np.concatenate([rows, np.full((len(rows), 1), L - 1)], 1).astype(np.int64))
    nblk = (L + block_size - 1) // block_size
    kk_top = nblk if full_attention else topk
    kbar = pool(kk, block_size, pooling, weights)
    sel, s_last, s_next = select(qf, kbar, Hkv, block_size, kk_top, rows)
    out, lse = attend(qf, kk, vv, block_size, kk_top, rows, sel)
    return {"rows": rows, "sel": sel, "s_last": s_last, "s_next": s_next, "out": out, "lse": lse}


def near_tie(s_last: np.ndarray, s_next: np.ndarray, rel: float = 1e-5) -> np.ndarray:
    """Rows whose boundary is a near tie: the last selected and the first unselected past
    scores differ by less than `rel` relative to the larger magnitude of the two,
    |s_last - s_next| < rel * max(|s_last|, |s_next|). Equal scores (zero included) differ
    by nothing and count as a tie. Rows without a boundary (every past block selected, so
    both scores are NaN, or nothing selected by score, so s_last is NaN) are never ties.

    This is the exemption rule of the selection check: only at such rows may another
    implementation's selection differ from the oracle's, because the order of two
    scores that close depends on rounding."""
    s_last = np.asarray(s_last, dtype=np.float64)
    s_next = np.asarray(s_next, dtype=np.float64)
    a = np.abs(s_last - s_next)
    m = np.maximum(np.abs(s_last), np.abs(s_next))
    with np.errstate(invalid="ignore"):
        tie = (a < rel * m) | (a == 0)
    return tie & np.isfinite(s_last) & np.isfinite(s_next)
