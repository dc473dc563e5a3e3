"""Helpers of the GPU parity tests: the selection check over every row and the output
comparison, both against the fp64 oracle.

Selection rule: the library's block indices must equal the oracle's bit for bit.
Only rows where the oracle's last kept and first dropped past scores differ by
less than 1e-5 relative (`oracle.near_tie`) may differ; every such excused row is
counted, printed and bounded (at most EXCUSE_FRAC of the rows checked), and its
outputs are re-checked with the oracle's selection injected by the caller.
Output bar (bf16 I/O): max-abs 2e-2, mean-abs 2e-3, lse max-abs 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3
EXCUSE_FRAC = 1e-4


def sample_rows(B, Hq, N, bs, topk, per_head=256, seed=0):
    """Seeded rows per (b, hq): random tokens plus block edges, the first and last block
    and the rows with c <= k - 1."""
    rng = np.random.default_rng(seed)
    special = {0, N - 1, min(bs - 1, N - 1), min(bs, N - 1), min((topk - 1) * bs, N - 1),
               min(topk * bs, N - 1), min(max(topk * bs - 1, 0), N - 1), N // 2}
    rows = []
    for b in range(B):
        for h in range(Hq):
            ts = set(rng.integers(0, N, size=min(per_head, N)).tolist()) | special
            rows += [(b, h, t) for t in sorted(ts)]
    return np.array(rows, dtype=np.int64)


def stratified_rows(B, Hq, N, bs, per_block, seed=0):
    """Seeded rows covering every block of every head: the first and last token of each
    block plus `per_block` random tokens inside it."""
    rng = np.random.default_rng(seed)
    nblk = (N + bs - 1) // bs
    rows = []
    for b in range(B):
        for h in range(Hq):
            starts = np.arange(nblk, dtype=np.int64) * bs
            ends = np.minimum(starts + bs, N) - 1
            rnd = starts[:, None] + (rng.random((nblk, per_block)) * (ends - starts + 1)[:, None]).astype(np.int64)
            ts = np.unique(np.concatenate([starts, ends, rnd.ravel()]))
            rows.append(np.stack([np.full(ts.size, b), np.full(ts.size, h), ts], axis=1))
    return np.ascontiguousarray(np.concatenate(rows).astype(np.int64))


class SelectionReport:
    """Counts of one selection comparison (rows checked, oracle near ties, excused rows)."""

    def __init__(self, what):
        self.what = what
        self.rows = 0
        self.near_ties = 0
        self.excused = 0

    def add(self, gsel, sel, s_last, s_next, exact_ties_strict=False):
        """Compare one batch of rows; returns the boolean mask of excused rows."""
        tie = oracle.near_tie(s_last, s_next)
        if exact_ties_strict:  # equal scores must follow the lower-index rule exactly
            tie &= ~(s_last == s_next)
        mism = (np.asarray(gsel) != sel).any(axis=1)
        bad = mism & ~tie
        assert not bad.any(), (f"{self.what}: {int(bad.sum())} selection mismatches outside near ties, "
                               f"first at batch row {int(np.argmax(bad))}")
        self.rows += len(sel)
        self.near_ties += int(tie.sum())
        self.excused += int(mism.sum())
        return mism

    def finish(self):
        bound = int(EXCUSE_FRAC * self.rows)
        print(f"[selection] {self.what}: {self.rows} rows checked, {self.near_ties} oracle near ties, "
              f"{self.excused} excused mismatches (bound {bound})", flush=True)
        assert self.excused <= bound, (self.what, self.excused, bound)
        return self


def check_selection_all_rows(idx_dev, q_h, k_h, Hkv, bs, topk, what, exact_ties_strict=False, pooling="mean",
                             weights=None):
    """Every row of the device selection idx [B, Hq, N, topk] against the oracle, one head
    at a time (the oracle pools K once, with the given pooling)."""
    B, N, Hq, _ = q_h.shape
    kbar = oracle.pool(k_h, bs, pooling, weights)
    rep = SelectionReport(what + " (all rows)")
    t = np.arange(N, dtype=np.int64)
    for b in range(B):
        for h in range(Hq):
            rows = np.ascontiguousarray(np.stack([np.full(N, b), np.full(N, h), t], axis=1))
            sel, s_last, s_next = oracle.select(q_h, kbar, Hkv, bs, topk, rows)
            gsel = idx_dev[b, h].cpu().numpy()
            rep.add(gsel, sel, s_last, s_next, exact_ties_strict)
    return rep.finish()


def gather_rows(out, lse, rows):
    """Device out [B, N, Hq, d] / lse [B, Hq, N] at the listed (b, hq, t) rows, as numpy."""
    rt = torch.as_tensor(rows, device=out.device)
    o = out[rt[:, 0], rt[:, 2], rt[:, 1]].float().cpu().numpy()
    l = lse[rt[:, 0], rt[:, 1], rt[:, 2]].cpu().numpy()
    return o, l


def gather_idx(idx, rows):
    rt = torch.as_tensor(rows, device=idx.device)
    return idx[rt[:, 0], rt[:, 1], rt[:, 2]].cpu().numpy()


def compare_outputs(out, lse, ref_out, ref_lse, what=""):
    err = np.abs(out.astype(np.float64) - ref_out)
    lerr = np.abs(lse.astype(np.float64) - ref_lse)
    assert np.isfinite(out).all() and np.isfinite(lse).all(), what
    if err.size:
        assert err.max() <= OUT_MAX, (what, err.max())
        assert err.mean() <= OUT_MEAN, (what, err.mean())
        assert lerr.max() <= LSE_MAX, (what, lerr.max())
        return float(err.max()), float(err.mean()), float(lerr.max())
    return 0.0, 0.0, 0.0
