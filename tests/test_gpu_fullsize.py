"""GPU parity at the full sizes of the long-context workloads, in the launch path the
benchmark times (moba_forward_ws with a caller workspace).

Selection: at 128K, 512K and 1M tokens EVERY row's block indices are compared with the
fp64 oracle's (one head at a time); at 10M tokens a seeded stratified sample of about
10^6 rows covering every block (its first and last token plus random ones). Outputs: a
seeded sample of rows (every head, random tokens plus block edges) element by element
against the oracle, with the same near-tie / tolerance rules as the small cases. On
every row, properties that hold at any size:
  - each selection row is well formed: ascending distinct earlier blocks, then the row's
    own block, then -1 padding, with min(k, c + 1) entries;
  - out and lse are finite everywhere.
"""
import gc

import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import (SelectionReport, check_selection_all_rows, compare_outputs, gather_idx,
                         gather_rows, sample_rows, stratified_rows)

pytestmark = pytest.mark.gpu

LONG = [  # B, N, Hq, Hkv, block_size, topk, seed, sampled output rows per head, selection rows
    (1, 131072, 32, 8, 4096, 12, 3, 24, "all"),     # Llama-3.1-8B attention shape at 128K
    (1, 524288, 32, 8, 4096, 12, 3, 12, "all"),     # ... at 512K
    (1, 1048576, 32, 8, 4096, 12, 3, 8, "all"),     # ... at 1M (the benchmark's workload)
    (1, 10485760, 1, 1, 4096, 12, 4, 256, 420),     # 10M tokens, one head: 420 random rows per block
]


def _well_formed(idx, N, bs, topk):
    """Device-side check of every selection row (see the module docstring)."""
    B, H, n, k = idx.shape
    t = torch.arange(n, device=idx.device, dtype=torch.int64)
    c = (t // bs).view(1, 1, n)
    cnt = torch.clamp(c + 1, max=topk)                        # entries a row must hold
    valid = idx >= 0
    assert torch.equal(valid.sum(-1), cnt.expand(B, H, n)), "entry count"
    pos = torch.arange(k, device=idx.device).view(1, 1, 1, k)
    assert bool((valid == (pos < cnt.unsqueeze(-1))).all()), "-1 padding only at the end"
    last = idx.gather(-1, (cnt - 1).unsqueeze(-1).expand(B, H, n, 1)).squeeze(-1)
    assert torch.equal(last.long(), c.expand(B, H, n)), "own block last"
    inc = (idx[..., 1:] > idx[..., :-1]) | ~valid[..., 1:]
    assert bool(inc.all()), "ascending distinct"


@pytest.mark.parametrize("case", LONG, ids=lambda c: f"N{c[1]}_H{c[2]}")
def test_long_context(moba, cuda_dev, case):
    B, N, Hq, Hkv, bs, topk, seed, per_head, sel_rows = case
    gc.collect()
    torch.cuda.empty_cache()  # blocks cached by earlier cases count as used in mem_get_info
    free, _ = torch.cuda.mem_get_info(cuda_dev)
    need = moba.workspace_size(B, Hq, Hkv, N, 128, bs, topk) + 3 * B * N * Hq * 128 * 2 + (4 << 30)
    if free < need:
        pytest.skip(f"needs {need / 2**30:.0f} GiB of device memory, {free / 2**30:.0f} GiB free")
    q_h, k_h, v_h = synth.inputs(B, N, Hq, Hkv, 128, bs, seed)
    q, k, v = q_h.to(cuda_dev), k_h.to(cuda_dev), v_h.to(cuda_dev)
    ws = torch.empty(moba.workspace_size(B, Hq, Hkv, N, 128, bs, topk), dtype=torch.uint8, device=cuda_dev)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device=cuda_dev)
    moba.forward(q, k, v, bs, topk, out=out, lse=lse, workspace=ws)
    idx = moba.gate(q, k, bs, topk)
    assert moba.sync_status() == 0
    del ws
    _well_formed(idx, N, bs, topk)
    assert bool(torch.isfinite(lse).all()) and bool(torch.isfinite(out).all())

    what = f"N={N} Hq={Hq} Hkv={Hkv} bs={bs} k={topk}"
    kbar = oracle.pool(k_h, bs)
    if sel_rows == "all":
        check_selection_all_rows(idx, q_h, k_h, Hkv, bs, topk, what)
    else:
        srows = stratified_rows(B, Hq, N, bs, sel_rows, seed)
        rep = SelectionReport(what + " (stratified rows)")
        for i0 in range(0, len(srows), 1 << 18):
            part = srows[i0:i0 + (1 << 18)]
            sel, s_last, s_next = oracle.select(q_h, kbar, Hkv, bs, topk, part)
            rep.add(gather_idx(idx, part), sel, s_last, s_next)
        rep.finish()
        assert rep.rows >= 1_000_000

    rows = sample_rows(B, Hq, N, bs, topk, per_head, seed)
    gidx = gather_idx(idx, rows)
    go, gl = gather_rows(out, lse, rows)
    sel, _, _ = oracle.select(q_h, kbar, Hkv, bs, topk, rows)
    ref_out, ref_lse = oracle.attend(q_h, k_h, v_h, bs, topk, rows, sel)
    mism = (gidx != sel).any(axis=1)  # excused near ties (checked above)
    ok = ~mism
    compare_outputs(go[ok], gl[ok], ref_out[ok], ref_lse[ok], f"N={N}")
    if mism.any():  # near ties: the oracle's selection injected for the affected rows
        full = idx.clone()
        mt = torch.as_tensor(rows[mism], device=cuda_dev)
        full[mt[:, 0], mt[:, 1], mt[:, 2]] = torch.from_numpy(sel[mism]).to(cuda_dev).to(full.dtype)
        o2, l2 = moba.forward_selected(q, k, v, full, bs, topk)
        assert moba.sync_status() == 0
        go2, gl2 = gather_rows(o2, l2, rows[mism])
        compare_outputs(go2, gl2, ref_out[mism], ref_lse[mism], "injected")
    del q, k, v, out, lse, idx
    gc.collect()
    torch.cuda.empty_cache()
