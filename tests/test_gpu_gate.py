"""The tensor-core gate against the fp64 CUDA-core gate, bit for bit.

Both must produce the oracle's selection: the tensor-core gate re-scores every
candidate near the boundary exactly, so any disagreement here is a bug in its
error bound or its boundary logic. Inputs include the workload's distribution,
keys without block offsets (scores crowded near the boundary, which exercises the
exact re-scoring and its fallback) and duplicated blocks (exact ties)."""
import numpy as np
import pytest
import torch

import synth
from parity_util import check_selection_all_rows

pytestmark = pytest.mark.gpu


def _gates(moba, q, k, bs, topk):
    moba.set_gate_impl(1)
    try:
        ref = moba.gate(q, k, bs, topk)
    finally:
        moba.set_gate_impl(0)
    got = moba.gate(q, k, bs, topk)
    assert moba.sync_status() == 0
    return got, ref


@pytest.mark.parametrize("case", [
    (1, 131072, 8, 2, 4096, 12, 3),    # headline shape, fewer heads
    (2, 32768, 8, 2, 256, 32, 2),      # fine granularity, top-32
    (1, 65536, 2, 1, 512, 5, 9),
    (1, 40000, 4, 4, 300, 7, 5),       # ragged, block not a multiple of 128
    (1, 300000, 1, 1, 128, 12, 4),     # many candidate steps (2343 blocks)
])
def test_tc_gate_matches_fp64_gate(moba, cuda_dev, case):
    B, N, Hq, Hkv, bs, topk, seed = case
    q, k, _ = synth.inputs(B, N, Hq, Hkv, 128, bs, seed)
    got, ref = _gates(moba, q.to(cuda_dev), k.to(cuda_dev), bs, topk)
    assert torch.equal(got, ref)
    check_selection_all_rows(got, q, k, Hkv, bs, topk, f"gate case {case}")


def test_tc_gate_crowded_scores(moba, cuda_dev):
    """No block offsets: every block mean is small noise, scores crowd near the boundary.
    Both gates equal each other and the oracle's selection on every row."""
    B, N, Hq, Hkv, bs, topk = 1, 65536, 4, 1, 256, 16
    q = synth.normal(21, synth.Q_ID, (B, N, Hq, 128))
    k = synth.normal(21, synth.K_ID, (B, N, Hkv, 128))
    got, ref = _gates(moba, q.to(cuda_dev), k.to(cuda_dev), bs, topk)
    assert torch.equal(got, ref)
    check_selection_all_rows(got, q, k, Hkv, bs, topk, "crowded scores")


def test_tc_gate_exact_ties(moba, cuda_dev):
    """Blocks repeated verbatim tie exactly; the lower block index must win in both gates."""
    B, N, Hq, Hkv, bs, topk = 1, 32768, 2, 1, 512, 4
    q, k, _ = synth.inputs(B, N, Hq, Hkv, 128, bs, 6)
    k = k.clone()
    for j in range(8, 64, 8):  # block j repeats block j - 5
        k[:, j * bs:(j + 1) * bs] = k[:, (j - 5) * bs:(j - 4) * bs]
    got, ref = _gates(moba, q.to(cuda_dev), k.to(cuda_dev), bs, topk)
    assert torch.equal(got, ref)
    # against the oracle on every row; exact ties are not excused: the lower index must win
    check_selection_all_rows(got, q, k, Hkv, bs, topk, "exact ties", exact_ties_strict=True)
    # the duplicated blocks really produced exact ties at the boundary of some rows
    import oracle
    rows = oracle.all_rows(B, Hq, N)
    _, s_last, s_next = oracle.select(q, oracle.pool(k, bs), Hkv, bs, topk, rows)
    assert int((s_last == s_next).sum()) > 100
