"""Pins of the oracle's selection-boundary outputs and of the near-tie exemption rule.

The selection check allows another implementation to differ from the oracle only
at a near tie: the last selected and the first unselected past scores differ by
less than 1e-5 relative. These tests pin, against values fixed by hand and by an
independent route (torch's block means and matmul, then a plain Python sort):
  - `near_tie` on constructed score pairs on both sides of the threshold, with
    either sign, mixed signs, zero, equality and the NaN of rows without a boundary;
  - `s_last` / `s_next` (the two scores the rule compares) on random inputs, on
    rows that keep every past block and with topk = 1.
A flipped comparison, a wrong threshold, NaN rows counted as ties or a boundary
score taken from the wrong rank each fail one of them.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

NAN = float("nan")

# (s_last, s_next, expected near tie); s_last is the weaker kept score, s_next the best dropped one
PAIRS = [
    (1.0, 1.0 - 0.5e-5, True),        # relative gap 5e-6 < 1e-5
    (1.0, 1.0 - 2e-5, False),         # relative gap 2e-5
    (1.0, 1.0 - 0.99e-5, True),
    (1.0, 1.0 - 1.01e-5, False),
    (100.0, 100.0 - 5e-4, True),      # the rule is relative: 5e-6 of 100
    (100.0, 100.0 - 2e-3, False),     # 2e-5 of 100
    (1e-3, 1e-3 - 2e-9, True),        # small magnitudes scale the threshold down
    (1e-3, 1e-3 - 2e-7, False),
    (-1.0, -1.0 - 0.5e-5, True),      # negative scores
    (-1.0, -1.0 - 2e-5, False),
    (-3.0, -3.0 - 3e-4, False),       # 1e-4 relative
    (1e-6, -1e-6, False),             # mixed signs: the gap is twice the larger magnitude
    (0.5, -0.5, False),
    (2.5, 2.5, True),                 # equal scores: an exact tie
    (-7.0, -7.0, True),
    (0.0, 0.0, True),                 # equal at zero
    (0.0, 1e-300, False),             # different, one of them zero
    (NAN, NAN, False),                # every past block kept: no boundary
    (NAN, 0.75, False),               # topk = 1: nothing kept by score
    (0.75, NAN, False),
]


@pytest.mark.parametrize("s_last,s_next,want", PAIRS)
def test_near_tie_constructed_pairs(s_last, s_next, want):
    got = oracle.near_tie(np.array([s_last]), np.array([s_next]))
    assert got.dtype == bool and got.shape == (1,)
    assert bool(got[0]) == want


def test_near_tie_is_symmetric_and_vectorised():
    a = np.array([p[0] for p in PAIRS])
    b = np.array([p[1] for p in PAIRS])
    want = np.array([p[2] for p in PAIRS])
    np.testing.assert_array_equal(oracle.near_tie(a, b), want)
    np.testing.assert_array_equal(oracle.near_tie(b, a), want)


def test_near_tie_threshold_argument():
    """A looser threshold admits the 2e-5 pair, a tighter one rejects the 5e-6 pair."""
    assert oracle.near_tie(np.array([1.0]), np.array([1.0 - 2e-5]), rel=1e-4)[0]
    assert not oracle.near_tie(np.array([1.0]), np.array([1.0 - 0.5e-5]), rel=1e-6)[0]


def _torch_scores(q, k, bs, Hq, Hkv):
    """Scores <q_t, mean of block j's keys> by torch (fp64): [B, Hq, N, nfull]."""
    B, N, _, d = q.shape
    nfull = N // bs
    G = Hq // Hkv
    kbar = k[:, : nfull * bs].double().reshape(B, nfull, bs, Hkv, d).mean(dim=2)
    kbar = kbar.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    return (q.double().permute(0, 2, 1, 3) @ kbar.transpose(-1, -2)).numpy()


@pytest.mark.parametrize("case", [(1, 600, 2, 1, 16, 40, 4), (2, 333, 4, 2, 32, 30, 5), (1, 512, 1, 1, 128, 16, 9)])
def test_boundary_scores_match_sorted_torch_scores(case):
    """s_last is the (k-1)-th best past score and s_next the k-th, in the order (score desc, index
    asc), for rows with more than k - 1 past blocks; NaN for the rows that keep every past block."""
    B, N, Hq, Hkv, d, bs, k = case
    q, kk, _ = synth.inputs(B, N, Hq, Hkv, d, bs, seed=17)
    rows = oracle.all_rows(B, Hq, N)
    sel, s_last, s_next = oracle.select(q, oracle.pool(kk, bs), Hkv, bs, k, rows)
    S = _torch_scores(q, kk, bs, Hq, Hkv)
    for i, (b, h, t) in enumerate(rows):
        c = t // bs
        if c <= k - 1:
            assert np.isnan(s_last[i]) and np.isnan(s_next[i])
            continue
        order = sorted(range(c), key=lambda j: (-S[b, h, t, j], j))
        assert abs(s_last[i] - S[b, h, t, order[k - 2]]) <= 1e-12 * max(1.0, abs(s_last[i]))
        assert abs(s_next[i] - S[b, h, t, order[k - 1]]) <= 1e-12 * max(1.0, abs(s_next[i]))
        assert s_last[i] >= s_next[i]
        assert sorted(order[: k - 1]) == list(sel[i][: k - 1])


def test_boundary_scores_with_topk_one():
    """topk = 1 keeps only the own block: s_last is NaN and s_next is the best past score."""
    B, N, Hq, Hkv, d, bs = 1, 200, 1, 1, 16, 20
    q, kk, _ = synth.inputs(B, N, Hq, Hkv, d, bs, seed=3)
    rows = oracle.all_rows(B, Hq, N)
    sel, s_last, s_next = oracle.select(q, oracle.pool(kk, bs), Hkv, bs, 1, rows)
    S = _torch_scores(q, kk, bs, Hq, Hkv)
    assert np.isnan(s_last).all()
    for i, (b, h, t) in enumerate(rows):
        c = t // bs
        assert sel[i][0] == c
        if c == 0:
            assert np.isnan(s_next[i])
        else:
            assert abs(s_next[i] - S[b, h, t, :c].max()) <= 1e-12 * max(1.0, abs(s_next[i]))
    assert not oracle.near_tie(s_last, s_next).any()


def test_constructed_near_tie_rows_are_flagged():
    """Two blocks whose means differ by a relative 1e-6 along q make a near tie at the boundary;
    a relative 1e-3 does not."""
    B, N, Hq, Hkv, d, bs, k = 1, 48, 1, 1, 8, 8, 2
    q = torch.ones(B, N, Hq, d, dtype=torch.bfloat16)
    base = np.zeros((B, N, Hkv, d))
    # block means along the all-ones query: 8 * a_j; blocks 1 and 3 compete for the one past slot
    for j, a in enumerate([0.0, 1.0, -1.0, 1.0, -2.0, 0.0]):
        base[:, j * bs:(j + 1) * bs] = a
    kk = torch.from_numpy(base).to(torch.bfloat16).contiguous()
    rows = oracle.all_rows(B, Hq, N)
    kbar = oracle.pool(kk, bs)
    kb_close = kbar.copy()
    kb_close[0, 0, 3, 0] += 8e-6  # score of block 3: 8 + 8e-6 (relative 1e-6 above block 1)
    kb_far = kbar.copy()
    kb_far[0, 0, 3, 0] -= 8e-3    # 8 - 8e-3 (relative 1e-3 below)
    _, a1, b1 = oracle.select(q, kb_close, Hkv, bs, k, rows)
    _, a2, b2 = oracle.select(q, kb_far, Hkv, bs, k, rows)
    late = rows[:, 2] // bs >= 4
    assert oracle.near_tie(a1, b1)[late].all()
    assert not oracle.near_tie(a2, b2)[late].any()
