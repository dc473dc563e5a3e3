"""Pins of the fp64 oracle against facts the MoBA pages and mathematics fix.

Each test checks the oracle against something other than itself: a library
routine (torch's scaled_dot_product_attention, torch mean / matmul), brute force
over subsets, closed forms on constructed inputs, or numbers printed on the pages.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from block_sparse_long_gate_b200 import flops


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float64).to(torch.float32).to(torch.bfloat16).contiguous()


def _sdpa_causal(q, k, v):
    """Dense causal attention from torch (fp64, CPU), GQA by repeating kv heads: head h -> h // G."""
    B, N, Hq, d = q.shape
    G = Hq // k.shape[2]
    qq = q.double().permute(0, 2, 1, 3)
    kk = k.double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vv = v.double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    out = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True)
    logits = qq @ kk.transpose(-1, -2) / math.sqrt(d)
    mask = torch.ones(N, N, dtype=torch.bool).tril()
    lse = torch.logsumexp(logits.masked_fill(~mask, float("-inf")), dim=-1)
    return out.permute(0, 2, 1, 3).numpy(), lse.numpy()  # [B, N, Hq, d], [B, Hq, N]


DENSE_CASES = [  # B, N, Hq, Hkv, d, block_size, topk
    (1, 1, 1, 1, 8, 4, 1),
    (1, 7, 1, 1, 8, 2, 4),
    (1, 64, 2, 1, 16, 8, 8),
    (2, 257, 4, 2, 32, 32, 9),
    (1, 300, 2, 2, 128, 64, 5),
    (1, 200, 4, 1, 64, 256, 1),  # block_size >= N: one block
]


@pytest.mark.parametrize("case", DENSE_CASES)
def test_full_selection_is_dense_causal(case):
    """topk >= number of blocks (or block_size >= N) must be dense causal attention.

    The "MoBA tech-report summary" (section 2) and the feature list of the
    aliyun article say MoBA switches seamlessly to full attention; with every
    past block selected that is exactly causal softmax attention."""
    B, N, Hq, Hkv, d, bs, k = case
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, seed=11)
    r = oracle.forward(q, kk, v, bs, k)
    ref_out, ref_lse = _sdpa_causal(q, kk, v)
    rows = r["rows"]
    ref_o = ref_out[rows[:, 0], rows[:, 2], rows[:, 1]]
    ref_l = ref_lse[rows[:, 0], rows[:, 1], rows[:, 2]]
    np.testing.assert_allclose(r["out"], ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], ref_l, rtol=0, atol=1e-12)


def test_early_rows_equal_dense_causal():
    """Rows whose own block index c <= k - 1 select every past block, so they equal dense causal."""
    B, N, Hq, Hkv, d, bs, k = 1, 640, 2, 1, 32, 64, 3
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, seed=5)
    r = oracle.forward(q, kk, v, bs, k)
    ref_out, ref_lse = _sdpa_causal(q, kk, v)
    rows = r["rows"]
    early = rows[:, 2] // bs <= k - 1
    late = ~early
    np.testing.assert_allclose(r["out"][early], ref_out[rows[early, 0], rows[early, 2], rows[early, 1]],
                               atol=1e-12, rtol=0)
    np.testing.assert_allclose(r["lse"][early], ref_lse[rows[early, 0], rows[early, 1], rows[early, 2]],
                               atol=1e-12, rtol=0)
    # and later rows really are sparse: they differ from dense attention
    diff = np.abs(r["lse"][late] - ref_lse[rows[late, 0], rows[late, 1], rows[late, 2]])
    assert diff.min() > 1e-6


def _scores_by_torch(q, k, bs, Hq, Hkv):
    """Scores <q_t, mean(K_block_j)> from torch's own mean and matmul (fp64)."""
    B, N, _, d = q.shape
    nfull = N // bs
    G = Hq // Hkv
    kbar = k[:, : nfull * bs].double().reshape(B, nfull, bs, Hkv, d).mean(dim=2)  # [B, nfull, Hkv, d]
    kbar = kbar.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)  # [B, Hq, nfull, d]
    qq = q.double().permute(0, 2, 1, 3)  # [B, Hq, N, d]
    return (qq @ kbar.transpose(-1, -2)).numpy()  # [B, Hq, N, nfull]


@pytest.mark.parametrize("case", [(1, 96, 1, 1, 8, 8, 3), (2, 130, 4, 2, 16, 16, 4), (1, 77, 2, 1, 128, 9, 2)])
def test_selection_matches_subset_brute_force(case):
    """The selection equals the best-scoring (k-1)-subset of past blocks plus the own block.

    Scores come from torch (mean of each block's keys, then a matmul), and the
    subset is found by enumerating every (k-1)-subset of the past blocks - an
    independent route to the gating of the "MoBA project hub" Step 2 and the
    causal rules of the "KIMI MoBA" blog, section 3."""
    B, N, Hq, Hkv, d, bs, k = case
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, seed=3)
    r = oracle.forward(q, kk, v, bs, k)
    S = _scores_by_torch(q, kk, bs, Hq, Hkv)
    for i, (b, h, t) in enumerate(r["rows"]):
        c = t // bs
        past = list(range(c))
        if c <= k - 1:
            best = past
        else:
            best, best_sum = None, -np.inf
            for sub in itertools.combinations(past, k - 1):
                s = sum(S[b, h, t, j] for j in sub)
                if s > best_sum + 1e-12:
                    best, best_sum = list(sub), s
        want = sorted(best) + [c] + [-1] * (k - 1 - len(best))
        assert list(r["sel"][i]) == want, (b, h, t)


def test_exact_ties_go_to_lower_block():
    """Two blocks with identical keys tie exactly; the lower block index must win the last slot."""
    B, N, Hq, Hkv, d, bs, k = 1, 48, 1, 1, 8, 8, 2
    base = np.zeros((B, N, Hkv, d))
    offs = [0.0, 2.0, -1.0, 0.5, 2.0, -0.5]  # blocks 1 and 4 tie for the top score
    for j, c in enumerate(offs):
        base[:, j * bs:(j + 1) * bs] = c
    kk = _bf16(base)
    q = _bf16(np.abs(np.random.default_rng(0).normal(size=(B, N, Hq, d))) + 0.25)  # positive sum
    v = synth.normal(1, synth.V_ID, (B, N, Hkv, d))
    r = oracle.forward(q, kk, v, bs, k)
    for i, (_, _, t) in enumerate(r["rows"]):
        c = t // bs
        if c >= 5:  # both 1 and 4 are past blocks
            assert list(r["sel"][i]) == [1, c], t
            assert r["s_last"][i] == r["s_next"][i]  # an exact tie at the boundary


def test_constant_blocks_closed_form():
    """Keys constant inside each block give closed forms for scores, selection, lse and out.

    With K[u] = a_j * 1 for u in block j: Kbar_j = a_j * 1, s_j = a_j * sum(q), every
    key of block j has logit a_j * sum(q) / sqrt(d), so lse = ln sum_j n_j exp(a_j sum(q)/sqrt(d))
    and out is the matching weighted mean of V over the allowed keys (n_j = keys used
    from block j; the own block contributes t - cB + 1 keys)."""
    B, N, Hq, Hkv, d, bs, k = 1, 80, 2, 1, 16, 10, 3
    a = np.array([0.5, -1.0, 1.5, 0.25, -0.75, 1.0, 2.0, -2.0])
    kk = _bf16(np.repeat(a, bs)[None, :, None, None] * np.ones((B, N, Hkv, d)))
    rng = np.random.default_rng(4)
    q = _bf16(rng.normal(size=(B, N, Hq, d)))
    v = _bf16(rng.normal(size=(B, N, Hkv, d)))
    r = oracle.forward(q, kk, v, bs, k)
    qd, vd = q.double().numpy(), v.double().numpy()
    for i, (b, h, t) in enumerate(r["rows"]):
        c = t // bs
        sq = qd[b, t, h].sum()
        order = sorted(range(c), key=lambda j: (-a[j] * sq, j))
        past = sorted(order[: k - 1])
        assert list(r["sel"][i][: len(past) + 1]) == past + [c]
        blocks = [(j, j * bs, (j + 1) * bs) for j in past] + [(c, c * bs, t + 1)]
        lw = [math.log(hi - lo) + a[j] * sq / math.sqrt(d) for j, lo, hi in blocks]
        lse = np.logaddexp.reduce(lw)
        out = sum(math.exp(a[j] * sq / math.sqrt(d) - lse) * vd[b, lo:hi, 0].sum(axis=0) for j, lo, hi in blocks)
        assert abs(r["lse"][i] - lse) < 1e-12
        np.testing.assert_allclose(r["out"][i], out, atol=1e-12, rtol=0)


def test_first_token_closed_form():
    """Token 0 attends only itself: out = v_0 and lse = q.k / sqrt(d)."""
    q, kk, v = synth.inputs(1, 5, 1, 1, 128, 4, seed=9)
    r = oracle.forward(q, kk, v, 4, 2)
    np.testing.assert_array_equal(r["out"][0], v[0, 0, 0].double().numpy())
    want = (q[0, 0, 0].double() * kk[0, 0, 0].double()).sum().item() / math.sqrt(128)
    assert abs(r["lse"][0] - want) < 1e-12


def test_future_and_unselected_blocks_have_no_effect():
    """No query reads a future block or an unselected past block ("MoBA tech-report summary",
    section 2, causality paragraph): rewriting them leaves every affected row unchanged, bit for bit."""
    B, N, Hq, Hkv, d, bs, k = 1, 256, 2, 1, 32, 32, 3
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, seed=21)
    r = oracle.forward(q, kk, v, bs, k)
    rows = r["rows"]
    # future blocks: rewrite K and V from token 160 on; rows t < 160 must not move
    k2, v2 = kk.clone(), v.clone()
    k2[:, 160:] = _bf16(np.random.default_rng(1).normal(size=k2[:, 160:].shape) * 3)
    v2[:, 160:] = _bf16(np.random.default_rng(2).normal(size=v2[:, 160:].shape) * 3)
    r2 = oracle.forward(q, k2, v2, bs, k)
    keep = rows[:, 2] < 160
    np.testing.assert_array_equal(r["sel"][keep], r2["sel"][keep])
    np.testing.assert_array_equal(r["out"][keep], r2["out"][keep])
    np.testing.assert_array_equal(r["lse"][keep], r2["lse"][keep])
    # an unselected past block: rewrite its V; rows that did not select it must not move
    j = 2
    v3 = v.clone()
    v3[:, j * bs:(j + 1) * bs] = _bf16(np.random.default_rng(3).normal(size=(B, bs, Hkv, d)) * 5)
    out3, lse3 = oracle.attend(q, kk, v3, bs, k, rows, r["sel"])
    unsel = ~(r["sel"] == j).any(axis=1)
    assert unsel.sum() > 50 and (~unsel).sum() > 50
    np.testing.assert_array_equal(out3[unsel], r["out"][unsel])
    np.testing.assert_array_equal(lse3[unsel], r["lse"][unsel])
    assert np.abs(out3[~unsel] - r["out"][~unsel]).max() > 1e-3


@pytest.mark.parametrize("case", [(1, 4096, 1, 1, 128, 512, 3), (2, 333, 4, 2, 64, 40, 4)])
def test_blockwise_lse_merge_equals_direct(case):
    """Per-block partials merged by log-sum-exp ("MoBA project hub", Step 3) equal the single softmax."""
    B, N, Hq, Hkv, d, bs, k = case
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, seed=2)
    rows = oracle.all_rows(B, Hq, N)[::7]
    kbar = oracle.pool(kk, bs)
    sel, _, _ = oracle.select(q, kbar, Hkv, bs, k, rows)
    o1, l1 = oracle.attend(q, kk, v, bs, k, rows, sel)
    o2, l2 = oracle.attend(q, kk, v, bs, k, rows, sel, blockwise=True)
    np.testing.assert_allclose(o1, o2, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l1, l2, atol=1e-12, rtol=0)


def test_pool_is_block_mean():
    """Kbar equals torch's mean over each full block (score_pooling = mean, "KIMI MoBA" section 3)."""
    B, N, Hkv, d, bs = 2, 100, 3, 16, 32
    kk = synth.keys(8, B, N, Hkv, d, bs)
    kbar = oracle.pool(kk, bs)
    want = kk[:, :96].double().reshape(B, 3, bs, Hkv, d).mean(dim=2).permute(0, 2, 1, 3).numpy()
    assert kbar.shape == (B, Hkv, 3, d)
    np.testing.assert_allclose(kbar, want, atol=1e-15, rtol=0)


def test_injected_selection_rejects_future_blocks():
    q, kk, v = synth.inputs(1, 64, 1, 1, 8, 8, seed=1)
    rows = np.array([[0, 0, 20]], dtype=np.int64)
    with pytest.raises(ValueError):
        oracle.attend(q, kk, v, 8, 2, rows, np.array([[2, 3]], dtype=np.int32))  # 3 is a future block
    with pytest.raises(ValueError):
        oracle.attend(q, kk, v, 8, 2, rows, np.array([[0, 1]], dtype=np.int32))  # own block missing


def _golden_rows():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "p1_block_topk_table.txt")
    out = []
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            kind, N, bs, k, pct, digits = line.split()
            out.append((kind, int(N), int(bs), int(k), float(pct), int(digits)))
    return out


@pytest.mark.parametrize("row", _golden_rows())
def test_nominal_sparsity_matches_page_table(row):
    kind, N, bs, k, pct, digits = row
    assert round(100 * flops.nominal_sparsity(N, bs, k), digits) == pct
    if kind == "toy":
        assert k * bs == 1536  # the simulation's "1536 tokens"


@pytest.mark.parametrize("case", [(1, 300, 1, 1, 8, 32, 3), (1, 256, 2, 1, 8, 64, 2), (1, 100, 1, 1, 8, 7, 20)])
def test_useful_pairs_count_matches_oracle_selection(case):
    """The work count used for TFLOP/s equals the number of keys the oracle attends."""
    B, N, Hq, Hkv, d, bs, k = case
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, seed=0)
    r = oracle.forward(q, kk, v, bs, k)
    n = 0
    for (b, h, t), s in zip(r["rows"], r["sel"]):
        c = t // bs
        n += sum(bs for j in s if 0 <= j < c) + (t - c * bs + 1)
    assert n == B * Hq * flops.useful_pairs_per_head(N, bs, k)
    if k >= flops.nblocks(N, bs):
        assert n == B * Hq * flops.dense_causal_pairs_per_head(N)
