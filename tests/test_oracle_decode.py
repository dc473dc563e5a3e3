"""Pins of the oracle's decode step (one new query against its KV cache).

A decode step is the prefill definition at the last row, so it is pinned against what does not
come from the oracle itself: torch's scaled_dot_product_attention of the single query over all
keys when every block is kept (the full-attention decode of a hybrid model, "KIMI MoBA" blog,
section 3: MoBA for prefill, full attention for decode), the brute-force best subset of earlier
blocks (scores from torch's block means), and causality (keys after the query's position and
unselected blocks have no effect)."""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def _sdpa_last_row(q, k, v, L):
    """torch fp64 attention of the query q [B, Hq, d] over keys 0..L-1 (GQA by repetition)."""
    B, Hq, d = q.shape
    G = Hq // k.shape[2]
    kk = k[:, :L].double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)  # [B, Hq, L, d]
    vv = v[:, :L].double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    qq = q.double().unsqueeze(2)  # [B, Hq, 1, d]
    out = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, :, 0]
    lse = torch.logsumexp((qq @ kk.transpose(-1, -2))[:, :, 0] / math.sqrt(d), dim=-1)
    return out.reshape(B * Hq, d).numpy(), lse.reshape(B * Hq).numpy()


@pytest.mark.parametrize("case", [(1, 100, 2, 1, 16, 10, 3), (2, 257, 4, 2, 32, 32, 2), (1, 64, 1, 1, 128, 64, 1)])
def test_full_attention_decode_is_sdpa(case):
    B, L, Hq, Hkv, d, bs, k = case
    q, kk, v = synth.inputs(B, L + 5, Hq, Hkv, d, bs, 40)  # a cache longer than the sequence
    qd = q[:, 0].contiguous()
    r = oracle.decode(qd, kk, v, bs, k, L, full_attention=True)
    o, l = _sdpa_last_row(qd, kk, v, L)
    np.testing.assert_allclose(r["out"], o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(r["lse"], l, atol=1e-12, rtol=0)


def test_decode_selection_is_the_best_subset():
    B, L, Hq, Hkv, d, bs, k = 1, 90, 3, 1, 8, 8, 4
    q, kk, v = synth.inputs(B, L, Hq, Hkv, d, bs, 41)
    qd = synth.normal(42, synth.Q_ID, (B, Hq, d))
    r = oracle.decode(qd, kk, v, bs, k, L)
    c = (L - 1) // bs
    kbar = kk[:, : c * bs].double().reshape(B, c, bs, Hkv, d).mean(dim=2)[0, :, 0]  # [c, d]
    for h in range(Hq):
        s = (qd[0, h].double() @ kbar.T).numpy()
        best = max(itertools.combinations(range(c), k - 1), key=lambda sub: (sum(s[j] for j in sub), [-j for j in sub]))
        assert list(r["sel"][h]) == sorted(best) + [c]


def test_decode_ignores_keys_after_the_query_and_unselected_blocks():
    B, L, Hq, Hkv, d, bs, k = 1, 150, 2, 1, 16, 16, 3
    q, kk, v = synth.inputs(B, L + 40, Hq, Hkv, d, bs, 43)
    qd = q[:, 3].contiguous()
    r = oracle.decode(qd, kk, v, bs, k, L)
    k2, v2 = kk.clone(), v.clone()
    k2[:, L:] = 7.0  # beyond the sequence
    v2[:, L:] = -3.0
    unsel = [j for j in range((L - 1) // bs) if all(j not in row for row in r["sel"])]
    assert unsel
    j = unsel[0]
    v2[:, j * bs:(j + 1) * bs] = 5.0  # an unselected block's values
    r2 = oracle.decode(qd, k2, v2, bs, k, L)
    np.testing.assert_array_equal(r["sel"], r2["sel"])
    np.testing.assert_array_equal(r["out"], r2["out"])
    np.testing.assert_array_equal(r["lse"], r2["lse"])
