"""Randomised pins of the fp64 oracle (hypothesis, derandomised so every run checks the same cases).

Each property compares the oracle with an independent route on shapes drawn at random:
  - selection: torch's own block means and matmul, then a plain sort by (score desc, index asc);
  - topk >= number of blocks: torch's causal scaled_dot_product_attention;
  - the blockwise form merged by log-sum-exp equals the direct softmax over the union of keys.
"""
import math

import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle
import synth

SETTINGS = dict(max_examples=25, deadline=None, derandomize=True)


@st.composite
def shapes(draw, max_n=160):
    hkv = draw(st.integers(1, 2))
    g = draw(st.integers(1, 3))
    return dict(B=draw(st.integers(1, 2)), N=draw(st.integers(1, max_n)), Hq=hkv * g, Hkv=hkv,
                d=draw(st.sampled_from([8, 16, 32])), bs=draw(st.integers(1, 48)), k=draw(st.integers(1, 6)),
                seed=draw(st.integers(0, 10 ** 6)))


@settings(**SETTINGS)
@given(shapes())
def test_selection_is_sorted_torch_scores(s):
    B, N, Hq, Hkv, d, bs, k = s["B"], s["N"], s["Hq"], s["Hkv"], s["d"], s["bs"], s["k"]
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, s["seed"])
    r = oracle.forward(q, kk, v, bs, k)
    nfull = N // bs
    G = Hq // Hkv
    if nfull > 0:
        kbar = kk[:, : nfull * bs].double().reshape(B, nfull, bs, Hkv, d).mean(dim=2)
        kbar = kbar.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)        # [B, Hq, nfull, d]
        S = (q.double().permute(0, 2, 1, 3) @ kbar.transpose(-1, -2)).numpy()
    for i, (b, h, t) in enumerate(r["rows"]):
        c = t // bs
        order = sorted(range(c), key=lambda j: (-S[b, h, t, j], j)) if c > 0 else []
        kept = sorted(order[: k - 1])
        want = kept + [c] + [-1] * (k - 1 - len(kept))
        assert list(r["sel"][i]) == want, (b, h, t)


@settings(**SETTINGS)
@given(shapes(max_n=96))
def test_full_selection_is_torch_dense_causal(s):
    B, N, Hq, Hkv, d, bs = s["B"], s["N"], s["Hq"], s["Hkv"], s["d"], s["bs"]
    k = -(-N // bs)  # every block
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, s["seed"])
    r = oracle.forward(q, kk, v, bs, k)
    G = Hq // Hkv
    qq = q.double().permute(0, 2, 1, 3)
    k2 = kk.double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    v2 = v.double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    out = torch.nn.functional.scaled_dot_product_attention(qq, k2, v2, is_causal=True).permute(0, 2, 1, 3).numpy()
    logits = qq @ k2.transpose(-1, -2) / math.sqrt(d)
    lse = torch.logsumexp(logits.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf")), -1).numpy()
    rows = r["rows"]
    np.testing.assert_allclose(r["out"], out[rows[:, 0], rows[:, 2], rows[:, 1]], atol=1e-12, rtol=0)
    np.testing.assert_allclose(r["lse"], lse[rows[:, 0], rows[:, 1], rows[:, 2]], atol=1e-12, rtol=0)


@settings(**SETTINGS)
@given(shapes())
def test_blockwise_merge_equals_direct(s):
    B, N, Hq, Hkv, d, bs, k = s["B"], s["N"], s["Hq"], s["Hkv"], s["d"], s["bs"], s["k"]
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, s["seed"])
    rows = oracle.all_rows(B, Hq, N)
    kbar = oracle.pool(kk, bs)
    sel, _, _ = oracle.select(q, kbar, Hkv, bs, k, rows)
    o1, l1 = oracle.attend(q, kk, v, bs, k, rows, sel)
    o2, l2 = oracle.attend(q, kk, v, bs, k, rows, sel, blockwise=True)
    np.testing.assert_allclose(o2, o1, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l2, l1, atol=1e-12, rtol=0)
