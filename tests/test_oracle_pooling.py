"""Pins of the oracle's pooling variants (the "KIMI MoBA" blog, section 6, suggests max pooling
or weighted pooling of a block's keys as alternatives to the mean).

Readings: max pooling is the feature-wise maximum over the block's keys; weighted pooling is
sum_p w[p] K[jB + p] / sum_p w[p] with one caller-given non-negative weight per position inside a
block. Checked against torch / numpy library routines, closed forms (equal weights give the mean,
a one-hot weight picks one key), and the selection they induce against a plain sort."""
import numpy as np
import pytest
import torch

import oracle
import synth


def test_max_pooling_is_blockwise_amax():
    B, N, Hkv, d, bs = 2, 100, 3, 16, 32
    k = synth.keys(8, B, N, Hkv, d, bs)
    got = oracle.pool(k, bs, "max")
    want = k[:, :96].double().reshape(B, 3, bs, Hkv, d).amax(dim=2).permute(0, 2, 1, 3).numpy()
    assert got.shape == (B, Hkv, 3, d)
    np.testing.assert_array_equal(got, want)


def test_weighted_pooling_is_the_weighted_mean():
    B, N, Hkv, d, bs = 1, 130, 2, 8, 40
    k = synth.keys(9, B, N, Hkv, d, bs)
    w = np.random.default_rng(1).random(bs).astype(np.float32).astype(np.float64)
    got = oracle.pool(k, bs, "weighted", w)
    kb = k[:, :120].double().reshape(B, 3, bs, Hkv, d).numpy()
    want = np.einsum("p,bjphe->bhje", w, kb) / w.sum()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


def test_equal_weights_give_the_mean_and_one_hot_weights_pick_a_key():
    B, N, Hkv, d, bs = 1, 64, 1, 16, 16
    k = synth.keys(10, B, N, Hkv, d, bs)
    np.testing.assert_array_equal(oracle.pool(k, bs, "weighted", np.full(bs, 0.25)), oracle.pool(k, bs))
    p = 5
    w = np.zeros(bs)
    w[p] = 3.0
    got = oracle.pool(k, bs, "weighted", w)
    want = k[0, p::bs][:4, 0].double().numpy()  # key p of each block
    np.testing.assert_array_equal(got[0, 0], want)


@pytest.mark.parametrize("pooling", ["max", "weighted"])
def test_selection_with_pooling_matches_a_sort_of_library_scores(pooling):
    """Top-(k-1) earlier blocks by <q, pooled block> (score desc, index asc) plus the own block,
    with the pooled blocks computed by torch."""
    B, N, Hq, Hkv, d, bs, kk = 1, 400, 2, 1, 16, 25, 4
    q, k, _ = synth.inputs(B, N, Hq, Hkv, d, bs, 12)
    w = np.random.default_rng(2).random(bs)
    r = oracle.forward(q, k, _, bs, kk, pooling=pooling, weights=w if pooling == "weighted" else None)
    nfull = N // bs
    blocks = k[:, : nfull * bs].double().reshape(B, nfull, bs, Hkv, d)
    if pooling == "max":
        pooled = blocks.amax(dim=2)
    else:
        pooled = torch.einsum("p,bjphe->bjhe", torch.from_numpy(w), blocks) / float(w.sum())
    S = (q.double().permute(0, 2, 1, 3) @ pooled.permute(0, 2, 3, 1)).numpy()  # [B, Hq, N, nfull] (Hkv = 1)
    for i, (b, h, t) in enumerate(r["rows"]):
        c = t // bs
        order = sorted(range(c), key=lambda j: (-S[b, h, t, j], j))
        past = sorted(order[: kk - 1])
        assert list(r["sel"][i][: len(past) + 1]) == past + [c], (t, pooling)


@pytest.mark.parametrize("pooling", ["mean", "max", "weighted"])
def test_pooling_does_not_change_the_attention_given_the_selection(pooling):
    """Pooling only decides the selection: with every block selected the forward is the same."""
    B, N, Hq, Hkv, d, bs = 1, 96, 2, 2, 16, 16
    q, k, v = synth.inputs(B, N, Hq, Hkv, d, bs, 13)
    w = np.linspace(0.5, 1.5, bs)
    r0 = oracle.forward(q, k, v, bs, 8)
    r1 = oracle.forward(q, k, v, bs, 8, pooling=pooling, weights=w if pooling == "weighted" else None)
    np.testing.assert_array_equal(r0["out"], r1["out"])
    np.testing.assert_array_equal(r0["sel"], r1["sel"])
