"""Pins of the oracle's packed (varlen) form. Reading: every packed sequence is its own context -
its blocks start at its first token and no query attends another sequence's keys (the pages'
FlashAttention pipeline, "MoBA tech-report summary" section 2, runs a variable-length kernel over
sequences). Pinned by: equal lengths equal the batched forward; keys of other sequences have no
effect (rewriting them leaves every row bit for bit); a sequence of length at most one block, or
with every block kept, equals torch's causal SDPA of that sequence alone."""
import math

import numpy as np
import torch

import oracle
import synth


def test_equal_lengths_equal_the_batched_forward():
    B, N, Hq, Hkv, d, bs, k = 3, 200, 2, 1, 16, 32, 3
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, 70)
    r = oracle.forward(q, kk, v, bs, k)
    pv = oracle.forward_varlen(q.reshape(B * N, Hq, d), kk.reshape(B * N, Hkv, d), v.reshape(B * N, Hkv, d),
                               [0, N, 2 * N, 3 * N], bs, k)
    rows = r["rows"]
    np.testing.assert_array_equal(pv["sel"][rows[:, 1], rows[:, 0] * N + rows[:, 2]], r["sel"])
    np.testing.assert_array_equal(pv["out"][rows[:, 0] * N + rows[:, 2], rows[:, 1]], r["out"])
    np.testing.assert_array_equal(pv["lse"][rows[:, 1], rows[:, 0] * N + rows[:, 2]], r["lse"])


def test_other_sequences_have_no_effect():
    cu = [0, 150, 151, 400, 400, 777]
    total, Hq, Hkv, d, bs, k = cu[-1], 2, 2, 16, 40, 3
    q, kk, v = synth.inputs(1, total, Hq, Hkv, d, bs, 71)
    q, kk, v = q[0], kk[0], v[0]
    a = oracle.forward_varlen(q, kk, v, cu, bs, k)
    k2, v2 = kk.clone(), v.clone()
    k2[151:400] = 9.0  # the third sequence's keys and values
    v2[151:400] = -9.0
    b = oracle.forward_varlen(q, k2, v2, cu, bs, k)
    keep = np.r_[0:151, 400:777]
    np.testing.assert_array_equal(a["out"][keep], b["out"][keep])
    np.testing.assert_array_equal(a["lse"][:, keep], b["lse"][:, keep])
    np.testing.assert_array_equal(a["sel"][:, keep], b["sel"][:, keep])


def test_short_sequences_are_dense_causal():
    cu = [0, 30, 95, 96]
    total, Hq, Hkv, d, bs, k = cu[-1], 2, 1, 8, 128, 2
    q, kk, v = synth.inputs(1, total, Hq, Hkv, d, bs, 72)
    q, kk, v = q[0], kk[0], v[0]
    r = oracle.forward_varlen(q, kk, v, cu, bs, k)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        qq = q[a:b].double().permute(1, 0, 2)
        kr = kk[a:b].double().repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
        vr = v[a:b].double().repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
        o = torch.nn.functional.scaled_dot_product_attention(qq, kr, vr, is_causal=True).permute(1, 0, 2)
        logits = (qq @ kr.transpose(-1, -2)) / math.sqrt(d)
        mask = torch.ones(b - a, b - a, dtype=torch.bool).tril()
        l = torch.logsumexp(logits.masked_fill(~mask, float("-inf")), dim=-1)
        np.testing.assert_allclose(r["out"][a:b], o.numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(r["lse"][:, a:b], l.numpy(), atol=1e-12, rtol=0)
