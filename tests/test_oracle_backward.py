"""Pins of the oracle's backward (dq, dk, dv of sum(dout * out) with the selection held fixed).

Reading: the top-k choice is discrete, so gradients flow only through the attention of the kept
keys and the block summaries receive none. Pinned against torch autograd in fp64 (dense causal
attention when every block is kept; attention masked by the oracle's selection otherwise, which
checks the sparse pattern, the causal own block and GQA accumulation), and against central
finite differences of the same loss evaluated in fp64 on a tiny case."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def _torch_grads(q, k, v, dout, allowed):
    """fp64 autograd of softmax(q k^T / sqrt(d)) v under a boolean mask allowed [B, Hq, N, N]."""
    B, N, Hq, d = q.shape
    G = Hq // k.shape[2]
    qq = q.double().requires_grad_(True)
    kk = k.double().requires_grad_(True)
    vv = v.double().requires_grad_(True)
    qh = qq.permute(0, 2, 1, 3)
    kh = kk.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vh = vv.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    logits = (qh @ kh.transpose(-1, -2)) / math.sqrt(d)
    p = torch.softmax(logits.masked_fill(~allowed, float("-inf")), dim=-1)
    out = (p @ vh).permute(0, 2, 1, 3)
    (out * dout.double()).sum().backward()
    return qq.grad.numpy(), kk.grad.numpy(), vv.grad.numpy()


def _mask_from_selection(sel, N, bs):
    """allowed[b, h, t, u]: u in a kept earlier block of row t, or in t's own block with u <= t."""
    B, Hq = sel.shape[:2]
    allowed = torch.zeros(B, Hq, N, N, dtype=torch.bool)
    for b in range(B):
        for h in range(Hq):
            for t in range(N):
                c = t // bs
                for j in sel[b, h, t]:
                    if j < 0:
                        continue
                    lo = j * bs
                    hi = t + 1 if j == c else (j + 1) * bs
                    allowed[b, h, t, lo:hi] = True
    return allowed


@pytest.mark.parametrize("case", [(1, 64, 2, 1, 16, 8, 8), (2, 50, 4, 2, 8, 10, 6)])
def test_every_block_kept_is_dense_causal_autograd(case):
    B, N, Hq, Hkv, d, bs, k = case
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, 90)
    dout = synth.normal(91, synth.V_ID, (B, N, Hq, d))
    dq, dk, dv = oracle.backward(q, kk, v, dout, bs, k)
    causal = torch.ones(N, N, dtype=torch.bool).tril().expand(B, Hq, N, N)
    tq, tk, tv = _torch_grads(q, kk, v, dout, causal)
    for a, b in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(a, b, atol=1e-11, rtol=0)


@pytest.mark.parametrize("case", [(1, 96, 2, 1, 16, 8, 3), (2, 70, 4, 2, 8, 10, 2), (1, 40, 2, 2, 8, 4, 1)])
def test_sparse_selection_is_masked_autograd(case):
    B, N, Hq, Hkv, d, bs, k = case
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, 92)
    dout = synth.normal(93, synth.V_ID, (B, N, Hq, d))
    rows = oracle.all_rows(B, Hq, N)
    sel, _, _ = oracle.select(q, oracle.pool(kk, bs), Hkv, bs, k, rows)
    sel = sel.reshape(B, Hq, N, k)
    dq, dk, dv = oracle.backward(q, kk, v, dout, bs, k, sel)
    tq, tk, tv = _torch_grads(q, kk, v, dout, _mask_from_selection(sel, N, bs))
    for a, b in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(a, b, atol=1e-11, rtol=0)


def test_central_differences_of_the_forward():
    """d/dx sum(dout * out) by central differences of the forward in fp64 with the oracle's selection
    held fixed (perturbations far smaller than any score gap of this input)."""
    B, N, Hq, Hkv, d, bs, k = 1, 24, 1, 1, 4, 6, 2
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, 94)
    dout = synth.normal(95, synth.V_ID, (B, N, Hq, d))
    dq, dk, dv = oracle.backward(q, kk, v, dout, bs, k)
    rows = oracle.all_rows(B, Hq, N)
    sel, _, _ = oracle.select(q, oracle.pool(kk, bs), Hkv, bs, k, rows)

    def loss(qd, kd, vd):
        # the forward in fp64 on fp64 inputs, through torch (rows' allowed keys from the selection)
        allowed = _mask_from_selection(sel.reshape(B, Hq, N, k), N, bs)
        logits = (qd.permute(0, 2, 1, 3) @ kd.permute(0, 2, 3, 1)) / math.sqrt(d)
        p = torch.softmax(logits.masked_fill(~allowed, float("-inf")), dim=-1)
        out = (p @ vd.permute(0, 2, 1, 3)).permute(0, 2, 1, 3)
        return float((out * dout.double()).sum())

    base = [q.double(), kk.double(), v.double()]
    h = 1e-6
    rng = np.random.default_rng(0)
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in base[which].shape)
            plus = [x.clone() for x in base]
            minus = [x.clone() for x in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd = (loss(*plus) - loss(*minus)) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-6, (which, idx, fd, grad[idx])
