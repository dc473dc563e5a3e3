"""GPU parity of the backward (moba_backward) against the fp64 oracle's gradients.

The GPU uses its own forward output and lse (bf16 / fp32) and rounds P and dS to bf16 for the
tensor-core products, as the forward rounds P; each of those roundings is relative 2^-9, so the
bar, per gradient tensor, is: max-abs error <= 1e-2 of the largest reference magnitude and
mean-abs error <= 1e-2 of the mean reference magnitude. Cases: the tiny reference configuration,
GQA with a ragged last block, block size not a multiple of 128, fine granularity with top-k
larger than the number of blocks (dense causal), a single query head group of 8, and the
selection given by the caller (equal to the gate's, so the gradients agree to rounding: the query
lists are filled with atomics, so the order of the fp32 sums over a list can change between runs)."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

REL_MAX, REL_MEAN = 1e-2, 1e-2


def _compare(name, got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    scale_max, scale_mean = np.abs(ref).max(), np.abs(ref).mean()
    assert np.isfinite(g).all(), name
    print(f"[backward] {name}: max err {err.max():.3e} (ref max {scale_max:.3e}), "
          f"mean err {err.mean():.3e} (ref mean {scale_mean:.3e})", flush=True)
    assert err.max() <= REL_MAX * scale_max, (name, err.max(), scale_max)
    assert err.mean() <= REL_MEAN * scale_mean, (name, err.mean(), scale_mean)


CASES = [  # B, N, Hq, Hkv, block_size, topk, seed
    (1, 4096, 1, 1, 512, 3, 0),
    (2, 1000, 4, 2, 128, 3, 101),
    (1, 1500, 2, 2, 200, 4, 102),
    (1, 2048, 2, 1, 256, 16, 103),
    (1, 2304, 8, 1, 256, 4, 104),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"N{c[1]}_H{c[2]}x{c[3]}_bs{c[4]}_k{c[5]}")
def test_backward_against_the_oracle(moba, cuda_dev, case):
    B, N, Hq, Hkv, bs, topk, seed = case
    q_h, k_h, v_h = synth.inputs(B, N, Hq, Hkv, 128, bs, seed)
    g_h = synth.normal(seed + 7, synth.V_ID, (B, N, Hq, 128))
    q, k, v, g = q_h.to(cuda_dev), k_h.to(cuda_dev), v_h.to(cuda_dev), g_h.to(cuda_dev)
    out, lse = moba.forward(q, k, v, bs, topk)
    idx = moba.gate(q, k, bs, topk)
    dq, dk, dv = moba.backward(q, k, v, out, lse, g, bs, topk)
    assert moba.sync_status() == 0
    rows = oracle.all_rows(B, Hq, N)
    sel, _, _ = oracle.select(q_h, oracle.pool(k_h, bs), Hkv, bs, topk, rows)
    sel = sel.reshape(B, Hq, N, topk)
    assert (idx.cpu().numpy() == sel).all()  # no near tie decides anything here
    rq, rk, rv = oracle.backward(q_h, k_h, v_h, g_h, bs, topk, sel)
    _compare(f"dq {case}", dq, rq)
    _compare(f"dk {case}", dk, rk)
    _compare(f"dv {case}", dv, rv)
    # the caller's selection (the gate's) gives the same gradients up to the order of fp32 sums
    dq2, dk2, dv2 = moba.backward(q, k, v, out, lse, g, bs, topk, idx=idx)
    assert moba.sync_status() == 0
    for a, b in ((dq, dq2), (dk, dk2), (dv, dv2)):
        assert (a.float() - b.float()).abs().max().item() <= 1e-2 * a.float().abs().max().item()
