"""GPU parity of the pooling variants and of the hybrid-layer switch, through the extended
entry points (moba_gate_ex / moba_forward_ex), against the fp64 oracle.

Max pooling and weighted pooling ("KIMI MoBA" blog, section 6) change only the block summary the
gate scores; the selection of every row must equal the oracle's (same near-tie rule as the mean),
and the outputs must meet the usual bar (max-abs 2e-2, mean-abs 2e-3, lse 1e-3). A full-attention
layer (the switch of a hybrid model, section 3 hybrid_layers) must equal dense causal attention."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import check_selection_all_rows, compare_outputs, gather_idx, gather_rows, sample_rows

pytestmark = pytest.mark.gpu


def _weights(bs, seed):
    # fp32 values (what the device reads), handed to the oracle in fp64
    return np.random.default_rng(seed).uniform(0.25, 2.0, bs).astype(np.float32)


CASES = [  # B, N, Hq, Hkv, block_size, topk, seed
    (1, 4096, 1, 1, 512, 3, 0),
    (2, 3000, 4, 2, 200, 4, 31),
    (1, 131072, 8, 2, 4096, 12, 3),
    (2, 32768, 8, 2, 256, 32, 2),
]


@pytest.mark.parametrize("pooling", ["max", "weighted"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"N{c[1]}_bs{c[4]}_k{c[5]}")
def test_pooling_variants_against_the_oracle(moba, cuda_dev, case, pooling):
    B, N, Hq, Hkv, bs, topk, seed = case
    q_h, k_h, v_h = synth.inputs(B, N, Hq, Hkv, 128, bs, seed)
    q, k, v = q_h.to(cuda_dev), k_h.to(cuda_dev), v_h.to(cuda_dev)
    w = _weights(bs, seed) if pooling == "weighted" else None
    wd = torch.from_numpy(w).to(cuda_dev) if w is not None else None
    w64 = w.astype(np.float64) if w is not None else None
    idx = moba.gate(q, k, bs, topk, pooling=pooling, pool_weights=wd)
    out, lse = moba.forward(q, k, v, bs, topk, pooling=pooling, pool_weights=wd)
    assert moba.sync_status() == 0
    check_selection_all_rows(idx, q_h, k_h, Hkv, bs, topk, f"{pooling} pooling {case}", pooling=pooling, weights=w64)
    rows = oracle.all_rows(B, Hq, N) if B * Hq * N <= 20000 else sample_rows(B, Hq, N, bs, topk, 48, seed)
    kbar = oracle.pool(k_h, bs, pooling, w64)
    sel, _, _ = oracle.select(q_h, kbar, Hkv, bs, topk, rows)
    ref_out, ref_lse = oracle.attend(q_h, k_h, v_h, bs, topk, rows, sel)
    mism = (gather_idx(idx, rows) != sel).any(axis=1)  # excused near ties (checked above)
    go, gl = gather_rows(out, lse, rows)
    compare_outputs(go[~mism], gl[~mism], ref_out[~mism], ref_lse[~mism], pooling)


def test_weighted_pooling_with_equal_weights_is_the_mean(moba, cuda_dev):
    B, N, Hq, Hkv, bs, topk = 1, 20000, 4, 2, 300, 6
    q, k, _ = synth.inputs(B, N, Hq, Hkv, 128, bs, 32)
    q, k = q.to(cuda_dev), k.to(cuda_dev)
    w = torch.full((bs,), 0.75, dtype=torch.float32, device=cuda_dev)
    a = moba.gate(q, k, bs, topk)
    b = moba.gate(q, k, bs, topk, pooling="weighted", pool_weights=w)
    assert moba.sync_status() == 0
    assert torch.equal(a, b)


def test_invalid_pooling_weights_are_reported(moba, cuda_dev):
    B, N, Hq, Hkv, bs, topk = 1, 2048, 1, 1, 256, 3
    q, k, _ = synth.inputs(B, N, Hq, Hkv, 128, bs, 33)
    q, k = q.to(cuda_dev), k.to(cuda_dev)
    w = torch.ones(bs, dtype=torch.float32, device=cuda_dev)
    w[7] = -1.0
    moba.gate(q, k, bs, topk, pooling="weighted", pool_weights=w)
    assert moba.sync_status() == 10  # MOBA_ERR_VALUE
    assert moba.sync_status() == 0   # cleared


def test_full_attention_layer_is_dense_causal(moba, cuda_dev):
    """The hybrid-layer switch: full_attention=True ignores the gate and attends every earlier key."""
    B, N, Hq, Hkv, bs, topk = 1, 1500, 4, 2, 128, 3
    q_h, k_h, v_h = synth.inputs(B, N, Hq, Hkv, 128, bs, 34)
    q, k, v = q_h.to(cuda_dev), k_h.to(cuda_dev), v_h.to(cuda_dev)
    out, lse = moba.forward(q, k, v, bs, topk, full_attention=True)
    assert moba.sync_status() == 0
    rows = oracle.all_rows(B, Hq, N)
    nblk = (N + bs - 1) // bs
    r = oracle.forward(q_h, k_h, v_h, bs, nblk, rows)  # every block selected: dense causal
    go, gl = gather_rows(out, lse, rows)
    compare_outputs(go, gl, r["out"], r["lse"], "full attention layer")
