"""GPU parity of the decode step (moba_pool_cache + moba_decode) against the fp64 oracle.

The step is the prefill definition at the last row: the selection of every (sequence, head) must
equal the oracle's (near ties excused, counted and bounded as in the prefill tests), the outputs
must meet max-abs 2e-2 / mean-abs 2e-3 and the lse 1e-3. Cases cover grouped-query heads (G = 1, 4,
8, 16), a cache longer than the sequence, lengths that end anywhere in a block (including the first
key of a block and a single token), few blocks (every earlier block kept), fine granularity
(block 256, top-32), max pooling, incremental pooling of a growing cache, and the full-attention
decode of a hybrid model."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import SelectionReport, compare_outputs

pytestmark = pytest.mark.gpu


def _run(moba, dev, B, L, Lmax, Hq, Hkv, bs, topk, seed, full=False, pooling="mean"):
    q_c, k_h, v_h = synth.inputs(B, Lmax, Hq, Hkv, 128, bs, seed)
    qd = synth.normal(seed + 1000, synth.Q_ID, (B, Hq, 128))
    k, v = k_h.to(dev), v_h.to(dev)
    kbar = moba.pool_cache(k, bs, L, pooling=pooling)
    out, lse, idx = moba.decode(qd.to(dev), k, v, kbar, bs, topk, L, full_attention=full)
    assert moba.sync_status() == 0
    r = oracle.decode(qd, k_h, v_h, bs, topk, L, pooling=pooling, full_attention=full)
    what = f"decode B={B} L={L} Hq={Hq} Hkv={Hkv} bs={bs} k={topk}" + (" full" if full else "") + f" {pooling}"
    mism = np.zeros(B * Hq, dtype=bool)
    if not full:
        rep = SelectionReport(what)
        mism = rep.add(idx.reshape(B * Hq, topk).cpu().numpy(), r["sel"], r["s_last"], r["s_next"])
        rep.finish()
    o = out.reshape(B * Hq, 128).float().cpu().numpy()
    l = lse.reshape(B * Hq).cpu().numpy()
    compare_outputs(o[~mism], l[~mism], r["out"][~mism], r["lse"][~mism], what)
    return kbar


CASES = [  # B, L, Lmax, Hq, Hkv, block_size, topk, seed
    (2, 5000, 5000, 8, 2, 512, 3, 50),          # GQA 4, ragged length
    (1, 131072, 131072, 32, 8, 4096, 12, 51),   # Llama-3.1-8B shape at 128K
    (3, 32768, 40000, 8, 1, 256, 32, 52),       # fine granularity, GQA 8, cache longer than the sequence
    (1, 20480, 20480, 16, 1, 2048, 4, 53),      # GQA 16; L - 1 is the last key of a block
    (2, 4097, 4200, 4, 4, 4096, 12, 54),        # the query is the first key of block 1
    (1, 1, 64, 2, 1, 128, 3, 55),               # a single token
    (1, 1500, 1500, 2, 2, 128, 20, 56),         # fewer blocks than k: every earlier block kept
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"L{c[1]}_H{c[3]}x{c[4]}_bs{c[5]}_k{c[6]}")
def test_decode_against_the_oracle(moba, cuda_dev, case):
    B, L, Lmax, Hq, Hkv, bs, topk, seed = case
    _run(moba, cuda_dev, B, L, Lmax, Hq, Hkv, bs, topk, seed)


@pytest.mark.parametrize("case", [(2, 5000, 5000, 8, 2, 512, 3, 60), (1, 65536, 65536, 8, 2, 4096, 12, 61)])
def test_full_attention_decode(moba, cuda_dev, case):
    B, L, Lmax, Hq, Hkv, bs, topk, seed = case
    _run(moba, cuda_dev, B, L, Lmax, Hq, Hkv, bs, topk, seed, full=True)


def test_decode_with_max_pooling(moba, cuda_dev):
    _run(moba, cuda_dev, 1, 70000, 70000, 8, 2, 1024, 6, 62, pooling="max")


def test_pool_cache_grows_with_the_cache(moba, cuda_dev):
    """Pooling only the newly full blocks of a growing cache gives the summaries of pooling all."""
    B, Lmax, Hkv, bs = 2, 9000, 2, 1000
    _, k_h, _ = synth.inputs(B, Lmax, 2, Hkv, 128, bs, 63)
    k = k_h.to(cuda_dev)
    rows = Lmax // bs
    grow = torch.zeros((B, Hkv, rows, 128), dtype=torch.float64, device=cuda_dev)
    done = 0
    for L in (999, 1000, 3500, 6001, 9000):
        moba.pool_cache(k, bs, L, kbar=grow, first_block=done)
        done = L // bs
    whole = moba.pool_cache(k, bs, Lmax)
    assert moba.sync_status() == 0
    assert torch.equal(grow, whole)
    np.testing.assert_allclose(whole.cpu().numpy(), oracle.pool(k_h, bs), rtol=0, atol=1e-15)
