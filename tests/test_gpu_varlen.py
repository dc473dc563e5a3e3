"""GPU parity of packed (varlen) batches against the oracle's per-sequence definition: the
selection of every token (near ties excused, counted and bounded), the outputs and lse of every
token. Lengths mix sequences shorter than a block, a single token, empty sequences, runs of equal
length (batched together) and lengths that are not multiples of the block size."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import SelectionReport, compare_outputs, sample_rows

pytestmark = pytest.mark.gpu


def _packed(lens, Hq, Hkv, bs, seed):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    total = int(cu[-1])
    q, k, v = synth.inputs(1, total, Hq, Hkv, 128, bs, seed)
    return cu, q[0], k[0], v[0]


CASES = [  # lengths, Hq, Hkv, block_size, topk, seed
    ([5000, 1, 4096, 300, 0, 12345, 777], 4, 2, 512, 3, 80),
    ([2048, 2048, 2048, 1000, 1000, 3000], 8, 2, 256, 5, 81),
    ([65536, 131072, 32768], 8, 2, 4096, 12, 82),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n{len(c[0])}_bs{c[3]}_k{c[4]}")
def test_varlen_against_the_oracle(moba, cuda_dev, case):
    """Selection of every token; outputs of every token of short sequences and of a seeded row
    sample (block edges included) of long ones."""
    lens, Hq, Hkv, bs, topk, seed = case
    cu, q_h, k_h, v_h = _packed(lens, Hq, Hkv, bs, seed)
    q, k, v = q_h.to(cuda_dev), k_h.to(cuda_dev), v_h.to(cuda_dev)
    out, lse = moba.forward_varlen(q, k, v, cu, bs, topk)
    idx = moba.gate_varlen(q, k, cu, bs, topk)
    assert moba.sync_status() == 0
    rep = SelectionReport(f"varlen {lens}")
    gsel = idx.cpu().numpy()  # [Hq, total, topk]
    o = out.float().cpu().numpy()  # [total, Hq, d]
    l = lse.cpu().numpy()          # [Hq, total]
    for s in range(len(lens)):
        a, b = int(cu[s]), int(cu[s + 1])
        if b <= a:
            continue
        qs, ks, vs = (x[a:b].unsqueeze(0).contiguous() for x in (q_h, k_h, v_h))
        kbar = oracle.pool(ks, bs)
        rows = oracle.all_rows(1, Hq, b - a)
        sel, s_last, s_next = oracle.select(qs, kbar, Hkv, bs, topk, rows)
        mism = rep.add(gsel[rows[:, 1], a + rows[:, 2]], sel, s_last, s_next)
        orows = rows if (b - a) * Hq <= 40000 else sample_rows(1, Hq, b - a, bs, topk, 64, seed + s)
        osel, _, _ = oracle.select(qs, kbar, Hkv, bs, topk, orows)
        ref_o, ref_l = oracle.attend(qs, ks, vs, bs, topk, orows, osel)
        bad = (gsel[orows[:, 1], a + orows[:, 2]] != osel).any(axis=1)  # excused near ties
        go = o[a + orows[:, 2], orows[:, 1]]
        gl = l[orows[:, 1], a + orows[:, 2]]
        compare_outputs(go[~bad], gl[~bad], ref_o[~bad], ref_l[~bad], f"varlen sequence {s}")
    rep.finish()


def test_varlen_full_attention_layer(moba, cuda_dev):
    lens = [3000, 17, 2500]
    cu, q_h, k_h, v_h = _packed(lens, 4, 1, 256, 83)
    q, k, v = q_h.to(cuda_dev), k_h.to(cuda_dev), v_h.to(cuda_dev)
    out, lse = moba.forward_varlen(q, k, v, cu, 256, 3, full_attention=True)
    assert moba.sync_status() == 0
    r = oracle.forward_varlen(q_h, k_h, v_h, cu, 256, 64)  # every block kept: dense causal per sequence
    compare_outputs(out.float().cpu().numpy().reshape(-1, 128), lse.cpu().numpy().T.reshape(-1),
                    r["out"].reshape(-1, 128), r["lse"].T.reshape(-1), "varlen full attention")
