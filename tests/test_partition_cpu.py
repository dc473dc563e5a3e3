"""The split of one forward across ranks by kv-head groups, on CPU: which heads each rank
owns, and that the per-rank results reassembled on rank 0 equal the one-rank forward.

Two gloo ranks each draw only their own head slices of the seeded inputs and run the
fp64 oracle on them (the CPU stand-in for the per-rank GPU forward); rank 0 gathers the
slices and reassembles them. Every row depends only on its own head, so the result must
equal the oracle on the whole layout bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_gate_b200 import partition

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPE = dict(B=2, N=300, Hq=8, Hkv=4, d=16, bs=32, topk=3, seed=13)


@pytest.mark.parametrize("Hq,Hkv,world", [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8), (32, 8, 3),
                                          (12, 6, 4), (5, 5, 5), (4, 1, 1)])
def test_head_slices_cover_every_head_once(Hq, Hkv, world):
    sl = partition.head_slices(Hq, Hkv, world)
    assert [s.rank for s in sl] == list(range(world))
    kv = [h for s in sl for h in range(s.hkv0, s.hkv1)]
    qh = [h for s in sl for h in range(s.hq0, s.hq1)]
    assert kv == list(range(Hkv)) and qh == list(range(Hq))
    sizes = [s.n_kv for s in sl]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    G = Hq // Hkv
    for s in sl:  # a rank's query heads are exactly those that read its kv heads
        assert all(s.hkv0 <= h // G < s.hkv1 for h in range(s.hq0, s.hq1))


def test_cannot_split_fewer_kv_heads_than_ranks():
    assert not partition.can_split(1, 1, 2)
    with pytest.raises(ValueError):
        partition.head_slices(8, 2, 4)


def _to_layout(r, B, N, nq, d):
    """Oracle rows (b, h, t) -> out [B, N, nq, d], lse [B, nq, N] tensors."""
    out = torch.zeros(B, N, nq, d, dtype=torch.float64)
    lse = torch.zeros(B, nq, N, dtype=torch.float64)
    rows = torch.from_numpy(r["rows"])
    out[rows[:, 0], rows[:, 2], rows[:, 1]] = torch.from_numpy(r["out"])
    lse[rows[:, 0], rows[:, 1], rows[:, 2]] = torch.from_numpy(r["lse"])
    return out, lse


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    import synth
    from block_sparse_long_gate_b200 import partition as part
    S = SHAPE
    sl = part.head_slices(S["Hq"], S["Hkv"], world)[rank]
    qh, kh, vh = synth.inputs_heads(S["B"], S["N"], S["Hq"], S["Hkv"], S["d"], S["bs"], S["seed"], sl.hkv0, sl.hkv1)
    r = oracle.forward(qh, kh, vh, S["bs"], S["topk"])
    out, lse = _to_layout(r, S["B"], S["N"], sl.n_q, S["d"])
    outs = [torch.zeros_like(out) for _ in range(world)] if rank == 0 else None
    lses = [torch.zeros_like(lse) for _ in range(world)] if rank == 0 else None
    dist.gather(out, outs, dst=0)
    dist.gather(lse, lses, dst=0)
    if rank == 0:
        slices = part.head_slices(S["Hq"], S["Hkv"], world)
        full_out, full_lse = part.assemble(list(zip(slices, outs, lses)), S["Hq"], S["Hkv"])
        q.put((full_out.numpy(), full_lse.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reassemble_the_one_rank_forward():
    import oracle
    import synth
    S = SHAPE
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, qq)) for r in range(2)]
    for p in procs:
        p.start()
    got_out, got_lse = qq.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    q, k, v = synth.inputs(S["B"], S["N"], S["Hq"], S["Hkv"], S["d"], S["bs"], S["seed"])
    want_out, want_lse = _to_layout(oracle.forward(q, k, v, S["bs"], S["topk"]), S["B"], S["N"], S["Hq"], S["d"])
    np.testing.assert_array_equal(got_out, want_out.numpy())
    np.testing.assert_array_equal(got_lse, want_lse.numpy())


def test_assemble_rejects_missing_or_repeated_heads():
    sl = partition.head_slices(8, 4, 2)
    o = torch.zeros(1, 4, 4, 16)
    l = torch.zeros(1, 4, 4)
    with pytest.raises(ValueError):
        partition.assemble([(sl[0], o, l)], 8, 4)
    with pytest.raises(ValueError):
        partition.assemble([(sl[0], o, l), (sl[0], o, l)], 8, 4)


def test_synth_head_slices_equal_the_whole_tensors():
    import synth
    q, k, v = synth.inputs(2, 200, 8, 4, 32, 48, 5)
    for h0, h1 in [(0, 4), (1, 3), (3, 4)]:
        a, b, c = synth.inputs_heads(2, 200, 8, 4, 32, 48, 5, h0, h1)
        assert torch.equal(a, q[:, :, 2 * h0:2 * h1]) and torch.equal(b, k[:, :, h0:h1])
        assert torch.equal(c, v[:, :, h0:h1])
