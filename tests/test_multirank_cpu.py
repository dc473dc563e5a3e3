"""The N > 1 host logic of bench.py on CPU: two gloo ranks combine their timings as
max-over-ranks elapsed time and summed work, exactly as the NCCL path does on GPUs."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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
    import bench
    ms, units = bench.aggregate(100.0 + 50.0 * rank, 1e12 * (rank + 1), world)
    q.put((rank, ms, units))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_like_the_bench():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, ms, units in res:
        assert ms == 150.0          # the slowest rank's time
        assert units == 3e12        # work of both ranks


def test_single_rank_aggregate_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(12.5, 7.0, 1) == (12.5, 7.0)


def test_reference_arm_on_cpu_prints_contract_line(capsys):
    import json
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0", "--seq-len", "8192",
                       "--sample-rows", "64"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
