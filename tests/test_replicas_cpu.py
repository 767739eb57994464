"""Multi-rank host logic of bench.py on CPU: two gloo ranks, as `torchrun --nproc-per-node 2` starts them.

The decode step has no exchange step, so `bench.py --gpus N` runs N independent replicas; the only
cross-rank traffic is the timing reduction (max over ranks) and the barrier around the timed region.
These tests run that logic with world size 2 on the gloo backend: no GPU is involved.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

HERE = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, HERE)
    import torch
    import bench
    w, r, local = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    dist.barrier()
    # each rank's timed region; the job time is the slowest rank's
    t_ms = 10.0 * (r + 1)
    t_max = bench.max_over_ranks(t_ms, w, torch.device("cpu"))
    us = bench.whole_job_us_per_layer(t_max, 5, w)
    # the reference arm runs on rank 0 only; the other ranks return without work
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    other = bench.reference_arm(args, w, r) if r != 0 else (None, r)
    q.put((r, w, local, t_max, us, other[0] is None))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_time_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    for rank, world, local, t_max, us, no_ref_work in res:
        assert world == 2 and local == rank
        assert t_max == pytest.approx(20.0)  # the slower rank's 20 ms on both ranks
        assert us == pytest.approx(20.0 * 1000.0 / (5 * 2))  # whole job: 10 layer-steps in 20 ms
        assert no_ref_work
