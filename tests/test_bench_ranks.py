"""Host logic of bench.py's multi-rank path on CPU: two gloo ranks check the
max-over-ranks device time, the whole-job sum of useful work and the
per-rank seed offsets that make the replicas' batches independent."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        ms = 10.0 + 5.0 * r                      # rank 1 is the slower one
        useful = 1.0e12 * (r + 1)
        out.put((r, w, local, bench.max_over_ranks(ms, w), bench.sum_over_ranks(useful, w),
                 bench.rank_seed_offset(r)))
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions_and_seeds():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, w, local, ms_max, useful_sum, seed_off) in enumerate(res):
        assert (rank, w, local) == (r, world, r)
        assert ms_max == 15.0                    # the max over ranks, on every rank
        assert useful_sum == 3.0e12              # whole-job work
    assert len({x[5] for x in res}) == world     # independent draws per rank
    assert res[0][5] == 0                        # rank 0 keeps the single-GPU seed


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(2.0, 1) == 2.0
