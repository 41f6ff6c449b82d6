"""Multi-rank plumbing of bench.py on CPU: two gloo ranks (127.0.0.1), each with
its own seed (weak scaling: every rank decodes its own batch) and the max of
their timings taken over ranks. No GPU, no data-path collective."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.dist_env()
        seed = bench.rank_seed("omni3b-b1", r)
        mine = [10.0 + r, 5.0 - r]
        got = bench.max_over_ranks(mine, torch.device("cpu"), w)
        dist.barrier()
        results[rank] = (w, seed, got)
    finally:
        dist.destroy_process_group()


def test_two_ranks_seeds_and_max():
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(results)
    assert res[0][0] == 2 and res[1][0] == 2
    assert res[0][1] != res[1][1]                    # each rank its own batch
    assert res[0][2] == res[1][2] == [11.0, 5.0]     # max over ranks, elementwise


def test_single_rank_max_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu"), 1) == [3.0, 4.0]
