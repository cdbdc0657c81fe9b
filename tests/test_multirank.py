"""The multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank runs an independent batch (weak scaling); the only collectives are
the barrier around the timed region and the max-over-ranks reduction of the
elapsed time, which these tests exercise without a GPU.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    assert bench.dist_init(w, "gloo")
    bench.barrier(None)
    mx = bench.reduce_max(float(10 * rank + 3), None)
    bench.barrier(None)
    import torch.distributed as dist
    dist.destroy_process_group()
    out[rank] = (mx, bench.rank_seed(0, rank))


def test_two_gloo_ranks_max_and_seeds():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 13.0          # max over ranks
    assert out[0][1] != out[1][1]                   # independent batches per rank


def test_single_rank_needs_no_process_group():
    assert bench.dist_init(1, "gloo") is False
    assert bench.reduce_max(4.5, None) == 4.5
