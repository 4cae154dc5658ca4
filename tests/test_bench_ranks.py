"""bench.py's multi-rank plumbing on CPU (gloo, two ranks): the reported time is the slowest rank's,
and every rank quantizes its own layer of the same shape."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from post_weight_quantization_21_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, world, rank)
        ms = bench.slowest_rank_ms(10.0 + 5.0 * rank, torch.device("cpu"))
        L = bench.layer_for_rank(wl.LAYERS["tiny_64x128"], rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, L.seed)
        out[rank] = (ms, tuple(seeds), (L.m, L.d, L.n_tokens))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_time_and_own_layers():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0          # max over ranks
    assert len(set(res[0][1])) == world             # distinct layer seeds
    assert res[0][2] == res[1][2]                   # same shape on every rank


def test_single_process_time_is_unchanged():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.slowest_rank_ms(3.25, torch.device("cpu")) == 3.25
