"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Data-parallel replicas: every rank draws its own tokens with the shared
weights, the timed value is the max over ranks, and only rank 0 reports.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    import workloads as W
    r, w, _ = bench.dist_init(world, backend="gloo")
    assert (r, w) == (rank, world)
    cfg = bench.rank_config(W.CONFIGS["tiny"], r)
    x = W.make_input(cfg, "x")
    wr = W.make_input(W.CONFIGS["tiny"], "w_r")
    bench.barrier(w)
    ms = 1.0 + 2.0 * r
    mx = bench.max_over_ranks(ms, w, "cpu")
    import torch.distributed as dist
    xs = [torch.empty_like(x) for _ in range(w)]
    dist.all_gather(xs, x)
    wrs = [torch.empty_like(wr) for _ in range(w)]
    dist.all_gather(wrs, wr)
    out[rank] = (mx, not torch.equal(xs[0], xs[1]), torch.equal(wrs[0], wrs[1]))
    dist.destroy_process_group()


def test_two_rank_replicas_gloo():
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    for r in range(2):
        mx, tokens_differ, weights_same = out[r]
        assert mx == 3.0                  # max over ranks
        assert tokens_differ and weights_same
