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


def _aux_worker(rank, world, port, out):
    """One data-parallel rank of the OLMoE-shaped reduced layer (aux + z
    loss, sentinel slots, no capacity limit) holding half of the batch: its
    local statistics go through the package's exchange functions, then the
    oracle's formulas on the summed statistics must give the full batch's
    losses, its rows of the router gradient, and (after the weight-gradient
    all-reduce) the full batch's weight gradients."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    import numpy as np
    import torch.distributed as dist
    import workloads as W
    from oracle import moe_oracle as O
    from tests.helpers import oracle_layer
    from mixture_experts_routing_fp32_b200.dist import allreduce_aux_stats, \
        allreduce_weight_grads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    cfg = W.REDUCED["olmoe"]
    T, E, K = cfg.T, cfg.E, cfg.K
    L = oracle_layer(cfg)
    o = O.opts_of(cfg)
    dy = W.make_input(cfg, "dy").double().numpy()
    fw = O.forward(L, o)
    bw = O.backward(L, o, fw, dy)          # the whole batch (the target)
    # this rank's half of the batch
    rows = np.arange(rank * T // world, (rank + 1) * T // world)
    from dataclasses import replace
    Lh = replace(L, x=L.x[rows], sentinel_mask=L.sentinel_mask.reshape(T, K)[rows].reshape(-1))
    fh = O.forward(Lh, o)
    Rh, Dh = fh["R"], fh["Dp"]
    counts = torch.tensor(Dh.counts, dtype=torch.int32)
    sums = torch.tensor(np.concatenate([Rh.p.sum(0), [(Rh.lse ** 2).sum()]]),
                        dtype=torch.float64)
    allreduce_aux_stats(counts, sums)
    n_tok = T
    aux = O.aux_loss_from_stats(counts.numpy(), sums[:E].numpy(), n_tok, cfg.aux_alpha, E)
    z = cfg.z_lambda * float(sums[E]) / n_tok
    # this rank's share of the gradient of the global losses
    dsh = O.router_backward(Rh, bw["dg"][rows], o, counts.numpy(), T_total=n_tok)
    bh = O.backward(Lh, o, fh, dy[rows])
    dw_r = torch.from_numpy(dsh.T @ Lh.x)
    dw13 = torch.from_numpy(np.stack([bh["dw13"][e] for e in range(E)]))
    dwd = torch.from_numpy(np.stack([bh["dwd"][e] for e in range(E)]))
    allreduce_weight_grads([dw_r, dw13, dwd], bucket_bytes=1 << 16)
    rel = lambda a, b: float(np.linalg.norm(a - b) / np.linalg.norm(b))
    out[rank] = dict(
        aux=abs(aux - fw["aux"]) / fw["aux"], z=abs(z - fw["z"]) / fw["z"],
        ds=rel(dsh, bw["ds"][rows]), dw_r=rel(dw_r.numpy(), bw["dw_r"]),
        dw13=rel(dw13.numpy(), np.stack([bw["dw13"][e] for e in range(E)])),
        dwd=rel(dwd.numpy(), np.stack([bw["dwd"][e] for e in range(E)])),
        local_aux_differs=abs(fh["aux"] - fw["aux"]) > 1e-6 * fw["aux"])
    dist.destroy_process_group()


def test_global_aux_stats_and_weight_grads_two_ranks_gloo():
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_aux_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    for r in range(2):
        d = dict(out[r])
        assert d.pop("local_aux_differs")     # the exchange is what makes them agree
        for k, v in d.items():
            assert v < 1e-12, (r, k, v)
