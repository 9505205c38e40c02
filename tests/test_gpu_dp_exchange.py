"""The data-parallel statistics exchange through the C ABI on one GPU.

Two ranks are emulated by two half-batch layers run one after the other
(no kernel waits on another); their statistics (moe_aux_stats) and expert
counts are summed, as the all-reduce would, and moe_aux_loss_global /
moe_backward with cfg.loss_tokens = the whole batch's token count must give
the whole batch's losses, each half's rows of the router gradient and, once
summed, the weight gradients — against the oracle on the whole batch
([STA324] §8.5: the balance statistic over the whole batch or all devices).
The layer's own path (MoELayer(aux_group=...)) runs on a one-rank NCCL group.
"""
from __future__ import annotations

import socket

import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O
from tests.helpers import oracle_layer, rel_l2
from tests.test_gpu_parity import gpu_inputs, host, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_routing_fp32_b200.build import build
    build()


def test_global_aux_matches_whole_batch_oracle_two_halves():
    from mixture_experts_routing_fp32_b200 import (MoELayer, api, config_from,
                                                   moe_check_status)
    cfg = W.REDUCED["olmoe"]          # aux + z, sentinels, no capacity limit
    T, E, K = cfg.T, cfg.E, cfg.K
    L = oracle_layer(cfg)
    o = O.opts_of(cfg)
    fw = O.forward(L, o)
    bw = O.backward(L, o, fw, W.make_input(cfg, "dy").double().numpy())
    inp = gpu_inputs(cfg)
    halves = [np.arange(0, T // 2), np.arange(T // 2, T)]
    layers, sums = [], []
    for rows in halves:
        sub = cfg.replace(T=len(rows))
        lay = MoELayer(config_from(sub, loss_tokens=T))
        r = torch.from_numpy(rows).cuda()
        mask = inp["sentinel_mask"].view(T, K)[r].reshape(-1).contiguous()
        x = inp["x"][r].contiguous()
        lay.forward(x, inp["w_r"], inp["w13"], inp["w_down"], sentinel_mask=mask)
        s = torch.empty(E + 1, dtype=torch.float32, device="cuda")
        api.moe_aux_stats(lay.cfg, lay.probs, lay.lse, s, lay.ws)
        layers.append((lay, r))
        sums.append(s)
    # the all-reduce of two ranks
    counts_g = layers[0][0].counts + layers[1][0].counts
    sums_g = sums[0] + sums[1]
    losses = torch.empty(2, dtype=torch.float32, device="cuda")
    api.moe_aux_loss_global(layers[0][0].cfg, counts_g, sums_g, losses)
    assert abs(float(losses[0]) - fw["aux"]) <= 1e-5 * fw["aux"]
    assert abs(float(losses[1]) - fw["z"]) <= 1e-5 * fw["z"]
    dw_r = torch.zeros(E, cfg.D, dtype=torch.float32, device="cuda")
    dw13 = torch.zeros(E, 2 * cfg.F, cfg.D, dtype=torch.float32, device="cuda")
    for lay, r in layers:
        dy = inp["dy"][r].contiguous()
        lay.backward(dy, loss_counts=counts_g)
        rows = r.cpu().numpy()
        assert rel_l2(host(lay.dlogits), bw["ds"][rows]) < 2e-2
        assert rel_l2(host(lay.dx), bw["dx"][rows]) < 2e-2
        dw_r += lay.dw_r
        dw13 += lay.dw13.float()
    assert moe_check_status() == 0
    assert rel_l2(host(dw_r), bw["dw_r"]) < 2e-2
    assert rel_l2(host(dw13), np.stack([bw["dw13"][e] for e in range(E)])) < 2e-2
    # the local (per-half) losses differ from the whole batch's: the exchange matters
    api.moe_aux_loss(layers[0][0].cfg, layers[0][0].probs, layers[0][0].lse,
                     layers[0][0].counts, losses, layers[0][0].ws)
    assert abs(float(losses[0]) - fw["aux"]) > 1e-4 * fw["aux"]


def test_global_aux_one_rank_equals_local_bit_for_bit():
    """With one rank the pooled path reproduces moe_aux_loss exactly, and
    MoELayer(aux_group=<one-rank NCCL group>) gives the same losses and
    gradients as the layer without a group."""
    import torch.distributed as dist
    from mixture_experts_routing_fp32_b200 import MoELayer, api, config_from
    cfg = W.REDUCED["olmoe"]
    ref, inp = run_gpu(cfg)
    s = torch.empty(cfg.E + 1, dtype=torch.float32, device="cuda")
    api.moe_aux_stats(ref.cfg, ref.probs, ref.lse, s, ref.ws)
    losses = torch.empty(2, dtype=torch.float32, device="cuda")
    api.moe_aux_loss_global(ref.cfg, ref.counts, s, losses)
    assert torch.equal(losses, ref.losses)
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0,
                            world_size=1)
    try:
        lay = MoELayer(config_from(cfg), aux_group=dist.group.WORLD)
        assert lay.cfg.loss_tokens == cfg.T
        lay.forward(inp["x"], inp["w_r"], inp["w13"], inp["w_down"],
                    sentinel_mask=inp["sentinel_mask"])
        lay.backward(inp["dy"])
        torch.cuda.synchronize()
        assert torch.equal(lay.counts_g, ref.counts)
        assert torch.equal(lay.losses, ref.losses)
        for a in ("dlogits", "dw_r", "dx", "dw13", "dw_down", "y"):
            assert torch.equal(getattr(lay, a), getattr(ref, a)), a
    finally:
        dist.destroy_process_group()
