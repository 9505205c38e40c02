"""Expert parallelism through the C ABI on one GPU (replicated-token form).

Each shard is a layer call holding a range of the routed experts
(cfg.expert_base, cfg.n_local_experts): it routes all tokens over all
experts, its dispatch turns the other experts' slots into sentinels (no
row, zero expert output, zero gate gradient — the [HF48687] requirement),
and its expert GEMMs run on its own experts only.  Two shards run one after
the other (no kernel waits on another); y, dx, dW_r, dlogits and dg summed
over the shards must equal the unsharded layer and the oracle on the whole
layer, and each shard's expert weight gradients must be the layer's for
those experts.  The aux and z losses are added on shard 0 only; they use
the global expert counts every shard's dispatch reports.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads as W
from tests.helpers import rel_l2
from tests.test_gpu_parity import gpu_inputs, host, oracle_on_gpu_routing, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_routing_fp32_b200.build import build
    build()


@pytest.mark.parametrize("name", ["olmoe", "mix", "mix_pair", "mm_mask"])
def test_expert_shards_sum_to_the_layer(name):
    from mixture_experts_routing_fp32_b200 import MoELayer, config_from, moe_check_status
    cfg = W.REDUCED[name]
    E = cfg.E
    full, inp = run_gpu(cfg)
    fw, bw, flips = oracle_on_gpu_routing(cfg, full)
    cuts = [0, E // 2, E] if E > 2 else [0, 1, E]
    tot = {}
    for i, (lo, hi) in enumerate(zip(cuts[:-1], cuts[1:])):
        c = config_from(cfg, expert_base=lo, n_local_experts=hi - lo,
                        aux_alpha=cfg.aux_alpha if i == 0 else 0.0,
                        z_lambda=cfg.z_lambda if i == 0 else 0.0)
        lay = MoELayer(c)
        lay.forward(inp["x"], inp["w_r"], inp["w13"][lo:hi].contiguous(),
                    inp["w_down"][lo:hi].contiguous(), logit_offset=inp["logit_offset"],
                    sel_bias=inp["sel_bias"], sentinel_mask=inp["sentinel_mask"])
        lay.backward(inp["dy"])
        assert moe_check_status() == 0
        # the same global routing and counts as the unsharded layer
        assert torch.equal(lay.topk_idx, full.topk_idx)
        assert torch.equal(lay.counts, full.counts)
        assert torch.equal(lay.kept, full.kept[lo:hi])
        if i == 0:
            assert torch.equal(lay.losses, full.losses)
        # slots of other shards' experts: no row, zero gate gradient
        sr = lay.slot_row.view(cfg.T, cfg.K)
        other = (full.topk_idx < lo) | (full.topk_idx >= hi)
        assert bool((sr[other] == -2).all())
        assert bool((lay.dg[sr < 0] == 0).all())
        # expert weight gradients: the layer's for these experts
        tl = 2e-2
        assert rel_l2(host(lay.dw13), np.stack([bw["dw13"][e] for e in range(lo, hi)])) < tl
        assert rel_l2(host(lay.dw_down), np.stack([bw["dwd"][e] for e in range(lo, hi)])) < tl
        assert rel_l2(host(lay.dw13), host(full.dw13[lo:hi])) < 1e-2
        for k in ("y", "dx", "dw_r", "dlogits", "dg"):
            v = getattr(lay, k).float()
            tot[k] = v if k not in tot else tot[k] + v
    for k, ref in (("y", fw["y"]), ("dx", bw["dx"]), ("dw_r", bw["dw_r"]),
                   ("dlogits", bw["ds"]), ("dg", bw["dg"])):
        assert rel_l2(host(tot[k]), ref) < 2e-2, k
        assert rel_l2(host(tot[k]), host(getattr(full, k))) < 1e-2, k
    print("%s: 2 expert shards sum to the layer (near-tie flips %d)" % (name, flips))
