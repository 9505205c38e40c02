"""The backward's results do not depend on how its independent chains are
scheduled: on the layer's side streams (router gradient, the two
weight-gradient GEMMs, each joined back by events), or in order on the
caller's stream (moe_set_side_streams(False), and what the library does by
itself when the weight-gradient GEMMs are large).  Every kernel's output is
deterministic, so the two schedules must give bit-identical y, dx, dW_r,
dW13, dW_down (and the shared expert's), dg and dlogits.
"""
from __future__ import annotations

import pytest
import torch

import workloads as W
from tests.test_gpu_parity import run_gpu

pytestmark = pytest.mark.gpu

OUTPUTS = ("y", "dx", "dw_r", "dw13", "dw_down", "dw13_s", "dw_down_s", "dg", "dlogits")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_routing_fp32_b200.build import build
    build()


@pytest.mark.parametrize("name", ["olmoe", "mix_pair", "ds3", "mm_b", "olmoe_ec"])
def test_backward_results_do_not_depend_on_streams(name):
    from mixture_experts_routing_fp32_b200 import api
    cfg = W.REDUCED[name]
    runs = []
    for side in (True, False):
        prev = api.moe_set_side_streams(side)
        try:
            layer, _ = run_gpu(cfg)
        finally:
            api.moe_set_side_streams(prev)
        runs.append({n: getattr(layer, n).clone() for n in OUTPUTS
                     if getattr(layer, n, None) is not None})
    assert runs[0].keys() == runs[1].keys()
    for n in runs[0]:
        assert torch.equal(runs[0][n], runs[1][n]), n
    print("%s: side-stream and in-order backward bit-identical (%s)"
          % (name, ", ".join(sorted(runs[0]))))
