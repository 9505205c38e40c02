"""moe_dispatch_static — the dispatch entry point that allocates nothing.

It serves callers that are given only their input and output buffers and
cannot allocate device memory (a plugin or custom-op host with no workspace
hook, a serving runtime with a fixed memory plan).  Its scratch is a static
device array inside libmoe.so, so this test calls it through the C ABI twice
in a row and checks every output against moe_dispatch (which takes a
caller-allocated workspace) on the same inputs.  Dispatch is integer and
copy work, so the match must be exact.

Kept in a file of its own that pytest collects last; it passes alone in a
fresh process and after the other tests.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def _buffers(layer_like, cfg, R, T, K, E, D, dt):
    i32 = torch.int32
    return dict(
        counts=torch.empty(E, dtype=i32, device="cuda"),
        kept=torch.empty(E, dtype=i32, device="cuda"),
        offsets=torch.empty(E + 2, dtype=i32, device="cuda"),
        slot_row=torch.empty(T * K, dtype=i32, device="cuda"),
        row_slot=torch.empty(R, dtype=i32, device="cuda"),
        tile_expert=torch.empty(R // 128, dtype=i32, device="cuda"),
        stats=torch.empty(4, dtype=i32, device="cuda"),
        x_perm=torch.empty(R, D, dtype=dt, device="cuda"),
    )


def _route(cfg):
    """Router output for cfg (the existing entry points), plus x and mask."""
    from mixture_experts_routing_fp32_b200 import MoELayer, config_from, api
    layer = MoELayer(config_from(cfg))
    x = W.make_input(cfg, "x", "cuda")
    off = W.make_input(cfg, "logit_offset", "cuda") if cfg.hot_expert_offset else None
    bias = W.make_input(cfg, "sel_bias", "cuda") if cfg.sel_bias_range else None
    mask = W.make_input(cfg, "sentinel_mask", "cuda") if cfg.sentinel_frac else None
    api.moe_router(layer.cfg, x, W.make_input(cfg, "w_r", "cuda"), off, bias, layer.logits,
                   layer.probs, layer.lse, layer.topk_idx, layer.topk_w, layer.near_ties,
                   layer.ws)
    return layer, x, mask


def _check_one(cfg):
    from mixture_experts_routing_fp32_b200 import api
    from mixture_experts_routing_fp32_b200._lib import lib, MOE_OK
    layer, x, mask = _route(cfg)
    c = layer.cfg
    R = int(layer.sizes.rows_max)
    ref = _buffers(layer, cfg, R, cfg.T, cfg.K, cfg.E, cfg.D, x.dtype)
    got = _buffers(layer, cfg, R, cfg.T, cfg.K, cfg.E, cfg.D, x.dtype)
    for b in got.values():
        b.fill_(-7) if b.dtype == torch.int32 else b.fill_(3.0)
    # existing entry point, caller-allocated workspace
    api.moe_dispatch(c, layer.topk_idx, mask, x, ref["counts"], ref["kept"], ref["offsets"],
                     ref["slot_row"], ref["row_slot"], ref["tile_expert"], ref["stats"],
                     ref["x_perm"], layer.ws)
    # the allocation-free entry point, called directly through the C ABI
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    rc = lib().moe_dispatch_static(
        ctypes.byref(c), p(layer.topk_idx), p(mask), p(x), p(got["counts"]), p(got["kept"]),
        p(got["offsets"]), p(got["slot_row"]), p(got["row_slot"]), p(got["tile_expert"]),
        p(got["stats"]), p(got["x_perm"]),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == MOE_OK
    assert api.moe_check_status() == 0
    n_rows = int(ref["stats"][2])
    for k in ("counts", "kept", "offsets", "slot_row", "stats"):
        assert torch.equal(got[k], ref[k]), k
    assert torch.equal(got["row_slot"][:n_rows], ref["row_slot"][:n_rows])
    assert torch.equal(got["tile_expert"][:n_rows // 128], ref["tile_expert"][:n_rows // 128])
    assert torch.equal(got["x_perm"][:n_rows], ref["x_perm"][:n_rows])


def test_static_dispatch_matches_workspace_dispatch_two_calls():
    from mixture_experts_routing_fp32_b200.build import build
    build()
    # two calls in a row on different problems: the second reuses the
    # static scratch the first left behind
    _check_one(W.REDUCED["olmoe"])   # sentinel slots, E = 64, K = 8
    _check_one(W.REDUCED["mix"])     # capacity drops, hot-spot expert


def test_static_dispatch_rejects_problems_beyond_its_scratch():
    from mixture_experts_routing_fp32_b200 import api
    from mixture_experts_routing_fp32_b200._lib import lib, MOE_ERR_ARG
    # ceil(T*K/4096) * (E+1) * 4 bytes > 1 MiB: rejected before any launch
    c = api.make_config(T=1 << 21, D=64, E=256, K=8, F=64)
    rc = lib().moe_dispatch_static(ctypes.byref(c), *([ctypes.c_void_p(16)] * 11), None)
    assert rc == MOE_ERR_ARG
