"""moe_dispatch_static — the dispatch entry point that allocates nothing.

It serves callers that are given only their input and output buffers and
cannot allocate device memory (a plugin or custom-op host with no workspace
hook, a serving runtime with a fixed memory plan).  Its scratch — the
per-block expert histograms of the multi-block dispatch — is a static device
array inside libmoe.so.  These tests call it through the C ABI on several
problems in a row, each large enough (more than 16384 slots) that the
histogram passes run on that array, and check every output against
moe_dispatch (which takes a caller-allocated workspace) on the same inputs;
then they pin the array's size limit from both sides.  Dispatch is integer
and copy work, so the match must be exact.

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
    assert cfg.T * cfg.K > SMALL_SLOTS     # the multi-block passes: scratch in use
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


KDISP = 4096          # slots per histogram block of the multi-block dispatch
SMALL_SLOTS = 16384   # up to this many slots one block does the whole dispatch


def _problems():
    """Three routed problems with more than SMALL_SLOTS slots, so each call
    runs the multi-block histogram / scan / rank passes whose per-block
    histograms live in the static scratch.  They differ in E and in block
    count, so scratch left behind by one call would show up in the next."""
    return [
        # DeepSeek-shaped options (sigmoid + bias, groups, shared expert), E = 256
        W.REDUCED["ds3"].replace(name="ds3_static", T=3000),
        # OLMoE-shaped: 10% sentinel slots, E = 64
        W.REDUCED["olmoe_multi"],
        # Mixtral-shaped: capacity drops on the hot-spot expert, E = 8
        W.REDUCED["mix"].replace(name="mix_static", T=9000, D=256),
    ]


def test_static_dispatch_matches_workspace_dispatch_consecutive_calls():
    from mixture_experts_routing_fp32_b200.build import build
    build()
    probs = _problems()
    for cfg in probs:
        assert cfg.T * cfg.K > SMALL_SLOTS, cfg.name
    assert len({(c.E, -(-c.T * c.K // KDISP)) for c in probs}) == len(probs)
    for cfg in probs + probs[:1]:     # and the first one again, after the others
        _check_one(cfg)


def _random_idx(T, K, E, seed):
    """Random expert ids (some -1 sentinels) made on the device."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    idx = torch.randint(0, E, (T, K), device="cuda", generator=g, dtype=torch.int32)
    sent = torch.rand((T, K), device="cuda", generator=g) < 0.05
    return torch.where(sent, torch.full_like(idx, -1), idx)


def _dispatch_both(c, T, K, E, D, idx):
    """moe_dispatch (workspace) and moe_dispatch_static on the same routing,
    layout only (x_perm NULL): the part of the dispatch that uses scratch."""
    from mixture_experts_routing_fp32_b200 import api
    from mixture_experts_routing_fp32_b200._lib import lib, MOE_OK
    sizes = api.moe_get_sizes(c)
    R = int(sizes.rows_max)
    x = torch.zeros(T, D, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(int(sizes.ws_bytes), dtype=torch.uint8, device="cuda")
    ref = _buffers(None, None, R, T, K, E, 8, torch.bfloat16)
    got = _buffers(None, None, R, T, K, E, 8, torch.bfloat16)
    for b in got.values():
        b.fill_(-7) if b.dtype == torch.int32 else b.fill_(3.0)
    api.moe_dispatch(c, idx, None, x, ref["counts"], ref["kept"], ref["offsets"],
                     ref["slot_row"], ref["row_slot"], ref["tile_expert"], ref["stats"],
                     None, ws)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib().moe_dispatch_static(
        ctypes.byref(c), p(idx), None, p(x), p(got["counts"]), p(got["kept"]),
        p(got["offsets"]), p(got["slot_row"]), p(got["row_slot"]), p(got["tile_expert"]),
        p(got["stats"]), None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == MOE_OK
    assert api.moe_check_status() == 0
    n_rows = int(ref["stats"][2])
    for k in ("counts", "kept", "offsets", "slot_row", "stats"):
        assert torch.equal(got[k], ref[k]), k
    assert torch.equal(got["row_slot"][:n_rows], ref["row_slot"][:n_rows])
    assert torch.equal(got["tile_expert"][:n_rows // 128], ref["tile_expert"][:n_rows // 128])


def test_static_dispatch_size_limit_both_sides():
    """The scratch holds ceil(T*K / 4096) * (E + 1) int32 entries.  At E = 256
    the largest accepted problem has 1020 histogram blocks (T*K = 4,177,920
    slots): it runs and matches moe_dispatch; one more block is rejected with
    MOE_ERR_ARG before any launch, although the config itself is valid."""
    from mixture_experts_routing_fp32_b200 import api
    from mixture_experts_routing_fp32_b200._lib import lib, MOE_ERR_ARG, MOE_OK
    E, K, D = 256, 8, 64
    limit = 1 << 20
    blocks = limit // ((E + 1) * 4)                # 1020
    T_ok = blocks * KDISP // K
    assert -(-T_ok * K // KDISP) * (E + 1) * 4 <= limit
    c = api.make_config(T=T_ok, D=D, E=E, K=K, F=64)
    _dispatch_both(c, T_ok, K, E, D, _random_idx(T_ok, K, E, seed=5))
    T_bad = (blocks + 1) * KDISP // K
    c_bad = api.make_config(T=T_bad, D=D, E=E, K=K, F=64)
    sz = api.MoeSizes()
    assert lib().moe_get_sizes(ctypes.byref(c_bad), ctypes.byref(sz)) == MOE_OK
    dummy = [ctypes.c_void_p(256)] * 11
    rc = lib().moe_dispatch_static(ctypes.byref(c_bad), *dummy, None)
    assert rc == MOE_ERR_ARG     # refused on the host: the dummy pointers are never used
