"""Python binding of the C ABI with the same entry-point names.

Each function takes torch tensors (device memory owned by the caller),
passes their data pointers and the current CUDA stream to libmoe.so and
raises MoEError on a non-zero status.  Nothing is computed here.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import MoeConfig, MoeSizes, MoEError, check, lib
from . import _lib as C


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_config(T, D, E, K, F, *, n_shared=0, dtype="bf16", score_fn=0,
                renorm=1, n_groups=1, topk_groups=1, group_score=0,
                capacity_factor=0.0, min_capacity=0, route_scale=1.0,
                aux_alpha=0.0, z_lambda=0.0, gemm_impl=0, seq_len=0,
                expert_choice=0, loss_tokens=0, expert_base=0,
                n_local_experts=0) -> MoeConfig:
    return MoeConfig(
        T=T, D=D, E=E, K=K, F=F, n_shared=n_shared,
        dtype=C.MOE_BF16 if dtype in ("bf16", torch.bfloat16) else C.MOE_FP32,
        score_fn=score_fn, renorm=renorm, n_groups=n_groups,
        topk_groups=topk_groups, group_score=group_score,
        capacity_factor=capacity_factor, min_capacity=min_capacity,
        route_scale=route_scale, aux_alpha=aux_alpha, z_lambda=z_lambda,
        gemm_impl=gemm_impl, seq_len=seq_len, expert_choice=expert_choice,
        loss_tokens=loss_tokens, expert_base=expert_base, n_local_experts=n_local_experts)


def config_from(obj, **over) -> MoeConfig:
    """MoeConfig from any object carrying the layer fields by name."""
    names = ("n_shared", "dtype", "score_fn", "renorm", "n_groups",
             "topk_groups", "group_score", "capacity_factor", "min_capacity",
             "route_scale", "aux_alpha", "z_lambda", "seq_len", "expert_choice",
             "loss_tokens", "expert_base", "n_local_experts")
    kw = {n: getattr(obj, n) for n in names if hasattr(obj, n)}
    kw.update(over)
    return make_config(obj.T, obj.D, obj.E, obj.K, obj.F, **kw)


def moe_get_sizes(cfg: MoeConfig) -> MoeSizes:
    out = MoeSizes()
    check(lib().moe_get_sizes(ctypes.byref(cfg), ctypes.byref(out)), "moe_get_sizes")
    return out


def moe_router(cfg, x, w_r, logit_offset, sel_bias, logits, probs, lse,
               topk_idx, topk_w, near_ties, ws, stream=None):
    check(lib().moe_router(ctypes.byref(cfg), _p(x), _p(w_r), _p(logit_offset),
                           _p(sel_bias), _p(logits), _p(probs), _p(lse),
                           _p(topk_idx), _p(topk_w), _p(near_ties), _p(ws),
                           _s(stream)), "moe_router")


def moe_dispatch(cfg, topk_idx, sentinel_mask, x, counts, kept, offsets,
                 slot_row, row_slot, tile_expert, stats, x_perm, ws, stream=None):
    check(lib().moe_dispatch(ctypes.byref(cfg), _p(topk_idx), _p(sentinel_mask),
                             _p(x), _p(counts), _p(kept), _p(offsets),
                             _p(slot_row), _p(row_slot), _p(tile_expert),
                             _p(stats), _p(x_perm), _p(ws), _s(stream)),
          "moe_dispatch")


def moe_dispatch_static(cfg, topk_idx, sentinel_mask, x, counts, kept, offsets,
                        slot_row, row_slot, tile_expert, stats, x_perm, stream=None):
    """moe_dispatch without a workspace, for callers that cannot allocate
    device memory (see include/moe.h): scratch is the library's static
    device array, so overlapping calls race."""
    check(lib().moe_dispatch_static(ctypes.byref(cfg), _p(topk_idx), _p(sentinel_mask),
                                    _p(x), _p(counts), _p(kept), _p(offsets),
                                    _p(slot_row), _p(row_slot), _p(tile_expert),
                                    _p(stats), _p(x_perm), _s(stream)),
          "moe_dispatch_static")


def moe_route_expert_choice(cfg, x, w_r, logit_offset, logits, probs, lse, topk_idx, topk_w,
                            sentinel_mask, near_ties, ws, stream=None):
    check(lib().moe_route_expert_choice(
        ctypes.byref(cfg), _p(x), _p(w_r), _p(logit_offset), _p(logits), _p(probs), _p(lse),
        _p(topk_idx), _p(topk_w), _p(sentinel_mask), _p(near_ties), _p(ws), _s(stream)),
        "moe_route_expert_choice")


def moe_aux_loss_seq(cfg, probs, lse, topk_idx, slot_row, losses, ws, stream=None):
    check(lib().moe_aux_loss_seq(ctypes.byref(cfg), _p(probs), _p(lse), _p(topk_idx),
                                 _p(slot_row), _p(losses), _p(ws), _s(stream)),
          "moe_aux_loss_seq")


def moe_bias_update(cfg, counts, sel_bias, gamma, stream=None):
    check(lib().moe_bias_update(ctypes.byref(cfg), _p(counts), _p(sel_bias),
                                ctypes.c_float(gamma), _s(stream)), "moe_bias_update")


def moe_aux_loss(cfg, probs, lse, counts, losses, ws, stream=None):
    check(lib().moe_aux_loss(ctypes.byref(cfg), _p(probs), _p(lse), _p(counts),
                             _p(losses), _p(ws), _s(stream)), "moe_aux_loss")


def moe_aux_stats(cfg, probs, lse, sums, ws, stream=None):
    """This batch's load statistics (sums [E+1]) for globally scoped losses."""
    check(lib().moe_aux_stats(ctypes.byref(cfg), _p(probs), _p(lse), _p(sums), _p(ws),
                              _s(stream)), "moe_aux_stats")


def moe_aux_loss_global(cfg, counts, sums, losses, stream=None):
    """Aux and z losses from all-reduced counts and sums (cfg.loss_tokens tokens)."""
    check(lib().moe_aux_loss_global(ctypes.byref(cfg), _p(counts), _p(sums), _p(losses),
                                    _s(stream)), "moe_aux_loss_global")


def moe_set_backward_streams(streams=None):
    """Caller-owned side streams (three torch.cuda.Stream) for moe_backward on
    this thread, or None for the library's own."""
    if streams is None:
        check(lib().moe_set_backward_streams(None), "moe_set_backward_streams")
        return
    arr = (ctypes.c_void_p * 3)(*[s.cuda_stream for s in streams])
    check(lib().moe_set_backward_streams(arr), "moe_set_backward_streams")


def moe_expert_ffn(cfg, x_perm, offsets, tile_expert, stats, w13, w_down,
                   w13_s, w_down_s, a13, h, o, ws, stream=None):
    check(lib().moe_expert_ffn(ctypes.byref(cfg), _p(x_perm), _p(offsets),
                               _p(tile_expert), _p(stats), _p(w13), _p(w_down),
                               _p(w13_s), _p(w_down_s), _p(a13), _p(h), _p(o),
                               _p(ws), _s(stream)), "moe_expert_ffn")


def moe_expert_ffn_gather(cfg, x, row_slot, offsets, tile_expert, stats, w13, w_down,
                          w13_s, w_down_s, a13, h, o, ws, stream=None):
    check(lib().moe_expert_ffn_gather(ctypes.byref(cfg), _p(x), _p(row_slot), _p(offsets),
                                      _p(tile_expert), _p(stats), _p(w13), _p(w_down),
                                      _p(w13_s), _p(w_down_s), _p(a13), _p(h), _p(o),
                                      _p(ws), _s(stream)), "moe_expert_ffn_gather")


def moe_expert_ffn_combine(cfg, x, x_perm, offsets, slot_row, row_slot, topk_w, tile_expert,
                           stats, w13, w_down, w13_s, w_down_s, a13, h, o, y, ws, stream=None):
    check(lib().moe_expert_ffn_combine(
        ctypes.byref(cfg), _p(x), _p(x_perm), _p(offsets), _p(slot_row), _p(row_slot),
        _p(topk_w), _p(tile_expert), _p(stats), _p(w13), _p(w_down), _p(w13_s), _p(w_down_s),
        _p(a13), _p(h), _p(o), _p(y), _p(ws), _s(stream)), "moe_expert_ffn_combine")


def moe_combine(cfg, o, slot_row, topk_w, offsets, y, stream=None):
    check(lib().moe_combine(ctypes.byref(cfg), _p(o), _p(slot_row), _p(topk_w),
                            _p(offsets), _p(y), _s(stream)), "moe_combine")


def moe_backward(cfg, x, w_r, logits, probs, lse, topk_idx, topk_w, counts,
                 kept, offsets, slot_row, row_slot, tile_expert, stats, x_perm,
                 a13, h, o, w13, w_down, w13_s, w_down_s, dy, dx, dw_r, dw13,
                 dw_down, dw13_s, dw_down_s, dg_out, dlogits_out, ws,
                 stream=None):
    check(lib().moe_backward(
        ctypes.byref(cfg), _p(x), _p(w_r), _p(logits), _p(probs), _p(lse),
        _p(topk_idx), _p(topk_w), _p(counts), _p(kept), _p(offsets),
        _p(slot_row), _p(row_slot), _p(tile_expert), _p(stats), _p(x_perm),
        _p(a13), _p(h), _p(o), _p(w13), _p(w_down), _p(w13_s), _p(w_down_s),
        _p(dy), _p(dx), _p(dw_r), _p(dw13), _p(dw_down), _p(dw13_s),
        _p(dw_down_s), _p(dg_out), _p(dlogits_out), _p(ws), _s(stream)),
        "moe_backward")


def moe_check_status(stream=None) -> int:
    bits = ctypes.c_uint32(0)
    rc = lib().moe_check_status(_s(stream), ctypes.byref(bits))
    if rc == C.MOE_ERR_DEVICE:
        raise MoEError("device error word set: 0x%x" % bits.value)
    check(rc, "moe_check_status")
    return bits.value


def moe_launch_count(reset: bool = False) -> int:
    return int(lib().moe_launch_count(1 if reset else 0))


def moe_set_side_streams(enable: bool) -> bool:
    """Side streams inside moe_backward for this thread; returns the previous setting."""
    return bool(lib().moe_set_side_streams(1 if enable else 0))


class LaunchProfile:
    """Per-launch CUDA-event timing of this thread's library launches."""

    def __init__(self, max_launches: int = 128):
        self.max = max_launches
        check(lib().moe_profile_enable(max_launches), "moe_profile_enable")

    def reset(self):
        lib().moe_profile_reset()

    def read(self):
        """[(kernel name, ms, on_side_stream)] of the launches since reset
        (the caller has synchronised)."""
        buf = (ctypes.c_float * self.max)()
        n = lib().moe_profile_read(buf, self.max)
        if n < 0:
            check(n, "moe_profile_read")
        return [(lib().moe_profile_name(i).decode(), float(buf[i]),
                 lib().moe_profile_side(i) == 1) for i in range(n)]

    def starts(self):
        """Start of each launch since reset, in ms after the first one."""
        buf = (ctypes.c_float * self.max)()
        n = lib().moe_profile_starts(buf, self.max)
        if n < 0:
            check(n, "moe_profile_starts")
        return [float(buf[i]) for i in range(n)]

    def close(self):
        lib().moe_profile_disable()


__all__ = ["LaunchProfile", "MoEError", "MoeConfig", "MoeSizes", "make_config", "config_from",
           "moe_get_sizes", "moe_router", "moe_dispatch", "moe_dispatch_static",
           "moe_aux_loss",
           "moe_expert_ffn", "moe_combine", "moe_backward", "moe_check_status",
           "moe_launch_count", "moe_set_side_streams", "moe_aux_loss_seq",
           "moe_bias_update", "moe_route_expert_choice", "moe_expert_ffn_gather",
           "moe_expert_ffn_combine", "moe_aux_stats", "moe_aux_loss_global",
           "moe_set_backward_streams"]
