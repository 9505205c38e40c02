"""One MoE layer on one GPU: buffers + the forward/backward call sequence.

The layer owns every device buffer the C ABI needs (allocated once with
torch, stable pointers, so a whole step can be captured in a CUDA graph)
and issues the entry points in order on the current stream:

  forward : moe_router -> moe_dispatch -> moe_expert_ffn_combine (expert
            FFN + combine), with moe_aux_loss on a side stream (joined
            before returning); gather=True: moe_dispatch computes the
            layout only and the gate/up GEMM reads the token rows of x
            itself (no permuted copy of x; bf16 layers)
  backward: moe_backward (its three side streams owned by the layer)

Expert shards (cfg.n_local_experts > 0, expert parallelism): the router and
the losses cover all E experts, the expert FFN only experts [expert_base,
expert_base + n_local_experts) (w13, w_down and their gradients hold those);
y, dx, dw_r, dlogits and dg of the shards sum to the whole layer's.

aux_group (a torch.distributed process group): the batch aux and z losses
are scoped over all ranks of the group (equal per-rank token counts): the
forward sums the ranks' expert counts and statistics (moe_aux_stats, then
an all-reduce, then moe_aux_loss_global) and the backward uses the summed
counts and the global token count.

No host synchronisation happens inside forward or backward.
"""
from __future__ import annotations

import torch

from . import api
from ._lib import MOE_BF16, MoeConfig


class MoELayer:
    def __init__(self, cfg, device="cuda", gather=False, aux_group=None):
        cfg = MoeConfig.from_buffer_copy(cfg)
        self.aux_group = aux_group
        if aux_group is not None:
            import torch.distributed as dist
            cfg.loss_tokens = cfg.T * dist.get_world_size(aux_group)
        self.cfg = cfg
        self.gather = bool(gather)
        self.device = torch.device(device)
        self.sizes = api.moe_get_sizes(cfg)
        c, z = cfg, self.sizes
        dev = self.device
        act = torch.bfloat16 if c.dtype == MOE_BF16 else torch.float32
        self.act_dtype = act
        T, D, E, K, F = c.T, c.D, c.E, c.K, c.F
        El = c.n_local_experts or E          # experts of this call's expert FFN
        self.n_local = El
        R = int(z.rows_max)
        f32, i32 = torch.float32, torch.int32
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
        self.logits, self.probs, self.lse = e((T, E), f32), e((T, E), f32), e((T,), f32)
        self.topk_idx, self.topk_w = e((T, K), i32), e((T, K), f32)
        self.near_ties = e((1,), i32)
        self.counts, self.kept = e((E,), i32), e((El,), i32)
        self.offsets = e((El + 2,), i32)
        self.slot_row, self.row_slot = e((T * K,), i32), e((R,), i32)
        self.tile_expert, self.stats = e((int(z.tiles_max),), i32), e((4,), i32)
        self.x_perm = None if self.gather else e((R, D), act)
        self.a13 = e((R, 2 * F), act)
        self.h, self.o = e((R, F), act), e((R, D), act)
        self.y = e((T, D), act)
        self.losses = torch.zeros(2, dtype=f32, device=dev)
        self.ws = e((max(int(z.ws_bytes), 256),), torch.uint8)
        # expert choice: 1 where expert e did not pick token t (slot t*E + e)
        self.ec_mask = e((T * K,), torch.uint8) if c.expert_choice else None
        if aux_group is not None:
            self.counts_g = e((E,), i32)          # counts summed over the group
            self.aux_sums = e((E + 1,), f32)      # sum_t p_{t,e}, sum_t lse_t^2
        self._grads_ready = False
        self._inputs = None
        self._aux_stream = None
        self._bwd_streams = None
        # aux/z losses on a side stream during the expert GEMMs (False: in
        # order on the caller's stream)
        self.side_streams = True

    def _alloc_grads(self):
        """Gradient buffers, allocated on the first backward (a forward-only
        user never holds them)."""
        if self._grads_ready:
            return
        c, dev, act, f32 = self.cfg, self.device, self.act_dtype, torch.float32
        T, D, E, K, F = c.T, c.D, c.E, c.K, c.F
        El = self.n_local
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
        self.dx = e((T, D), act)
        self.dw_r = e((E, D), f32)
        self.dw13, self.dw_down = e((El, 2 * F, D), act), e((El, D, F), act)
        self.dw13_s = e((2 * F, D), act) if c.n_shared else None
        self.dw_down_s = e((D, F), act) if c.n_shared else None
        self.dg = e((T, K), f32)
        self.dlogits = e((T, E), f32)
        self._grads_ready = True

    # -- forward -----------------------------------------------------------
    def forward(self, x, w_r, w13, w_down, w13_s=None, w_down_s=None,
                logit_offset=None, sel_bias=None, sentinel_mask=None):
        c = self.cfg
        if c.expert_choice:
            api.moe_route_expert_choice(c, x, w_r, logit_offset, self.logits, self.probs,
                                        self.lse, self.topk_idx, self.topk_w, self.ec_mask,
                                        self.near_ties, self.ws)
            sentinel_mask = self.ec_mask
        else:
            api.moe_router(c, x, w_r, logit_offset, sel_bias, self.logits, self.probs,
                           self.lse, self.topk_idx, self.topk_w, self.near_ties, self.ws)
        api.moe_dispatch(c, self.topk_idx, sentinel_mask, x, self.counts, self.kept,
                         self.offsets, self.slot_row, self.row_slot, self.tile_expert,
                         self.stats, self.x_perm, self.ws)
        main = torch.cuda.current_stream(self.device)
        aux = c.aux_alpha != 0.0 or c.z_lambda != 0.0
        if aux and self.aux_group is not None:
            self._global_aux()
            aux = False
        if aux and not self.side_streams:
            self._aux(None)
            aux = False
        if aux:
            # the losses depend only on the router and the dispatch: computed
            # on a side stream while the expert GEMMs run
            if self._aux_stream is None:
                self._aux_stream = torch.cuda.Stream(self.device)
            self._aux_stream.wait_stream(main)
            self._aux(self._aux_stream)
        # expert FFN + combine (one slot per token: the combine is done by
        # the down projection's epilogue)
        api.moe_expert_ffn_combine(c, x, self.x_perm, self.offsets, self.slot_row,
                                   self.row_slot, self.topk_w, self.tile_expert, self.stats,
                                   w13, w_down, w13_s, w_down_s, self.a13, self.h, self.o,
                                   self.y, self.ws)
        if aux:
            main.wait_stream(self._aux_stream)
        self._inputs = (x, w_r, w13, w_down, w13_s, w_down_s)
        return self.y

    def _aux(self, stream):
        c = self.cfg
        if c.seq_len > 0:
            api.moe_aux_loss_seq(c, self.probs, self.lse, self.topk_idx, self.slot_row,
                                 self.losses, self.ws, stream=stream)
        else:
            api.moe_aux_loss(c, self.probs, self.lse, self.counts, self.losses, self.ws,
                             stream=stream)

    def _global_aux(self):
        """Losses over the whole group: local statistics, all-reduce, losses."""
        from .dist import allreduce_aux_stats
        c = self.cfg
        api.moe_aux_stats(c, self.probs, self.lse, self.aux_sums, self.ws)
        self.counts_g.copy_(self.counts)
        allreduce_aux_stats(self.counts_g, self.aux_sums, self.aux_group)
        api.moe_aux_loss_global(c, self.counts_g, self.aux_sums, self.losses)

    def _loss_counts(self):
        return self.counts_g if self.aux_group is not None else self.counts

    def update_bias(self, sel_bias, gamma):
        """Selection-bias load-control step on this batch's counts (the
        group's summed counts with aux_group; in place, on the current
        stream; after forward)."""
        api.moe_bias_update(self.cfg, self._loss_counts(), sel_bias, gamma)
        return sel_bias

    # -- backward ----------------------------------------------------------
    def backward(self, dy, want_dg=True, want_dlogits=True, loss_counts=None):
        """All gradients (moe_backward).  loss_counts: the expert counts the
        aux-loss gradient uses (default: this batch's, or the group's sums
        with aux_group)."""
        self._alloc_grads()
        x, w_r, w13, w_down, w13_s, w_down_s = self._inputs
        if self._bwd_streams is None:
            self._bwd_streams = [torch.cuda.Stream(self.device) for _ in range(3)]
        api.moe_set_backward_streams(self._bwd_streams)
        try:
            api.moe_backward(
                self.cfg, x, w_r, self.logits, self.probs, self.lse, self.topk_idx,
                self.topk_w, self._loss_counts() if loss_counts is None else loss_counts,
                self.kept, self.offsets, self.slot_row,
                self.row_slot, self.tile_expert, self.stats, self.x_perm, self.a13,
                self.h, self.o, w13, w_down, w13_s, w_down_s, dy, self.dx, self.dw_r,
                self.dw13, self.dw_down, self.dw13_s, self.dw_down_s,
                self.dg if want_dg else None, self.dlogits if want_dlogits else None,
                self.ws)
        finally:
            api.moe_set_backward_streams(None)
        return self.dx

    def step(self, x, dy, **weights):
        """One forward + backward pass (the unit the benchmark times)."""
        self.forward(x, **weights)
        return self.backward(dy)
