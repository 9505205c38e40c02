"""The two data-parallel exchange steps of the layer (torch.distributed).

Data parallelism runs the whole layer on each rank's own tokens with
replicated weights.  Two quantities cross ranks:

* the load-balance statistics, when the aux and z losses are scoped over
  the global batch instead of one device's ([STA324] §8.5: the balance
  statistic may be taken over the whole batch or all devices): every rank's
  pre-drop expert counts [E] and its sums [E+1] (sum_t p_{t,e} and
  sum_t lse_t^2, from moe_aux_stats) are summed over the ranks, then
  moe_aux_loss_global gives the global losses on every rank and
  moe_backward (cfg.loss_tokens = global token count, the summed counts)
  gives each rank's share of their gradient;
* the weight gradients (dW_r, dW13, dW_down and the shared expert's), summed
  over the ranks after the backward (what the optimizer of a data-parallel
  job consumes).

Both are sums done by the collective backend (NCCL on GPUs, gloo on CPU);
this module only issues them.  Every rank must call these functions in the
same order with same-shaped tensors.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def allreduce_aux_stats(counts: torch.Tensor, sums: torch.Tensor, group=None):
    """Sum the per-rank expert counts [E] (int32) and statistics sums [E+1]
    (fp32) over `group`, in place."""
    dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(sums, op=dist.ReduceOp.SUM, group=group)
    return counts, sums


def weight_grads(layer):
    """The layer's weight-gradient tensors, in a fixed order."""
    out = [layer.dw_r, layer.dw13, layer.dw_down]
    if getattr(layer, "dw13_s", None) is not None:
        out += [layer.dw13_s, layer.dw_down_s]
    return out


def allreduce_weight_grads(grads, group=None, bucket_bytes: int = 256 << 20):
    """Sum each gradient tensor over `group`, in place.  Tensors are issued
    as asynchronous all-reduces in order; large ones are split into slices of
    about bucket_bytes so several are in flight, then all are waited on."""
    works = []
    for g in grads:
        flat = g.view(-1)
        n = max(1, bucket_bytes // flat.element_size())
        for i in range(0, flat.numel(), n):
            works.append(dist.all_reduce(flat[i:i + n], op=dist.ReduceOp.SUM, group=group,
                                         async_op=True))
    for w in works:
        w.wait()
    return grads
