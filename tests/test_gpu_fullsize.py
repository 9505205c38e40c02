"""GPU path vs the oracle at the five configs' FULL sizes, in the launch
configuration the benchmark times (same MoELayer, same kernels).

At full size the oracle cannot redo every GEMM, so it checks:
  * routing for every token (fp32 logits formed exactly, rounded once) and
    the whole dispatch (counts, kept, drops, sentinels, every slot's expert
    and rank) bit-exact, near-ties excepted;
  * sampled tokens exactly: y_t, dg_t, dlogits_t and dx_t from the token's
    own experts (weights regenerated per expert on the host);
  * sampled weight-gradient columns: dW13[e][j,:], dW13[e][F+j,:] and
    dW_down[e][:,j] from the expert's rows;
  * dW_r = dlogits^T x (a property that holds at any size) with dlogits
    itself checked on the sampled tokens; aux and z losses.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O
from tests.helpers import LazyLayer, np64, rel_l2
from tests.test_gpu_parity import (assert_gather_identical, check_dispatch, gpu_inputs, host,
                                   run_gpu)

pytestmark = pytest.mark.gpu

N_TOKENS = {"mm_a": 8, "mm_b": 8, "olmoe": 8, "mix": 5, "ds3": 4}


def sample_tokens(cfg, Dp, rng):
    T, K = cfg.T, cfg.K
    toks = {0, T - 1, T // 2}
    dropped = np.nonzero(Dp.dropped)[0] // K
    sent = np.nonzero(Dp.sentinel)[0] // K
    if dropped.size:
        toks.add(int(dropped[len(dropped) // 2]))
    if sent.size:
        toks.add(int(sent[0]))
    while len(toks) < N_TOKENS[cfg.name]:
        toks.add(int(rng.integers(0, T)))
    return sorted(toks)


@pytest.mark.parametrize("name", ["mm_b", "mm_a", "olmoe", "mix", "ds3"])
def test_parity_full_size(name):
    cfg = W.CONFIGS[name]
    tl = 2e-2
    layer, inp = run_gpu(cfg)
    torch.cuda.synchronize()
    # --- oracle: routing + dispatch for all tokens
    x = np64(W.make_input(cfg, "x"))
    L = LazyLayer(cfg, x)
    o = O.opts_of(cfg)
    R = O.route_layer(L, o)
    Dp = O.dispatch(R.idx, cfg.E, cfg.capacity_factor, cfg.min_capacity, L.sentinel_mask)
    flips = check_dispatch(cfg, layer, R, Dp)
    assert rel_l2(host(layer.logits), R.logits) < 1e-5
    same = (layer.topk_idx.cpu().numpy() == R.idx).all(axis=1)
    assert rel_l2(host(layer.topk_w)[same], R.g[same]) < 1e-5
    # losses
    if cfg.aux_alpha:
        aux, _, _ = O.aux_loss(Dp.counts, R.p, cfg.aux_alpha, cfg.E)
        assert abs(float(layer.losses[0]) - aux) <= 1e-4 * aux
    if cfg.z_lambda:
        z = O.z_loss(R.lse, cfg.z_lambda)
        assert abs(float(layer.losses[1]) - z) <= 1e-4 * z
    # --- sampled tokens
    rng = np.random.default_rng(0)
    toks = [t for t in sample_tokens(cfg, Dp, rng) if same[t]]
    dyt = np64(W.make_input(cfg, "dy", rows=np.array(toks)))
    ref = {k: [] for k in ("y", "dg", "ds", "dx")}
    for i, t in enumerate(toks):
        r = O.token_forward_backward(L, o, R, Dp, t, dyt[i])
        for k in ref:
            ref[k].append(r[k])
    got = {
        "y": host(layer.y[toks]), "dg": host(layer.dg[toks]),
        "ds": host(layer.dlogits[toks]), "dx": host(layer.dx[toks]),
    }
    for k in ref:
        assert rel_l2(got[k], np.stack(ref[k])) < tl, (k, rel_l2(got[k], np.stack(ref[k])))
    # masked slots: zero gate gradient
    masked = (host(layer.slot_row) < 0).reshape(cfg.T, cfg.K)
    assert np.all(host(layer.dg)[masked] == 0.0)
    # --- sampled weight-gradient columns (busiest and an ordinary expert)
    dy_rows = lambda rows: np64(W.make_input(cfg, "dy", rows=np.asarray(rows)))
    experts = {int(np.argmax(Dp.kept)), int(rng.integers(0, cfg.E))}
    for e in experts:
        j = int(rng.integers(0, cfg.F))
        g_gate, g_up, g_down = O.expert_column_grads(L, o, R, Dp, e, j, dy_rows)
        assert rel_l2(host(layer.dw13[e, j]), g_gate) < tl
        assert rel_l2(host(layer.dw13[e, cfg.F + j]), g_up) < tl
        assert rel_l2(host(layer.dw_down[e, :, j]), g_down) < tl
    # --- dW_r = dlogits^T x (fp64 reduction of the GPU's own dlogits)
    dwr = host(layer.dlogits).astype(np.float64).T @ x
    assert rel_l2(host(layer.dw_r), dwr) < 1e-4
    print("%s full: near-tie flips %d, GPU near-ties %d, drops %d, sentinels %d, "
          "sampled tokens %s" % (name, flips, int(layer.near_ties[0]), int(layer.stats[0]),
                                  int(layer.stats[1]), toks))


def test_expert_choice_full_size():
    """Expert choice on the OLMoE shape at full size (64 experts, each
    picking 2048 of 16384 tokens): every expert's picks against the oracle
    (near-ties excepted), then sampled tokens and weight-gradient columns."""
    from oracle import expert_choice as X
    cfg = W.CONFIGS["olmoe_ec"]
    tl = 2e-2
    layer, inp = run_gpu(cfg)
    torch.cuda.synchronize()
    x = np64(W.make_input(cfg, "x"))
    L = LazyLayer(cfg, x)
    R, chosen, C = X.route(L, cfg.capacity_factor, cfg.min_capacity)
    assert rel_l2(host(layer.logits), R.logits) < 1e-5
    assert rel_l2(host(layer.probs), R.p) < 1e-5
    got = layer.ec_mask.cpu().numpy().reshape(cfg.T, cfg.E) == 0
    assert np.all(got.sum(axis=0) == C)
    flip = (got != chosen).any(axis=0)
    assert np.all(X.ec_margin(R.p, C)[flip] < O.NEAR_TIE), np.nonzero(flip)[0]
    if flip.any():
        return
    L.sentinel_mask = ~chosen.reshape(-1)
    o = X.opts_for(cfg.E, cfg.z_lambda)
    Dp = O.dispatch(R.idx, cfg.E, 0.0, 0, L.sentinel_mask)
    assert np.array_equal(host(layer.counts), np.full(cfg.E, C))
    z = O.z_loss(R.lse, cfg.z_lambda)
    assert abs(float(layer.losses[1]) - z) <= 1e-4 * z
    rng = np.random.default_rng(1)
    picked = chosen.sum(axis=1)
    toks = sorted({0, cfg.T - 1, int(np.argmax(picked)), int(np.argmin(picked)),
                   *[int(t) for t in rng.integers(0, cfg.T, size=4)]})
    dyt = np64(W.make_input(cfg, "dy", rows=np.array(toks)))
    ref = {k: [] for k in ("y", "dg", "ds", "dx")}
    for i, t in enumerate(toks):
        r = O.token_forward_backward(L, o, R, Dp, t, dyt[i])
        for k in ref:
            ref[k].append(r[k])
    got = {"y": host(layer.y[toks]), "dg": host(layer.dg[toks]),
           "ds": host(layer.dlogits[toks]), "dx": host(layer.dx[toks])}
    for k in ref:
        assert rel_l2(got[k], np.stack(ref[k])) < tl, (k, rel_l2(got[k], np.stack(ref[k])))
    dy_rows = lambda rows: np64(W.make_input(cfg, "dy", rows=np.asarray(rows)))
    for e in (0, int(rng.integers(1, cfg.E))):
        j = int(rng.integers(0, cfg.F))
        g_gate, g_up, g_down = O.expert_column_grads(L, o, R, Dp, e, j, dy_rows)
        assert rel_l2(host(layer.dw13[e, j]), g_gate) < tl
        assert rel_l2(host(layer.dw13[e, cfg.F + j]), g_up) < tl
        assert rel_l2(host(layer.dw_down[e, :, j]), g_down) < tl
    dwr = host(layer.dlogits).astype(np.float64).T @ x
    assert rel_l2(host(layer.dw_r), dwr) < 1e-4
    print("olmoe_ec full: picks per token %d..%d, sampled tokens %s, GPU near-ties %d" % (
        picked.min(), picked.max(), toks, int(layer.near_ties[0])))


@pytest.mark.parametrize("n_seq", [1, 4])
def test_sequence_wise_aux_full_size(n_seq):
    """The sequence-wise aux loss on the full OLMoE-shaped layer against the
    oracle's own routing: one sequence equals the batch loss; four sequences
    follow oracle/balance.py."""
    from oracle import balance as B
    cfg = W.CONFIGS["olmoe"].replace(seq_len=W.CONFIGS["olmoe"].T // n_seq)
    layer, inp = run_gpu(cfg)
    torch.cuda.synchronize()
    x = np64(W.make_input(cfg, "x"))
    L = LazyLayer(cfg, x)
    o = O.opts_of(cfg)
    R = O.route_layer(L, o)
    Dp = O.dispatch(R.idx, cfg.E, cfg.capacity_factor, cfg.min_capacity, L.sentinel_mask)
    ref, _, _ = B.seq_aux_loss(R.p, Dp.expert, cfg.K, cfg.aux_alpha, cfg.seq_len, B.SOFTMAX)
    if n_seq == 1:
        batch, _, _ = O.aux_loss(Dp.counts, R.p, cfg.aux_alpha, cfg.E)
        assert abs(ref - batch) <= 1e-12 * batch
    assert abs(float(layer.losses[0]) - ref) <= 1e-4 * ref


@pytest.mark.parametrize("name", ["mm_b", "olmoe", "olmoe_ec"])
def test_fused_gather_full_size(name):
    """The fused-gather layer (tile::gather4 rows of x inside the gate/up GEMM
    and its weight gradient) at full size is bit-identical to the permuted-
    copy layer that test_parity_full_size and test_expert_choice_full_size
    check against the oracle; padding rows load as zeros."""
    cfg = W.CONFIGS[name]
    ref, inp = run_gpu(cfg)
    fused, _ = run_gpu(cfg, inp=inp, gather=True)
    torch.cuda.synchronize()
    assert_gather_identical(cfg, ref, fused)
