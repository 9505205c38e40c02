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

N_RANDOM_TOKENS = 64
N_COLS = 8


def sample_tokens(cfg, Dp, rng):
    """At least 64 tokens: the first, middle and last token, a dropped and a
    sentinel slot's token, the token of every expert's LAST kept row (the
    tail of its final tile), and random tokens."""
    T, K = cfg.T, cfg.K
    toks = {0, T - 1, T // 2}
    dropped = np.nonzero(Dp.dropped)[0] // K
    sent = np.nonzero(Dp.sentinel)[0] // K
    if dropped.size:
        toks.update(int(v) for v in dropped[[0, len(dropped) // 2, -1]])
    if sent.size:
        toks.update(int(v) for v in sent[[0, -1]])
    for e in range(cfg.E):
        js = np.nonzero((Dp.expert == e) & (Dp.rank >= 0))[0]
        if js.size:
            toks.add(int(js[np.argmax(Dp.rank[js])]) // K)
    extra = rng.choice(T, size=min(T, N_RANDOM_TOKENS), replace=False)
    toks.update(int(t) for t in extra)
    return np.array(sorted(toks))


def sample_experts(Dp, E, rng):
    """Four experts: the busiest, the least busy with rows, the last one and
    a random one (fewer when E < 4)."""
    kept = np.asarray(Dp.kept)
    ex = [int(np.argmax(kept))]
    nz = np.nonzero(kept > 0)[0]
    if nz.size:
        ex.append(int(nz[np.argmin(kept[nz])]))
    ex.append(E - 1)
    for e in rng.permutation(E):
        if len(set(ex)) >= min(4, E):
            break
        ex.append(int(e))
    return sorted(set(ex))


def check_sampled(cfg, layer, L, o, R, Dp, rng, tl=2e-2):
    """Sampled tokens (y, dg, dlogits, dx) and sampled weight-gradient
    columns (8 columns of dW13's gate and up halves and of dW_down for 4
    experts) against the oracle on the routing R / dispatch Dp."""
    toks = sample_tokens(cfg, Dp, rng)
    dyt = np64(W.make_input(cfg, "dy", rows=toks))
    ref = O.tokens_forward_backward(L, o, R, Dp, toks, dyt)
    tt = torch.from_numpy(toks).to(layer.y.device)
    got = {"y": host(layer.y[tt]), "dg": host(layer.dg[tt]),
           "ds": host(layer.dlogits[tt]), "dx": host(layer.dx[tt])}
    for k in ref:
        err = rel_l2(got[k], ref[k])
        assert err < tl, (k, err)
    dy_rows = lambda rows: np64(W.make_input(cfg, "dy", rows=np.asarray(rows)))
    experts = sample_experts(Dp, cfg.E, rng)
    for e in experts:
        js = sorted({0, cfg.F - 1, *[int(j) for j in rng.choice(cfg.F, N_COLS - 2,
                                                              replace=False)]})
        g_gate, g_up, g_down = O.expert_column_grads(L, o, R, Dp, e, js, dy_rows)
        jt = torch.tensor(js, device=layer.dw13.device)
        assert rel_l2(host(layer.dw13[e][jt]), g_gate) < tl, ("dw13 gate", e)
        assert rel_l2(host(layer.dw13[e][jt + cfg.F]), g_up) < tl, ("dw13 up", e)
        assert rel_l2(host(layer.dw_down[e][:, jt]).T, g_down) < tl, ("dw_down", e)
    return toks, experts


@pytest.mark.parametrize("name", ["mm_b", "mm_a", "olmoe", "mix", "ds3"])
def test_parity_full_size(name):
    cfg = W.CONFIGS[name]
    layer, inp = run_gpu(cfg)
    torch.cuda.synchronize()
    # --- oracle: routing for all tokens; dispatch of the GPU's selection
    x = np64(W.make_input(cfg, "x"))
    L = LazyLayer(cfg, x)
    o = O.opts_of(cfg)
    R_own = O.route_layer(L, o)
    flips, Dp = check_dispatch(cfg, layer, R_own)
    # the oracle's routing on the GPU's selection (== its own except on the
    # near-tie tokens counted in `flips`): gate weights by the same formulas
    R = O.route_layer(L, o, idx_given=layer.topk_idx.cpu().numpy())
    assert rel_l2(host(layer.logits), R.logits) < 1e-5
    assert rel_l2(host(layer.probs), R.p) < 1e-5
    assert rel_l2(host(layer.topk_w), R.g) < 1e-5
    # losses
    if cfg.aux_alpha:
        aux, _, _ = O.aux_loss(Dp.counts, R.p, cfg.aux_alpha, cfg.E)
        assert abs(float(layer.losses[0]) - aux) <= 1e-4 * aux
    if cfg.z_lambda:
        z = O.z_loss(R.lse, cfg.z_lambda)
        assert abs(float(layer.losses[1]) - z) <= 1e-4 * z
    # masked slots: zero gate gradient, exactly
    masked = (host(layer.slot_row) < 0).reshape(cfg.T, cfg.K)
    assert np.all(host(layer.dg)[masked] == 0.0)
    rng = np.random.default_rng(0)
    toks, experts = check_sampled(cfg, layer, L, o, R, Dp, rng)
    # --- dW_r = dlogits^T x (fp64 reduction of the GPU's own dlogits)
    dwr = host(layer.dlogits).astype(np.float64).T @ x
    assert rel_l2(host(layer.dw_r), dwr) < 1e-4
    print("%s full: near-tie flips %d, GPU near-ties %d, drops %d, sentinels %d, "
          "%d sampled tokens, weight-gradient columns of experts %s" % (
              name, flips, int(layer.near_ties[0]), int(layer.stats[0]),
              int(layer.stats[1]), len(toks), experts))


def test_expert_choice_full_size():
    """Expert choice on the OLMoE shape at full size (64 experts, each
    picking 2048 of 16384 tokens): every expert's picks against the oracle
    (near-ties excepted and counted), then, on the GPU's own picks, sampled
    tokens and weight-gradient columns."""
    from oracle import expert_choice as X
    cfg = W.CONFIGS["olmoe_ec"]
    layer, inp = run_gpu(cfg)
    torch.cuda.synchronize()
    x = np64(W.make_input(cfg, "x"))
    L = LazyLayer(cfg, x)
    R, chosen_own, C = X.route(L, cfg.capacity_factor, cfg.min_capacity)
    assert rel_l2(host(layer.logits), R.logits) < 1e-5
    assert rel_l2(host(layer.probs), R.p) < 1e-5
    chosen = layer.ec_mask.cpu().numpy().reshape(cfg.T, cfg.E) == 0
    assert np.all(chosen.sum(axis=0) == C)
    flip = (chosen != chosen_own).any(axis=0)
    assert np.all(X.ec_margin(R.p, C)[flip] < O.NEAR_TIE), np.nonzero(flip)[0]
    L.sentinel_mask = ~chosen.reshape(-1)
    o = X.opts_for(cfg.E, cfg.z_lambda)
    Dp = O.dispatch(R.idx, cfg.E, 0.0, 0, L.sentinel_mask)
    assert np.array_equal(host(layer.counts), np.full(cfg.E, C))
    assert np.array_equal(host(layer.slot_row) >= 0, Dp.rank >= 0)
    z = O.z_loss(R.lse, cfg.z_lambda)
    assert abs(float(layer.losses[1]) - z) <= 1e-4 * z
    rng = np.random.default_rng(1)
    toks, experts = check_sampled(cfg, layer, L, o, R, Dp, rng)
    dwr = host(layer.dlogits).astype(np.float64).T @ x
    assert rel_l2(host(layer.dw_r), dwr) < 1e-4
    picked = chosen.sum(axis=1)
    print("olmoe_ec full: near-tie flips %d (experts), picks per token %d..%d, %d sampled "
          "tokens, weight-gradient columns of experts %s, GPU near-ties %d" % (
              int(flip.sum()), picked.min(), picked.max(), len(toks), experts,
              int(layer.near_ties[0])))


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


@pytest.mark.parametrize("name", ["mm_b", "olmoe", "olmoe_ec", "mix"])
def test_fused_gather_full_size(name):
    """The fused-gather layer (rows of x copied by the gate/up GEMM's producer
    and its weight gradient) at full size is bit-identical to the permuted-
    copy layer that test_parity_full_size and test_expert_choice_full_size
    check against the oracle; padding rows load as zeros.  On the Mixtral
    shape the permuted-copy layer runs 512-wide tiles (TMA-store epilogues)
    where the gathering one runs 256-wide tiles."""
    cfg = W.CONFIGS[name]
    ref, inp = run_gpu(cfg)
    fused, _ = run_gpu(cfg, inp=inp, gather=True)
    torch.cuda.synchronize()
    assert_gather_identical(cfg, ref, fused)
