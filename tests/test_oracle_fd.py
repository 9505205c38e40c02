"""Central finite differences of the whole oracle layer (float64).

loss = <y, dy> + L_aux + L_z.  Routing and dispatch are piecewise constant,
so every perturbation whose routing or dispatch changes is skipped; f in the
aux loss is then constant, which is exactly the reading the analytic
gradient uses.  Logits stay float64 here (Opts.logits_fp32=False) so the
difference quotients are not polluted by the fp32 rounding of the router.
"""
from __future__ import annotations

import numpy as np
import pytest

import workloads as W
from oracle import moe_oracle as O
from tests.helpers import oracle_layer

H = 1e-5


def _loss(L, o, dy):
    fw = O.forward(L, o)
    return float((fw["y"] * dy).sum() + fw["aux"] + fw["z"]), fw


def _same_routing(fa, fb):
    return (np.array_equal(fa["R"].idx, fb["R"].idx)
            and np.array_equal(fa["Dp"].rank, fb["Dp"].rank))


def _fd_check(cfg, n_per_tensor=12, seed=0):
    L = oracle_layer(cfg)
    w13 = L._w13_all.copy()
    wd = L._wd_all.copy()
    L.w13 = lambda e: w13[e]
    L.wd = lambda e: wd[e]
    o = O.opts_of(cfg)
    o.logits_fp32 = False
    dy = W.make_input(cfg, "dy").double().numpy()
    base, fw = _loss(L, o, dy)
    bw = O.backward(L, o, fw, dy)
    rng = np.random.default_rng(seed)
    targets = [("x", L.x, bw["dx"]), ("w_r", L.w_r, bw["dw_r"]),
               ("w13", w13, np.stack([bw["dw13"][e] for e in range(cfg.E)])),
               ("wd", wd, np.stack([bw["dwd"][e] for e in range(cfg.E)]))]
    if cfg.n_shared:
        targets += [("w13_s", L.w13_s, bw["dw13_s"]), ("wd_s", L.wd_s, bw["dwd_s"])]
    checked = skipped = 0
    for name, arr, grad in targets:
        flat = arr.reshape(-1)
        gflat = grad.reshape(-1)
        for i in rng.choice(flat.size, size=min(n_per_tensor, flat.size),
                            replace=False):
            old = flat[i]
            flat[i] = old + H
            lp, fp = _loss(L, o, dy)
            flat[i] = old - H
            lm, fm = _loss(L, o, dy)
            flat[i] = old
            if not (_same_routing(fw, fp) and _same_routing(fw, fm)):
                skipped += 1
                continue
            fd = (lp - lm) / (2 * H)
            an = gflat[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)) + 1e-7, (name, i, fd, an)
            checked += 1
    assert checked >= 3 * skipped and checked > 0
    return checked


def test_fd_tiny_config():
    assert _fd_check(W.CONFIGS["tiny"], n_per_tensor=20) > 50


@pytest.mark.parametrize("variant", ["A_aux_z_sentinel_capacity",
                                     "B_capacity_hotspot",
                                     "sigmoid_groups_shared",
                                     "sigmoid_A_top2sum",
                                     "A_seq_aux",
                                     "sigmoid_B_seq_aux_groups"])
def test_fd_feature_configs(variant):
    base = W.CONFIGS["tiny"].replace(T=48, D=16, E=8, K=2, F=24, dtype="fp32")
    cfg = {
        "A_aux_z_sentinel_capacity": base.replace(
            renorm=0, aux_alpha=0.05, z_lambda=0.01, sentinel_frac=0.15,
            capacity_factor=0.75),
        "B_capacity_hotspot": base.replace(
            renorm=1, capacity_factor=1.0, hot_expert_offset=0.05,
            route_scale=1.7),
        "sigmoid_groups_shared": base.replace(
            score_fn=W.SIGMOID, renorm=1, n_groups=4, topk_groups=2,
            sel_bias_range=0.1, n_shared=1, K=3, z_lambda=0.01),
        "sigmoid_A_top2sum": base.replace(
            score_fn=W.SIGMOID, renorm=0, n_groups=4, topk_groups=3,
            group_score=W.GROUP_TOP2SUM, sel_bias_range=0.1),
        # sequence-wise aux loss (3 sequences of 16 tokens), softmax and
        # sigmoid scores, with sentinels / groups
        "A_seq_aux": base.replace(
            renorm=0, aux_alpha=0.2, seq_len=16, sentinel_frac=0.1),
        "sigmoid_B_seq_aux_groups": base.replace(
            score_fn=W.SIGMOID, renorm=1, n_groups=4, topk_groups=2,
            sel_bias_range=0.1, aux_alpha=0.2, seq_len=16),
    }[variant]
    cfg = cfg.replace(w_std=0.3)   # larger logits: routing decisions matter
    assert _fd_check(cfg) > 30


def test_sentinel_zero_gate_grad_and_negative_control():
    """Sentinel slots give dg = 0 and leave the router grad of the masked
    layer intact; the batched_mm-style negative control (clamp the id to
    expert 0, keep proj_out) has the same forward but a different router
    gradient (transformers issue: loss identical, router grad wrong)."""
    cfg = W.CONFIGS["tiny"].replace(T=64, D=16, E=4, K=2, F=24, renorm=0,
                                    sentinel_frac=0.2, w_std=0.3)
    L = oracle_layer(cfg)
    o = O.opts_of(cfg)
    dy = W.make_input(cfg, "dy").double().numpy()
    fw = O.forward(L, o)
    bw = O.backward(L, o, fw, dy)
    sj = fw["Dp"].sentinel.reshape(cfg.T, cfg.K)
    assert sj.sum() == cfg.n_sentinel > 0
    assert np.all(bw["dg"][sj] == 0.0)
    # bug mode: proj_out of expert 0 for the sentinel slots
    x = L.x
    _, _, _, o0 = O.swiglu_forward(np.repeat(x, cfg.K, axis=0), L.w13(0), L.wd(0))
    bw_bug = O.backward(L, o, fw, dy, sentinel_unmasked=o0)
    assert np.any(bw_bug["dg"][sj] != 0.0)
    assert np.linalg.norm(bw_bug["dw_r"] - bw["dw_r"]) > 1e-3 * np.linalg.norm(bw["dw_r"])
    # the expert weights' grads do not depend on the router-side leak
    for e in range(cfg.E):
        np.testing.assert_array_equal(bw_bug["dw13"][e], bw["dw13"][e])


@pytest.mark.parametrize("name", ["olmoe", "mix", "ds3"])
def test_sampled_helpers_match_full_oracle(name):
    """The per-token and per-column pieces used for full-size checks give the
    same values as the finite-difference-pinned full forward/backward."""
    from tests.helpers import LazyLayer
    cfg = W.REDUCED[name].replace(T=160, D=64, F=48)
    L = oracle_layer(cfg)
    o = O.opts_of(cfg)
    dy = W.make_input(cfg, "dy").double().numpy()
    fw = O.forward(L, o)
    bw = O.backward(L, o, fw, dy)
    R, Dp = fw["R"], fw["Dp"]
    for t in (0, 7, cfg.T - 1):
        r = O.token_forward_backward(L, o, R, Dp, t, dy[t])
        np.testing.assert_allclose(r["y"], fw["y"][t], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(r["dg"], bw["dg"][t], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(r["ds"], bw["ds"][t], rtol=1e-9, atol=1e-13)
        np.testing.assert_allclose(r["dx"], bw["dx"][t], rtol=1e-9, atol=1e-12)
    LL = LazyLayer(cfg, L.x)              # row/column slices regenerated on demand
    for e, j in ((0, 3), (cfg.E - 1, cfg.F - 1)):
        a, b, c = O.expert_column_grads(LL, o, R, Dp, e, j, lambda rows: dy[rows])
        np.testing.assert_allclose(a, bw["dw13"][e][j], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(b, bw["dw13"][e][cfg.F + j], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(c, bw["dwd"][e][:, j], rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("name", ["olmoe", "mix", "ds3"])
def test_batched_sampled_helpers_match_full_oracle(name):
    """The expert-major sampled-token pass and the multi-column weight
    gradients used by the full-size checks give the rows of the
    finite-difference-pinned full forward/backward."""
    from tests.helpers import LazyLayer
    cfg = W.REDUCED[name].replace(T=160, D=64, F=48)
    L = oracle_layer(cfg)
    o = O.opts_of(cfg)
    dy = W.make_input(cfg, "dy").double().numpy()
    fw = O.forward(L, o)
    bw = O.backward(L, o, fw, dy)
    R, Dp = fw["R"], fw["Dp"]
    toks = np.array([0, 7, 33, 34, 90, cfg.T - 1])
    r = O.tokens_forward_backward(L, o, R, Dp, toks, dy[toks])
    np.testing.assert_allclose(r["y"], fw["y"][toks], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["dg"], bw["dg"][toks], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["ds"], bw["ds"][toks], rtol=1e-9, atol=1e-13)
    np.testing.assert_allclose(r["dx"], bw["dx"][toks], rtol=1e-9, atol=1e-12)
    LL = LazyLayer(cfg, L.x)
    js = [0, 5, cfg.F - 1]
    for e in (0, cfg.E - 1):
        a, b, c = O.expert_column_grads(LL, o, R, Dp, e, js, lambda rows: dy[rows])
        np.testing.assert_allclose(a, bw["dw13"][e][js], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(b, bw["dw13"][e][[cfg.F + j for j in js]], rtol=1e-9,
                                   atol=1e-12)
        np.testing.assert_allclose(c, bw["dwd"][e][:, js].T, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("name", ["mix", "ds3", "olmoe"])
def test_given_selection_keeps_the_gate_formulas(name):
    """route(idx_given=...) with the oracle's own choices changes nothing;
    with another valid choice on one token it recomputes that token's gate
    weights by the same formula (A: the scores; B: renormalised over the
    given set) and leaves every other token as it was."""
    cfg = W.REDUCED[name].replace(T=40, D=32, F=16)
    L = oracle_layer(cfg)
    o = O.opts_of(cfg)
    R = O.route_layer(L, o)
    R2 = O.route_layer(L, o, idx_given=R.idx)
    for f in ("idx", "g", "margin"):
        np.testing.assert_array_equal(getattr(R2, f), getattr(R, f))
    idx = R.idx.copy()
    t = 3
    other = [e for e in range(cfg.E) if e not in idx[t]][0]
    idx[t, -1] = other
    R3 = O.route_layer(L, o, idx_given=idx)
    keep = np.arange(cfg.T) != t
    np.testing.assert_array_equal(R3.g[keep], R.g[keep])
    sel = R.p[t, idx[t]]
    if cfg.score_fn == O.SOFTMAX and cfg.renorm:
        exp = sel / sel.sum()
    elif cfg.renorm:
        exp = sel / (sel.sum() + O.SIGMOID_EPS)
    else:
        exp = sel
    np.testing.assert_allclose(R3.g[t], exp * cfg.route_scale, rtol=1e-12)


def shard_oracle(L, o, R, lo, hi):
    """The oracle of one expert shard [lo, hi) under expert parallelism
    ([HF48687]): the global routing R, slots of experts outside the shard
    marked as sentinels (no row, no output, zero gate gradient), no aux or
    z term (those are added once, from the global counts)."""
    from dataclasses import replace
    off = (R.idx < lo) | (R.idx >= hi)
    m = off.reshape(-1) if L.sentinel_mask is None else (off.reshape(-1) | L.sentinel_mask.astype(bool))
    Ls = replace(L, sentinel_mask=m)
    os_ = replace(o, aux_alpha=0.0, z_lambda=0.0)
    return Ls, os_, O.forward_routed(Ls, os_, R)


@pytest.mark.parametrize("name", ["olmoe", "mix"])
def test_expert_shards_sum_to_the_layer(name):
    """Expert parallelism in the replicated-token form: every shard routes
    all tokens over all experts and keeps only its own experts' slots (the
    others are sentinels whose expert output is zero); y, dx, dW_r, dlogits
    and dg summed over the shards, plus the aux and z terms taken once from
    the global counts, equal the unsharded layer, and each expert's weight
    gradient comes from its own shard.  Negative control ([HF48687]): with
    the sentinel slots' outputs not zeroed (expert 0's output leaking in)
    every shard's router gradient is wrong, and for variant A so is their
    sum (under variant B the leak adds the same constant to all K slots of
    a token, which the renormalisation cancels in the sum)."""
    cfg = W.REDUCED[name].replace(T=160, D=64, F=48)
    L = oracle_layer(cfg)
    o = O.opts_of(cfg)
    dy = W.make_input(cfg, "dy").double().numpy()
    fw = O.forward(L, o)
    bw = O.backward(L, o, fw, dy)
    R, E, K = fw["R"], cfg.E, cfg.K
    x, wr = O.f64(L.x), O.f64(L.w_r)
    # the aux / z part of the router gradient, once, from the global counts
    ds_aux = O.router_backward(R, np.zeros((cfg.T, K)), o, fw["Dp"].counts)
    tot = {"y": 0.0, "dg": 0.0, "ds": ds_aux, "dx": ds_aux @ wr, "dw_r": ds_aux.T @ x}
    leak = ds_aux
    _, _, _, o0 = O.swiglu_forward(np.repeat(x, K, axis=0), L.w13(0), L.wd(0))
    cuts = [0, E // 2, E]
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        Ls, os_, fs = shard_oracle(L, o, R, lo, hi)
        bs = O.backward(Ls, os_, fs, dy)
        tot["y"] = tot["y"] + fs["y"]
        for k in ("dx", "dw_r", "ds", "dg"):
            tot[k] = tot[k] + bs[k]
        for e in range(lo, hi):
            np.testing.assert_allclose(bs["dw13"][e], bw["dw13"][e], rtol=1e-10, atol=1e-14)
            np.testing.assert_allclose(bs["dwd"][e], bw["dwd"][e], rtol=1e-10, atol=1e-14)
        bl = O.backward(Ls, os_, fs, dy, sentinel_unmasked=o0)
        assert np.linalg.norm(bl["ds"] - bs["ds"]) > 1e-3 * np.linalg.norm(bs["ds"])
        leak = leak + bl["ds"]
    for k, ref in (("y", fw["y"]), ("dx", bw["dx"]), ("dw_r", bw["dw_r"]), ("ds", bw["ds"]),
                   ("dg", bw["dg"])):
        np.testing.assert_allclose(tot[k], ref, rtol=1e-9, atol=1e-12, err_msg=k)
    if not cfg.renorm:
        assert np.linalg.norm(leak - bw["ds"]) > 1e-3 * np.linalg.norm(bw["ds"])
