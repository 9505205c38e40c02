"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: a worked
example printed on a page (fixtures under tests/golden/, each with its
citation), a closed form, brute force on tiny inputs, a special case that
reduces to a library routine, or torch autograd as an independent
differentiator.  Finite differences of the whole layer live in
test_oracle_fd.py.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# Gate-weight variants: STA324 §8.2 worked example
# ---------------------------------------------------------------------------
def test_variant_a_b_worked_example():
    g = gold("ab_worked_example.json")
    probs = np.array([g["probs"]])
    logits = np.log(probs).astype(np.float32)   # softmax(logits) == probs
    for renorm, key in ((0, "variant_A"), (1, "variant_B")):
        R = O.route(logits, g["K"], renorm=renorm)
        dense = np.zeros(4)
        dense[R.idx[0]] = R.g[0]
        np.testing.assert_allclose(dense, g[key], atol=1e-7, rtol=0)
    assert list(R.idx[0]) == [0, 1]


def test_variant_b_equals_truncate_then_renormalise():
    # STA324 §8.2: B is the same as full softmax, truncate, renormalise.
    rng = np.random.default_rng(1)
    s = rng.normal(size=(50, 9)).astype(np.float32)
    for K in (1, 2, 3, 9):
        RA = O.route(s, K, renorm=0)
        RB = O.route(s, K, renorm=1)
        np.testing.assert_allclose(RB.g, RA.g / RA.g.sum(1, keepdims=True),
                                   rtol=1e-13)
        assert np.all(RA.g.sum(1) <= 1 + 1e-12)
    # K = E with B: weights are the full softmax
    RB = O.route(s, 9, renorm=1)
    dense = np.zeros_like(RB.p)
    np.put_along_axis(dense, RB.idx, RB.g, axis=1)
    np.testing.assert_allclose(dense, RB.p, rtol=1e-13)
    # the softmax matches torch's
    np.testing.assert_allclose(
        RB.p, torch.softmax(torch.tensor(s, dtype=torch.float64), 1).numpy(),
        rtol=1e-13)


# ---------------------------------------------------------------------------
# Top-K selection, ties, groups, sigmoid + bias: brute force
# ---------------------------------------------------------------------------
def _brute_topk(u, K):
    order = sorted(range(len(u)), key=lambda e: (-u[e], e))
    return order[:K]


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(2)
    for _ in range(200):
        E = int(rng.integers(2, 9))
        K = int(rng.integers(1, E + 1))
        s = rng.integers(-3, 4, size=(1, E)).astype(np.float32)  # many ties
        R = O.route(s, K)
        assert list(R.idx[0]) == _brute_topk(list(s[0].astype(float)), K)


def _brute_group_topk(u, K, n_groups, topk_groups, group_score):
    E = len(u)
    gs = E // n_groups
    scores = []
    for j in range(n_groups):
        grp = sorted(u[j * gs:(j + 1) * gs], reverse=True)
        scores.append(grp[0] if group_score == O.GROUP_MAX else grp[0] + grp[1])
    keep = sorted(range(n_groups), key=lambda j: (-scores[j], j))[:topk_groups]
    cand = [e for e in range(E) if e // gs in keep]
    return sorted(cand, key=lambda e: (-u[e], e))[:K]


@pytest.mark.parametrize("group_score", [O.GROUP_MAX, O.GROUP_TOP2SUM])
def test_group_limited_brute_force(group_score):
    rng = np.random.default_rng(3)
    for _ in range(200):
        n_groups, gsz = 4, 4
        E = n_groups * gsz
        topk_groups = int(rng.integers(1, n_groups + 1))
        K = int(rng.integers(1, topk_groups * gsz + 1))
        s = rng.normal(size=(1, E)).astype(np.float32)
        R = O.route(s, K, n_groups=n_groups, topk_groups=topk_groups,
                    group_score=group_score)
        assert list(R.idx[0]) == _brute_group_topk(
            list(s[0].astype(float)), K, n_groups, topk_groups, group_score)


def test_sigmoid_bias_selects_but_does_not_weight():
    # STA324 §8.6: the bias moves the choice, the weights use the raw affinity.
    rng = np.random.default_rng(4)
    s = rng.normal(size=(20, 8)).astype(np.float32)
    b = np.zeros(8)
    b[5] = 10.0                      # forces expert 5 into every token's set
    R = O.route(s, 2, score_fn=O.SIGMOID, renorm=1, sel_bias=b)
    assert np.all((R.idx == 5).any(axis=1))
    sig = 1 / (1 + np.exp(-s.astype(np.float64)))
    sel = np.take_along_axis(sig, R.idx, axis=1)
    np.testing.assert_allclose(R.g, sel / sel.sum(1, keepdims=True), rtol=1e-12)
    # a constant shift of every bias changes nothing
    R2 = O.route(s, 2, score_fn=O.SIGMOID, renorm=1, sel_bias=b + 3.0)
    assert np.array_equal(R.idx, R2.idx)
    np.testing.assert_array_equal(R.g, R2.g)


def test_near_tie_margin():
    s = np.array([[1.0, 0.5, 0.5 - 5e-6, -1.0]], dtype=np.float32)
    R = O.route(s, 2)
    assert R.margin[0] < O.NEAR_TIE
    R = O.route(np.array([[1.0, 0.5, 0.2, -1.0]], dtype=np.float32), 2)
    assert R.margin[0] > 0.29


# ---------------------------------------------------------------------------
# Capacity and dispatch
# ---------------------------------------------------------------------------
def test_capacity_lab_arithmetic():
    g = gold("capacity_lab.json")
    T, E, K = g["T"], g["E"], g["K"]
    c = g["capacity_factor_reading"]
    assert O.capacity(T, K, E, c) == g["capacity"]
    # build slot assignments with the printed hot-spot loads
    loads = g["hotspot_loads"]
    idx = np.zeros((T, K), dtype=np.int64)
    idx[:, 0] = 0
    second = np.repeat([1, 2, 3], loads[1:])
    assert second.size == T and loads[0] == T
    idx[:, 1] = second
    Dp = O.dispatch(idx, E, c)
    assert list(Dp.counts) == loads
    assert Dp.n_drop == g["dropped_assignments"]
    assert list(Dp.kept) == [min(n, g["capacity"]) for n in loads]
    # the balanced loads overflow nothing
    nl = g["no_hotspot_loads"]
    assert sum(max(0, n - g["capacity"]) for n in nl) == g["no_hotspot_dropped"]
    # a dropped assignment loses one branch only: every token keeps slot k=1
    assert np.all(Dp.rank.reshape(T, K)[:, 1] >= 0)


def test_dispatch_brute_force_and_invariants():
    rng = np.random.default_rng(5)
    for _ in range(60):
        T = int(rng.integers(1, 40))
        E = int(rng.integers(1, 7))
        K = int(rng.integers(1, E + 1))
        idx = rng.integers(-1, E, size=(T, K))
        mask = rng.random(T * K) < 0.1
        c = float(rng.choice([0.0, 0.5, 1.0, 1.25]))
        Dp = O.dispatch(idx, E, c, sentinel_mask=mask)
        ex = idx.reshape(-1).copy()
        ex[mask] = -1
        C = O.capacity(T, K, E, c)
        for j in range(T * K):
            if ex[j] < 0:
                assert Dp.rank[j] == -1 and Dp.sentinel[j]
                continue
            r = int(np.sum(ex[:j] == ex[j]))        # stable by flat slot index
            if C is None or r < C:
                assert Dp.rank[j] == r
            else:
                assert Dp.rank[j] == -1 and Dp.dropped[j]
        assert Dp.kept.sum() + Dp.n_drop + Dp.n_sentinel == T * K
        assert list(Dp.counts) == [int(np.sum(ex == e)) for e in range(E)]
        rows = Dp.row()
        kept_rows = np.sort(rows[rows >= 0])
        assert np.array_equal(kept_rows, np.arange(Dp.kept.sum()))   # bijection
        if C is None:
            assert Dp.n_drop == 0


# ---------------------------------------------------------------------------
# Losses
# ---------------------------------------------------------------------------
def test_aux_loss_worked_example_and_limits():
    g = gold("aux_loss_example.json")
    E = g["E"]
    # counts giving f = [.75,.25]; probabilities with column means [.6,.4]
    counts = np.array([3, 1])
    p = np.array([[0.7, 0.3], [0.5, 0.5]])
    L, f, P = O.aux_loss(counts, p, g["alpha"], E)
    np.testing.assert_allclose(f, g["f"])
    np.testing.assert_allclose(P, g["P"])
    assert abs(L - g["loss"]) < 1e-15
    for E in (2, 4, 8, 64):
        Lu, _, _ = O.aux_loss(np.full(E, 10), np.full((3, E), 1.0 / E), 0.01, E)
        assert abs(Lu - 0.01) < 1e-15                         # uniform -> alpha
        counts = np.zeros(E)
        counts[0] = 100
        p = np.zeros((5, E))
        p[:, 0] = 1.0
        Lc, _, _ = O.aux_loss(counts, p, 0.01, E)
        assert abs(Lc - 0.01 * E) < 1e-15                     # collapse -> alpha*E


def test_z_loss_closed_form():
    # logits all equal to c: lse = c + log(E)
    E, c = 8, 0.75
    s = np.full((4, E), c, dtype=np.float32)
    R = O.route(s, 2)
    assert abs(O.z_loss(R.lse, 1e-3) - 1e-3 * (c + math.log(E)) ** 2) < 1e-15
    rng = np.random.default_rng(6)
    s = rng.normal(size=(7, 5))
    R = O.route(s, 2)
    np.testing.assert_allclose(
        R.lse, torch.logsumexp(torch.tensor(s), 1).numpy(), rtol=1e-14)


# ---------------------------------------------------------------------------
# Router gradient: K=1 special case and the page's reproduction
# ---------------------------------------------------------------------------
def test_k1_variant_b_router_grad_exactly_zero():
    # STA324 §8.3 and the MiniMind issue §2: with K=1 the renormalised weight
    # is the constant 1, so the gate path gives the router no gradient;
    # variant A keeps p_selected and does.
    rng = np.random.default_rng(7)
    s = rng.normal(size=(64, 4)).astype(np.float32)
    dg = rng.normal(size=(64, 1))
    RB = O.route(s, 1, renorm=1)
    assert np.all(RB.g == 1.0)
    dsB = O.router_backward(RB, dg, O.Opts(K=1, renorm=1))
    assert np.all(dsB == 0.0)
    RA = O.route(s, 1, renorm=0)
    dsA = O.router_backward(RA, dg, O.Opts(K=1, renorm=0))
    assert np.linalg.norm(dsA) > 1e-2
    # with the aux loss on, B's router gradient is the aux gradient alone
    counts = np.array([10, 20, 30, 4])
    o = O.Opts(K=1, renorm=1, aux_alpha=5e-4)
    ds_full = O.router_backward(RB, dg, o, counts)
    ds_aux = O.router_backward(RB, np.zeros_like(dg), o, counts)
    assert np.array_equal(ds_full, ds_aux)
    assert np.linalg.norm(ds_aux) > 0


def _repro_tensors():
    g = gold("minimind_repro.json")
    torch.manual_seed(g["seed"])
    x = torch.randn(g["B"], g["H"])
    gate_w = torch.randn(g["E"], g["H"])
    ts = [torch.randn(g["B"], c["k"]) for c in g["cases"]]
    return g, x, gate_w, ts


def test_minimind_repro_printed_values():
    g, x, gate_w, ts = _repro_tensors()
    xs = x.double().numpy()
    logits = (x.double() @ gate_w.double().T).numpy().astype(np.float32)
    for case, t in zip(g["cases"], ts):
        k, norm = case["k"], int(case["renorm"])
        R = O.route(logits, k, renorm=norm)
        ds = O.router_backward(R, t.double().numpy(), O.Opts(K=k, renorm=norm))
        gnorm = float(np.linalg.norm(ds.T @ xs))
        if case["pinned"] is False:
            continue
        if k == 1 and norm:
            assert gnorm == 0.0 and gnorm <= case["grad_norm"]
        else:
            assert abs(gnorm - case["grad_norm"]) / case["grad_norm"] < 5e-4


def test_router_backward_matches_autograd():
    # torch autograd differentiates the forward definition independently
    g, x, gate_w, ts = _repro_tensors()
    xd = x.double()
    for case, t in zip(g["cases"], ts):
        for k, norm in ((case["k"], 0), (case["k"], 1), (3, 1), (3, 0)):
            tt = t if t.shape[1] == k else torch.randn(x.shape[0], k,
                                                       generator=torch.Generator().manual_seed(k))
            w = gate_w.double().clone().requires_grad_(True)
            s = xd @ w.T
            p = torch.softmax(s, 1)
            val, idx = torch.topk(p, k, dim=1)
            if norm:
                val = val / val.sum(1, keepdim=True)
            (val * tt.double()).sum().backward()
            R = O.route(s.detach().numpy(), k, renorm=norm)
            assert np.array_equal(R.idx, idx.numpy())
            ds = O.router_backward(R, tt.double().numpy(), O.Opts(K=k, renorm=norm))
            ref = w.grad.numpy()
            got = ds.T @ xd.numpy()
            if k == 1 and norm:
                assert np.all(got == 0) and np.abs(ref).max() < 1e-9
            else:
                np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_sigmoid_router_backward_matches_autograd():
    rng = np.random.default_rng(8)
    T, E, K, D = 16, 16, 4, 12
    x = torch.tensor(rng.normal(size=(T, D)))
    w = torch.tensor(rng.normal(size=(E, D)) * 0.3, requires_grad=True)
    b = rng.uniform(-0.1, 0.1, size=E)
    dg = rng.normal(size=(T, K))
    for renorm in (0, 1):
        for n_groups, topk_groups in ((1, 1), (4, 2)):
            w.grad = None
            s = x @ w.T
            sig = torch.sigmoid(s)
            R = O.route(s.detach().numpy(), K, score_fn=O.SIGMOID,
                        renorm=renorm, n_groups=n_groups,
                        topk_groups=topk_groups, sel_bias=b, route_scale=2.5)
            sel = torch.gather(sig, 1, torch.tensor(R.idx))
            gw = sel / (sel.sum(1, keepdim=True) + 1e-20) if renorm else sel
            (2.5 * gw * torch.tensor(dg)).sum().backward()
            np.testing.assert_allclose(R.g, 2.5 * gw.detach().numpy(), rtol=1e-13)
            ds = O.router_backward(R, dg, O.Opts(K=K, score_fn=O.SIGMOID,
                                                 renorm=renorm, route_scale=2.5))
            np.testing.assert_allclose(ds.T @ x.numpy(), w.grad.numpy(),
                                       rtol=1e-10, atol=1e-13)


def test_aux_and_z_gradients_match_autograd():
    rng = np.random.default_rng(9)
    T, E, K = 12, 6, 2
    s = torch.tensor(rng.normal(size=(T, E)), requires_grad=True)
    R = O.route(s.detach().numpy(), K, renorm=0)
    counts = np.bincount(R.idx.reshape(-1), minlength=E)
    alpha, lam = 0.01, 1e-3
    f = torch.tensor(counts / counts.sum())
    p = torch.softmax(s, 1)
    loss = alpha * E * (f * p.mean(0)).sum() + lam * (torch.logsumexp(s, 1) ** 2).mean()
    loss.backward()
    o = O.Opts(K=K, renorm=0, aux_alpha=alpha, z_lambda=lam)
    ds = O.router_backward(R, np.zeros((T, K)), o, counts)
    np.testing.assert_allclose(ds, s.grad.numpy(), rtol=1e-12, atol=1e-16)
    laux, _, _ = O.aux_loss(counts, R.p, alpha, E)
    assert abs(laux + O.z_loss(R.lse, lam) - float(loss)) < 1e-14


# ---------------------------------------------------------------------------
# Expert FFN and combine: reduce to a dense SwiGLU FFN (torch.nn.functional)
# ---------------------------------------------------------------------------
def _dense_swiglu(x, w13, wd):
    F = wd.shape[1]
    xt = torch.tensor(x)
    a = Fn.linear(xt, torch.tensor(w13[:F]))
    b = Fn.linear(xt, torch.tensor(w13[F:]))
    return Fn.linear(Fn.silu(a) * b, torch.tensor(wd)).numpy()


def test_single_expert_is_dense_ffn():
    rng = np.random.default_rng(10)
    T, D, F = 9, 6, 10
    x = rng.normal(size=(T, D))
    w13 = rng.normal(size=(1, 2 * F, D)) * 0.3
    wd = rng.normal(size=(1, D, F)) * 0.3
    for renorm in (0, 1):
        L = O.Layer(x=x, w_r=rng.normal(size=(1, D)), w13=lambda e: w13[e],
                    wd=lambda e: wd[e])
        fw = O.forward(L, O.Opts(K=1, renorm=renorm))
        g = fw["R"].g
        np.testing.assert_allclose(fw["y"], g * _dense_swiglu(x, w13[0], wd[0]),
                                   rtol=1e-12, atol=1e-14)


def test_identical_experts_variant_b_is_dense_ffn():
    rng = np.random.default_rng(11)
    T, D, F, E = 11, 8, 12, 5
    x = rng.normal(size=(T, D))
    w13 = rng.normal(size=(2 * F, D)) * 0.3
    wd = rng.normal(size=(D, F)) * 0.3
    w13s = rng.normal(size=(2 * F, D)) * 0.3
    wds = rng.normal(size=(D, F)) * 0.3
    L = O.Layer(x=x, w_r=rng.normal(size=(E, D)), w13=lambda e: w13,
                wd=lambda e: wd, w13_s=w13s, wd_s=wds)
    fw = O.forward(L, O.Opts(K=3, renorm=1))
    np.testing.assert_allclose(
        fw["y"], _dense_swiglu(x, w13, wd) + _dense_swiglu(x, w13s, wds),
        rtol=1e-11, atol=1e-13)


def test_swiglu_backward_matches_autograd():
    rng = np.random.default_rng(12)
    n, D, F = 7, 5, 6
    x = torch.tensor(rng.normal(size=(n, D)), requires_grad=True)
    w13 = torch.tensor(rng.normal(size=(2 * F, D)), requires_grad=True)
    wd = torch.tensor(rng.normal(size=(D, F)), requires_grad=True)
    do = rng.normal(size=(n, D))
    a = x @ w13[:F].T
    b = x @ w13[F:].T
    o = (Fn.silu(a) * b) @ wd.T
    (o * torch.tensor(do)).sum().backward()
    A, B, H, Oo = O.swiglu_forward(x.detach().numpy(), w13.detach().numpy(),
                                   wd.detach().numpy())
    np.testing.assert_allclose(Oo, o.detach().numpy(), rtol=1e-12)
    dx, dw13, dwd = O.swiglu_backward(x.detach().numpy(), A, B, H, do,
                                      w13.detach().numpy(), wd.detach().numpy())
    np.testing.assert_allclose(dx, x.grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dw13, w13.grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dwd, wd.grad.numpy(), rtol=1e-11, atol=1e-13)


def test_aux_loss_from_pooled_stats():
    """The pooled-statistics form gives the page's worked example (E=2,
    f=[.75,.25], P=[.6,.4], alpha=.01 -> .011, [STA324] §8.5) and equals the
    batch loss on the concatenated batch when split into two parts."""
    assert abs(O.aux_loss_from_stats([3, 1], [1.2, 0.8], 2, 0.01, 2) - 0.011) < 1e-15
    rng = np.random.default_rng(3)
    T, E, K = 50, 6, 2
    s = rng.normal(size=(T, E))
    R = O.route(s, K, renorm=0)
    Dp = O.dispatch(R.idx, E)
    full, _, _ = O.aux_loss(Dp.counts, R.p, 0.01, E)
    a, b = slice(0, 21), slice(21, T)
    ca = O.dispatch(R.idx[a], E).counts
    cb = O.dispatch(R.idx[b], E).counts
    pooled = O.aux_loss_from_stats(ca + cb, R.p[a].sum(0) + R.p[b].sum(0), T, 0.01, E)
    assert abs(pooled - full) < 1e-15
