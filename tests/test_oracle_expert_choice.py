"""Pins of the expert-choice oracle (oracle/expert_choice.py): the choice
against its definition by brute force, the reductions to a dense FFN and to
the all-experts soft mixture, ties, and whole-layer finite differences."""
from __future__ import annotations

import numpy as np
import pytest

import workloads as W
from oracle import expert_choice as X
from oracle import moe_oracle as O
from tests.helpers import oracle_layer


def _brute_ok(p, chosen, C):
    T, E = p.shape
    for e in range(E):
        ch = np.nonzero(chosen[:, e])[0]
        un = np.nonzero(~chosen[:, e])[0]
        assert ch.size == C
        for t in ch:
            for u in un:
                assert p[t, e] > p[u, e] or (p[t, e] == p[u, e] and t < u)


def test_choice_matches_definition_by_brute_force():
    rng = np.random.default_rng(0)
    for T, E, C in [(7, 3, 2), (12, 4, 5), (9, 2, 9), (10, 5, 1)]:
        p = O.softmax_rows(rng.normal(size=(T, E)))
        _brute_ok(p, X.choose(p, C), C)


def test_ties_go_to_the_lower_token():
    p = np.array([[0.5, 0.5], [0.5, 0.5], [0.7, 0.3], [0.5, 0.5]])
    ch = X.choose(p, 2)
    assert list(np.nonzero(ch[:, 0])[0]) == [0, 2]      # 0.7 first, then token 0
    assert list(np.nonzero(ch[:, 1])[0]) == [0, 1]      # all 0.5/0.3: tokens 0, 1


def test_capacity():
    assert X.ec_capacity(256, 4, 1.1) == 71                # ceil(1.1*256/4)
    assert X.ec_capacity(10, 4, 10.0) == 10                # at most T
    assert X.ec_capacity(64, 8, 0.5, min_capacity=6) == 6
    with pytest.raises(ValueError):
        X.ec_capacity(64, 8, 0.0)


def _cfg(E=4, T=24):
    return W.CONFIGS["tiny"].replace(T=T, D=16, E=E, K=E, F=24, renorm=0, w_std=0.3)


def test_one_expert_taking_every_token_is_a_dense_ffn():
    cfg = _cfg(E=1)
    L = oracle_layer(cfg)
    Lc, o, fw = X.forward(L, capacity_factor=1.0)
    assert fw["C"] == cfg.T and fw["chosen"].all()
    _, _, _, dense = O.swiglu_forward(L.x, L.w13(0), L.wd(0))     # g = softmax of one = 1
    np.testing.assert_allclose(fw["y"], dense, rtol=1e-12, atol=1e-12)


def test_every_expert_taking_every_token_is_the_soft_mixture():
    cfg = _cfg(E=3)
    L = oracle_layer(cfg)
    Lc, o, fw = X.forward(L, capacity_factor=3.0)
    p = fw["R"].p
    ref = np.zeros_like(fw["y"])
    for e in range(cfg.E):
        _, _, _, oe = O.swiglu_forward(L.x, L.w13(e), L.wd(e))
        ref += p[:, e:e + 1] * oe
    np.testing.assert_allclose(fw["y"], ref, rtol=1e-12, atol=1e-12)


def test_each_expert_holds_exactly_C_rows_in_token_order():
    cfg = _cfg(E=4, T=40)
    L = oracle_layer(cfg)
    Lc, o, fw = X.forward(L, capacity_factor=1.5)
    Dp, C = fw["Dp"], fw["C"]
    assert np.all(Dp.counts == C) and np.all(Dp.kept == C) and Dp.n_drop == 0
    for e in range(cfg.E):
        j = np.nonzero(Dp.expert == e)[0]            # slots t*E + e, increasing t
        np.testing.assert_array_equal(Dp.rank[j], np.arange(C))
    picked = fw["chosen"].sum(axis=1)
    assert picked.min() >= 0 and picked.max() <= cfg.E and picked.sum() == C * cfg.E


def test_finite_differences_with_choices_fixed():
    cfg = _cfg(E=4, T=32)
    L = oracle_layer(cfg)
    w13 = L._w13_all.copy()
    wd = L._wd_all.copy()
    L.w13 = lambda e: w13[e]
    L.wd = lambda e: wd[e]
    dy = W.make_input(cfg, "dy").double().numpy()
    Lc, o, fw = X.forward(L, 1.25, logits_fp32=False)
    bw = O.backward(Lc, o, fw, dy)
    h = 1e-5
    rng = np.random.default_rng(1)
    checked = 0
    for name, arr, grad in [("x", L.x, bw["dx"]), ("w_r", L.w_r, bw["dw_r"]),
                            ("w13", w13, np.stack([bw["dw13"][e] for e in range(cfg.E)])),
                            ("wd", wd, np.stack([bw["dwd"][e] for e in range(cfg.E)]))]:
        flat, gflat = arr.reshape(-1), grad.reshape(-1)
        for i in rng.choice(flat.size, size=12, replace=False):
            old = flat[i]
            vals = []
            for sgn in (1, -1):
                flat[i] = old + sgn * h
                _, _, f2 = X.forward(L, 1.25, logits_fp32=False)
                vals.append(((f2["y"] * dy).sum(), f2["chosen"]))
            flat[i] = old
            if not (np.array_equal(vals[0][1], fw["chosen"]) and
                    np.array_equal(vals[1][1], fw["chosen"])):
                continue
            fd = (vals[0][0] - vals[1][0]) / (2 * h)
            assert abs(fd - gflat[i]) <= 1e-6 * max(1.0, abs(gflat[i])) + 1e-7, (name, i)
            checked += 1
    assert checked >= 36
