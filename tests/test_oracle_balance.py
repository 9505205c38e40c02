"""Pins of the oracle's load-balance controls (oracle/balance.py): the
selection-bias update rule and the sequence-wise auxiliary loss, against
the direction the pages state, closed forms, the pages' worked aux example
evaluated per sequence, and the batch loss it must reduce to."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import balance as B
from oracle import moe_oracle as O


def test_bias_update_direction_and_closed_form():
    # [STA324] §8.6: overloaded experts' bias goes down, underloaded up
    counts = np.array([10, 2, 6, 6])          # mean 6
    b = np.array([0.1, -0.2, 0.0, 0.05])
    nb = B.bias_update(counts, b, 0.01)
    np.testing.assert_allclose(nb, [0.09, -0.19, 0.0, 0.05], rtol=0, atol=1e-15)
    assert nb[0] < b[0] and nb[1] > b[1]
    # balanced load: unchanged
    np.testing.assert_array_equal(B.bias_update([3, 3, 3], [1.0, 2.0, 3.0], 0.5), [1.0, 2.0, 3.0])


def _assign(T, K, E, rng):
    return rng.integers(0, E, size=(T, K)).reshape(-1)


def test_one_sequence_equals_batch_loss():
    rng = np.random.default_rng(3)
    T, K, E = 40, 2, 6
    s = rng.normal(size=(T, E))
    p = O.softmax_rows(s)
    ex = _assign(T, K, E, rng)
    ex[[3, 17]] = -1                                   # sentinels
    counts = np.bincount(ex[ex >= 0], minlength=E)
    lb, fb, Pb = O.aux_loss(counts, p, 0.03, E)
    ls, fs, Ps = B.seq_aux_loss(p, ex, K, 0.03, T, B.SOFTMAX)
    assert abs(ls - lb) <= 1e-15
    np.testing.assert_allclose(fs[0], fb, rtol=1e-15)
    np.testing.assert_allclose(Ps[0], Pb, rtol=1e-15)


def test_page_example_per_sequence():
    # [STA324] §8.5: E=2, f=[.75,.25], P=[.6,.4], alpha=.01 -> .011.  Two
    # sequences of 4 tokens (K=1), each built to have that f and P (the
    # second mirrored): the sequence-wise loss is the mean, .011.
    p1 = np.array([[0.6, 0.4]] * 4)
    p2 = np.array([[0.4, 0.6]] * 4)
    p = np.vstack([p1, p2])
    ex = np.array([0, 0, 0, 1, 1, 1, 1, 0])
    L, f, P = B.seq_aux_loss(p, ex, 1, 0.01, 4, B.SOFTMAX)
    np.testing.assert_allclose(f, [[0.75, 0.25], [0.25, 0.75]], rtol=1e-15)
    np.testing.assert_allclose(P, [[0.6, 0.4], [0.4, 0.6]], rtol=1e-15)
    assert abs(L - 0.011) < 1e-15


def test_uniform_routing_gives_alpha_for_both_score_functions():
    T, K, E, S = 32, 2, 4, 8
    ex = np.tile(np.arange(E), T * K // E)
    for fn in (B.SOFTMAX, B.SIGMOID):
        p = np.full((T, E), 0.25 if fn == B.SOFTMAX else 0.7)
        L, _, _ = B.seq_aux_loss(p, ex, K, 0.02, S, fn)
        assert abs(L - 0.02) < 1e-15


def test_sigmoid_normalisation_and_gradient_by_differences():
    # dL/ds through q = sigma / sum sigma, f held constant: against central
    # differences of the loss in the logits (routing fixed by construction)
    rng = np.random.default_rng(5)
    T, K, E, S = 12, 2, 5, 4
    s = rng.normal(size=(T, E))
    ex = _assign(T, K, E, rng)
    L0, f, _ = B.seq_aux_loss(O.sigmoid(s), ex, K, 0.3, S, B.SIGMOID)
    g = B.seq_aux_grad_scores(O.sigmoid(s), f, 0.3, S, B.SIGMOID)
    h = 1e-6
    for (t, e) in [(0, 0), (3, 4), (7, 2), (11, 1)]:
        sp, sm = s.copy(), s.copy()
        sp[t, e] += h
        sm[t, e] -= h
        lp = B.seq_aux_loss(O.sigmoid(sp), ex, K, 0.3, S, B.SIGMOID)[0]
        lm = B.seq_aux_loss(O.sigmoid(sm), ex, K, 0.3, S, B.SIGMOID)[0]
        assert abs((lp - lm) / (2 * h) - g[t, e]) < 1e-8


def test_seq_len_must_divide_T():
    with pytest.raises(ValueError):
        B.seq_aux_loss(np.ones((10, 2)) / 2, np.zeros(10, dtype=int), 1, 0.01, 4)
