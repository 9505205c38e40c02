"""Expert-choice routing — TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

[STA324] §8.4 (token choice, expert choice and global routing): in expert
choice every expert picks a fixed number of tokens from the batch, so the
expert side's load is fixed, and a token may be picked by several experts
or by none.  Readings (the page gives only this description):

* scores: p = softmax(s) over the experts of each token, the same router
  scores as token choice ([STA324] §8.2);
* capacity: each expert takes C = max(ceil(c * T / E), min_capacity) tokens
  ([STA324] §8.5's capacity formula with one choice per token: c is the
  average number of experts per token), C <= T;
* choice: expert e takes the C tokens with the largest p_{t,e}; equal
  scores go to the lower token index (the same tie rule as top-K);
* gate weight g_{t,e} = p_{t,e} (variant A: no renormalisation, since a
  token's number of experts varies), combine y_t = sum_{e picks t} g_{t,e}
  E_e(x_t) in increasing e;
* backward: with the choices fixed, dL/dp_{t,e} = <E_e(x_t), dy_t> for the
  chosen pairs and 0 elsewhere, then the softmax backward ([STA324] §8.3).

Expressed in the token-choice layer's own terms, so the rest of the oracle
is reused unchanged: every (t, e) pair is a slot (K = E, idx[t, k] = k),
g = p, variant A, and the pairs an expert did not choose are sentinel slots
(no row, no output, no gradient).  The dispatch then ranks each expert's
chosen tokens in increasing t and every expert holds exactly C rows.
"""
from __future__ import annotations

import math

import numpy as np

from . import moe_oracle as O


def ec_capacity(T, E, capacity_factor, min_capacity=0):
    if not capacity_factor > 0:
        raise ValueError("expert choice needs a capacity factor > 0")
    C = max(int(math.ceil(capacity_factor * T / E)), int(min_capacity))
    return min(C, T)


def choose(p, C):
    """chosen [T, E] bool: column e's C largest scores, lower t first on ties."""
    p = np.asarray(p)
    T, E = p.shape
    chosen = np.zeros((T, E), dtype=bool)
    for e in range(E):
        # stable sort on -p keeps the lower index first among equal scores
        order = np.argsort(-p[:, e], kind="stable")
        chosen[order[:C], e] = True
    return chosen


def route(L: O.Layer, capacity_factor, min_capacity=0, logits_fp32=True):
    """(Routing in slot form, chosen mask, C) for expert choice."""
    s = O.router_logits(L.x, L.w_r, L.logit_offset, logits_fp32)
    T, E = s.shape
    p = O.softmax_rows(s)
    lse = O.logsumexp_rows(s)
    C = ec_capacity(T, E, capacity_factor, min_capacity)
    chosen = choose(p, C)
    idx = np.tile(np.arange(E), (T, 1))
    R = O.Routing(logits=s, p=p, lse=lse, idx=idx, g=p.copy(),
                  margin=np.full(T, np.inf))
    return R, chosen, C


def layer_for(L: O.Layer, chosen) -> O.Layer:
    """The layer with the unchosen pairs as sentinel slots."""
    from dataclasses import replace
    return replace(L, sentinel_mask=~chosen.reshape(-1))


def opts_for(E, z_lambda=0.0) -> O.Opts:
    return O.Opts(K=E, score_fn=O.SOFTMAX, renorm=0, z_lambda=z_lambda)


def forward(L: O.Layer, capacity_factor, min_capacity=0, logits_fp32=True, z_lambda=0.0):
    """(layer with the unchosen pairs as sentinels, Opts, forward dict);
    O.backward(layer, opts, fw, dy) then gives every gradient."""
    R, chosen, C = route(L, capacity_factor, min_capacity, logits_fp32)
    E = chosen.shape[1]
    Lc = layer_for(L, chosen)
    o = opts_for(E, z_lambda)
    o.logits_fp32 = logits_fp32
    fw = O.forward_routed(Lc, o, R)
    fw["chosen"], fw["C"] = chosen, C
    return Lc, o, fw


def ec_margin(p, C):
    """Per expert, the gap between its C-th and (C+1)-th scores (inf if
    C == T): the choice is a near-tie where it is below NEAR_TIE."""
    p = np.asarray(p)
    T, E = p.shape
    m = np.full(E, np.inf)
    if C >= T:
        return m
    for e in range(E):
        v = np.sort(p[:, e])[::-1]
        m[e] = v[C - 1] - v[C]
    return m
