"""Shared test utilities: build oracle layers from the seeded workloads."""
from __future__ import annotations

import numpy as np
import torch

import workloads as W
from oracle import moe_oracle as O


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_layer(cfg: W.LayerConfig) -> O.Layer:
    """All inputs of `cfg` materialised on the host (small configs)."""
    w13 = np64(W.make_input(cfg, "w13"))
    wd = np64(W.make_input(cfg, "w_down"))
    L = O.Layer(
        x=np64(W.make_input(cfg, "x")),
        w_r=np64(W.make_input(cfg, "w_r")),
        w13=lambda e, _w=w13: _w[e],
        wd=lambda e, _w=wd: _w[e],
    )
    L._w13_all, L._wd_all = w13, wd
    if cfg.n_shared:
        L.w13_s = np64(W.make_input(cfg, "w13_s"))
        L.wd_s = np64(W.make_input(cfg, "w_down_s"))
    if cfg.hot_expert_offset:
        L.logit_offset = np64(W.make_input(cfg, "logit_offset"))
    if cfg.sel_bias_range:
        L.sel_bias = np64(W.make_input(cfg, "sel_bias").float())
    if cfg.sentinel_frac:
        L.sentinel_mask = W.make_input(cfg, "sentinel_mask").numpy()
    return L


class LazyLayer(O.Layer):
    """Full-size layer whose expert weights are regenerated on demand."""

    def __init__(self, cfg: W.LayerConfig, x: np.ndarray, cache_experts=8):
        super().__init__(
            x=x, w_r=np64(W.make_input(cfg, "w_r")),
            w13=self._w13, wd=self._wd)
        self.cfg = cfg
        self.F = cfg.F
        self._cache = {}
        self._cache_n = cache_experts
        if cfg.n_shared:
            self.w13_s = np64(W.make_input(cfg, "w13_s"))
            self.wd_s = np64(W.make_input(cfg, "w_down_s"))
        if cfg.hot_expert_offset:
            self.logit_offset = np64(W.make_input(cfg, "logit_offset"))
        if cfg.sel_bias_range:
            self.sel_bias = np64(W.make_input(cfg, "sel_bias").float())
        if cfg.sentinel_frac:
            self.sentinel_mask = W.make_input(cfg, "sentinel_mask").numpy()

    def _get(self, name, e):
        key = (name, e)
        if key not in self._cache:
            if len(self._cache) >= self._cache_n:
                self._cache.pop(next(iter(self._cache)))
            self._cache[key] = np64(W.make_input(self.cfg, name, expert=e))
        return self._cache[key]

    def _w13(self, e):
        return self._get("w13", e)

    def _wd(self, e):
        return self._get("w_down", e)

    def w13_rows(self, e, rows):
        c = self.cfg
        flat = ((e * 2 * c.F + np.asarray(rows))[:, None] * c.D
                + np.arange(c.D)[None, :])
        v = W.gen.normal_at((c.E, 2 * c.F, c.D), flat.reshape(-1), c.seed,
                            W.STREAM["w13"], c.w_std, dtype=W._dt(c))
        return np64(v).reshape(len(rows), c.D)

    def wd_col(self, e, j):
        c = self.cfg
        flat = e * c.D * c.F + np.arange(c.D) * c.F + j
        v = W.gen.normal_at((c.E, c.D, c.F), flat, c.seed, W.STREAM["w_down"],
                            c.w_std, dtype=W._dt(c))
        return np64(v)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))
