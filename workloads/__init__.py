"""Seeded synthetic workloads for the token-choice MoE layer.

This module is shared by the oracle (tests) and by the CUDA path (tests,
bench).  It holds shapes, options and seeded random inputs only — none of the
layer's arithmetic.  Every tensor is produced by the counter-hash generator in
:mod:`workloads.gen`, so the same element has the same value on the CPU and on
the GPU, and any slice (one expert's weights, a few tokens) can be regenerated
on its own without materialising the rest.

Shapes follow the five layer configurations the method is exercised on
(a tiny fp32 layer and layers shaped like MiniMind, OLMoE, Mixtral and
DeepSeek-V3); the reduced variants keep each configuration's options and
structure at sizes the plain CPU oracle finishes in seconds while still
spanning several 128-row tiles with ragged tails.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional

from . import gen  # noqa: F401  (re-exported)

# score functions / variants (mirrors the C enum values in include/moe.h)
SOFTMAX = 0
SIGMOID = 1
GROUP_MAX = 0
GROUP_TOP2SUM = 1


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int                      # tokens
    D: int                      # model dim
    E: int                      # routed experts
    K: int                      # experts per token
    F: int                      # expert FFN (SwiGLU) inner dim
    n_shared: int = 0           # shared experts (0 or 1)
    dtype: str = "bf16"         # "bf16" or "fp32" (activations + expert weights)
    score_fn: int = SOFTMAX
    renorm: int = 1             # 0 = variant A (truncate), 1 = variant B (renormalise)
    n_groups: int = 1
    topk_groups: int = 1
    group_score: int = GROUP_MAX
    capacity_factor: float = 0.0   # <= 0: unlimited
    min_capacity: int = 0
    route_scale: float = 1.0
    aux_alpha: float = 0.0
    z_lambda: float = 0.0
    seq_len: int = 0            # > 0: sequence-wise aux loss over seq_len tokens
    expert_choice: int = 0      # 1: each expert picks its C tokens (K = E slots per token)
    # input recipe
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    dy_std: float = 1.0
    hot_expert_offset: float = 0.0   # added to expert 0's logit (hot-spot router)
    sel_bias_range: float = 0.0      # b_e ~ U(-r, r) selection bias (sigmoid routing)
    sentinel_frac: float = 0.0       # fraction of slots overwritten with expert id -1

    def replace(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)

    @property
    def n_slots(self) -> int:
        return self.T * self.K

    @property
    def n_sentinel(self) -> int:
        return int(round(self.sentinel_frac * self.T * self.K))


# ---------------------------------------------------------------------------
# The five layer configurations (full size).
# ---------------------------------------------------------------------------
CONFIGS = {
    # tiny fp32 layer, variant B, no capacity limit
    "tiny": LayerConfig("tiny", T=64, D=32, E=4, K=2, F=64, dtype="fp32",
                        renorm=1),
    # MiniMind-shaped: K=1, both gate variants, Switch aux loss alpha=5e-4
    "mm_a": LayerConfig("mm_a", T=4096, D=768, E=4, K=1, F=2048, renorm=0,
                        aux_alpha=5e-4),
    "mm_b": LayerConfig("mm_b", T=4096, D=768, E=4, K=1, F=2048, renorm=1,
                        aux_alpha=5e-4),
    # OLMoE-shaped: variant A, aux + z-loss, 10% sentinel slots
    "olmoe": LayerConfig("olmoe", T=16384, D=2048, E=64, K=8, F=1024,
                         renorm=0, aux_alpha=0.01, z_lambda=1e-3,
                         sentinel_frac=0.10),
    # Mixtral-shaped: variant B, capacity 1.25, hot-spot +2.0 on expert 0
    "mix": LayerConfig("mix", T=32768, D=4096, E=8, K=2, F=14336, renorm=1,
                       capacity_factor=1.25, hot_expert_offset=2.0),
    # DeepSeek-V3-shaped: sigmoid + selection bias, 8 groups keep 4, 1 shared
    "ds3": LayerConfig("ds3", T=8192, D=7168, E=256, K=8, F=2048, n_shared=1,
                       score_fn=SIGMOID, renorm=1, n_groups=8, topk_groups=4,
                       sel_bias_range=0.1),
    # expert choice on the OLMoE shape: each of the 64 experts picks
    # C = 8*T/64 = 2048 tokens (the same expert FLOPs as top-8 token choice)
    "olmoe_ec": LayerConfig("olmoe_ec", T=16384, D=2048, E=64, K=64, F=1024, renorm=0,
                            capacity_factor=8.0, z_lambda=1e-3, expert_choice=1),
}

# Reduced variants: same options, sizes the oracle handles element by element.
REDUCED = {
    "tiny": CONFIGS["tiny"],
    "mm_a": CONFIGS["mm_a"].replace(name="mm_a_small", T=1000, D=256, F=512),
    "mm_b": CONFIGS["mm_b"].replace(name="mm_b_small", T=1000, D=256, F=512),
    "olmoe": CONFIGS["olmoe"].replace(name="olmoe_small", T=700, D=256, F=256),
    "mix": CONFIGS["mix"].replace(name="mix_small", T=2000, D=512, F=640),
    "ds3": CONFIGS["ds3"].replace(name="ds3_small", T=300, D=256, F=128),
    # enough rows per expert (>= 1536) that the expert GEMMs run on CTA pairs
    "mm_pair": CONFIGS["mm_b"].replace(name="mm_pair_small", T=6500, D=256, F=512),
    "mix_pair": CONFIGS["mix"].replace(name="mix_pair_small", T=7000, D=512, F=640),
    # one slot per token with capacity drops and sentinel slots: the tokens
    # without a row in the token-order (combine / dx) epilogues
    "mm_mask": CONFIGS["mm_a"].replace(name="mm_mask_small", T=1000, D=256, F=512,
                                       capacity_factor=0.9, sentinel_frac=0.05),
    # more than 16384 slots: the multi-block dispatch passes (ragged last block)
    "olmoe_multi": CONFIGS["olmoe"].replace(name="olmoe_multi_small", T=2600, D=128, F=128),
    # sequence-wise aux loss: softmax (OLMoE-shaped, 7 sequences) and sigmoid
    # affinities with groups and the shared expert (DeepSeek-shaped, 3 sequences)
    "olmoe_seq": CONFIGS["olmoe"].replace(name="olmoe_seq_small", T=700, D=256, F=256,
                                          seq_len=100),
    "ds3_seq": CONFIGS["ds3"].replace(name="ds3_seq_small", T=300, D=256, F=128,
                                      aux_alpha=1e-3, seq_len=100),
    # router split widths 16 and 32 (the E = 32 router runs on CTA pairs):
    # sigmoid + selection bias, variant B; softmax, variant A with aux + z
    "e16_sig": LayerConfig("e16_sig_small", T=900, D=256, E=16, K=4, F=256, score_fn=SIGMOID,
                           renorm=1, sel_bias_range=0.1),
    "e32": LayerConfig("e32_small", T=1500, D=384, E=32, K=2, F=256, renorm=0,
                       aux_alpha=0.01, z_lambda=1e-3),
    # 128 experts without a group limit: routing from the partial logits
    # with four lanes per token (the logits GEMM, then the routing kernel)
    "e128": LayerConfig("e128_small", T=600, D=256, E=128, K=4, F=128, renorm=1,
                        aux_alpha=0.01, z_lambda=1e-3, hot_expert_offset=1.0),
    # more tokens than one 128-row round of router tiles over all CTAs: several
    # tiles per CTA pair, ragged last tile
    "olmoe_tiles": CONFIGS["olmoe"].replace(name="olmoe_tiles_small", T=20000, D=128, F=128),
    # expert choice: 8 experts (with z-loss, C = 128 of 512 tokens) and the
    # OLMoE-shaped 64 experts at reduced size
    "ec8": LayerConfig("ec8_small", T=512, D=256, E=8, K=8, F=256, renorm=0,
                       capacity_factor=2.0, z_lambda=1e-3, expert_choice=1),
    "olmoe_ec": CONFIGS["olmoe_ec"].replace(name="olmoe_ec_small", T=1024, D=128, F=128,
                                            capacity_factor=2.0),
}


# Edge shapes of the routing path (same input recipe): a token count below
# one router or expert tile, select-all (K = E), expert counts that are not a
# split width (padding experts in the router's split), a count the four-lane
# routing kernel does not take, K = 1 in the fused router, sigmoid without a
# selection bias, 512 experts with a group limit, and few experts with a
# shared expert.
EDGE = {
    "t1_e64": CONFIGS["olmoe"].replace(name="edge_t1_e64", T=1, D=128, F=128),
    "t1_e4": CONFIGS["mm_b"].replace(name="edge_t1_e4", T=1, D=128, F=128),
    "t5_e8_cap": CONFIGS["mix"].replace(name="edge_t5_e8_cap", T=5, D=256, F=128),
    "t3_e256_groups": CONFIGS["ds3"].replace(name="edge_t3_e256_groups", T=3, D=256, F=128),
    "t130_e32": LayerConfig("edge_t130_e32", T=130, D=128, E=32, K=4, F=128, renorm=1,
                            aux_alpha=0.01),
    "k8_e8": LayerConfig("edge_k8_e8", T=300, D=128, E=8, K=8, F=128, renorm=1,
                         aux_alpha=0.01, z_lambda=1e-3),
    "k4_e4": LayerConfig("edge_k4_e4", T=200, D=128, E=4, K=4, F=128, renorm=0),
    "e48": LayerConfig("edge_e48", T=400, D=128, E=48, K=4, F=128, renorm=1,
                       z_lambda=1e-3, hot_expert_offset=1.0),
    "e12_sig": LayerConfig("edge_e12_sig", T=257, D=128, E=12, K=2, F=128,
                           score_fn=SIGMOID, renorm=1, route_scale=2.5),
    "e96_k6": LayerConfig("edge_e96_k6", T=333, D=128, E=96, K=6, F=128, renorm=0,
                          aux_alpha=0.01),
    "e64_k1": LayerConfig("edge_e64_k1", T=500, D=128, E=64, K=1, F=128, renorm=1,
                          aux_alpha=0.01),
    "e512_groups": LayerConfig("edge_e512_groups", T=64, D=128, E=512, K=8, F=128,
                               score_fn=SIGMOID, renorm=1, n_groups=16, topk_groups=4,
                               route_scale=2.5, sel_bias_range=0.1),
    # the router part of dx on CUDA cores (E <= 8) with a shared expert and
    # a row width that ends inside a 256-column slice; K = 1 with a shared
    # expert (no token-order epilogues)
    "e8_shared_d384": LayerConfig("edge_e8_shared_d384", T=300, D=384, E=8, K=2, F=128,
                                  n_shared=1, renorm=1, aux_alpha=0.01, capacity_factor=1.25),
    "e4_k1_shared": LayerConfig("edge_e4_k1_shared", T=333, D=256, E=4, K=1, F=128,
                                n_shared=1, renorm=0, aux_alpha=5e-4, sentinel_frac=0.05),
}


def get(name: str) -> LayerConfig:
    if name in CONFIGS:
        return CONFIGS[name]
    for c in list(REDUCED.values()) + list(EDGE.values()):
        if c.name == name:
            return c
    raise KeyError(name)


# ---------------------------------------------------------------------------
# Inputs
# ---------------------------------------------------------------------------
# Fixed stream ids per tensor (never Python's salted hash).
STREAM = {
    "x": 1, "w_r": 2, "w13": 3, "w_down": 4, "w13_s": 5, "w_down_s": 6,
    "dy": 7, "sel_bias": 8, "sentinel": 9,
}


def _dt(cfg: LayerConfig):
    import torch
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def make_input(cfg: LayerConfig, name: str, device="cpu", *, rows=None,
               expert=None):
    """One named input of `cfg` as a torch tensor on `device`.

    name: x [T,D] | dy [T,D] | w_r [E,D] fp32 | w13 [E,2F,D] | w_down [E,D,F]
          | w13_s [2F,D] | w_down_s [D,F] | logit_offset [E] fp32
          | sel_bias [E] fp32 | sentinel_mask [T*K] uint8
    rows:   optional 1-D index tensor of rows (tokens for x/dy) to produce
    expert: optional expert index for w13 / w_down (returns that expert only)
    Activations and expert weights are rounded (RNE) to the layer dtype;
    the router weight, offset and bias are fp32.
    """
    import torch
    dt = _dt(cfg)
    s = cfg.seed
    if name in ("x", "dy"):
        std = cfg.x_std if name == "x" else cfg.dy_std
        return gen.normal((cfg.T, cfg.D), s, STREAM[name], std, device,
                          rows=rows).to(dt)
    if name == "w_r":
        return gen.normal((cfg.E, cfg.D), s, STREAM[name], cfg.w_std,
                          device).to(torch.float32)
    if name == "w13":
        shape = (cfg.E, 2 * cfg.F, cfg.D)
        return gen.normal(shape, s, STREAM[name], cfg.w_std, device,
                          lead=expert).to(dt)
    if name == "w_down":
        shape = (cfg.E, cfg.D, cfg.F)
        return gen.normal(shape, s, STREAM[name], cfg.w_std, device,
                          lead=expert).to(dt)
    if name == "w13_s":
        return gen.normal((2 * cfg.F, cfg.D), s, STREAM[name], cfg.w_std,
                          device).to(dt)
    if name == "w_down_s":
        return gen.normal((cfg.D, cfg.F), s, STREAM[name], cfg.w_std,
                          device).to(dt)
    if name == "logit_offset":
        off = torch.zeros(cfg.E, dtype=torch.float32)
        off[0] = cfg.hot_expert_offset
        return off.to(device)
    if name == "sel_bias":
        return gen.uniform((cfg.E,), s, STREAM[name], -cfg.sel_bias_range,
                           cfg.sel_bias_range, device).to(torch.float32)
    if name == "sentinel_mask":
        m = torch.zeros(cfg.T * cfg.K, dtype=torch.uint8)
        n = cfg.n_sentinel
        if n > 0:
            g = torch.Generator().manual_seed(
                (s * 1000003 + STREAM["sentinel"]) & 0x7FFFFFFF)
            pick = torch.randperm(cfg.T * cfg.K, generator=g)[:n]
            m[pick] = 1
        return m.to(device)
    raise KeyError(name)


def optional_inputs(cfg: LayerConfig):
    """Names of the optional inputs this config uses."""
    out = []
    if cfg.hot_expert_offset != 0.0:
        out.append("logit_offset")
    if cfg.sel_bias_range != 0.0:
        out.append("sel_bias")
    if cfg.sentinel_frac > 0.0:
        out.append("sentinel_mask")
    return out
