"""GPU path vs the CPU oracle, element by element, on the reduced configs.

Every config keeps its full-size options (variants, sentinels, capacity,
groups, sigmoid + bias, shared expert) at sizes the oracle finishes in
seconds while spanning several 128-row tiles with ragged tails.

Bar (the layer's stated tolerances): routing indices, counts, kept,
drops, sentinels and the permutation bit-exact except top-k near-ties
(fp32 margin < 1e-5, counted); every float output and gradient within
relative L2 2e-2 for bf16 compute and 1e-4 for the fp32 config.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O
from tests.helpers import oracle_layer, rel_l2

pytestmark = pytest.mark.gpu


def tol(cfg):
    return 1e-4 if cfg.dtype == "fp32" else 2e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_routing_fp32_b200.build import build
    build()


def gpu_inputs(cfg, dev="cuda"):
    d = {n: W.make_input(cfg, n, dev) for n in ("x", "w_r", "w13", "w_down", "dy")}
    d["w13_s"] = W.make_input(cfg, "w13_s", dev) if cfg.n_shared else None
    d["w_down_s"] = W.make_input(cfg, "w_down_s", dev) if cfg.n_shared else None
    d["logit_offset"] = W.make_input(cfg, "logit_offset", dev) if cfg.hot_expert_offset else None
    d["sel_bias"] = W.make_input(cfg, "sel_bias", dev) if cfg.sel_bias_range else None
    d["sentinel_mask"] = W.make_input(cfg, "sentinel_mask", dev) if cfg.sentinel_frac else None
    return d


def run_gpu(cfg, gemm_impl=0, inp=None, gather=False):
    from mixture_experts_routing_fp32_b200 import MoELayer, config_from, moe_check_status
    layer = MoELayer(config_from(cfg, gemm_impl=gemm_impl), gather=gather)
    inp = inp or gpu_inputs(cfg)
    layer.forward(inp["x"], inp["w_r"], inp["w13"], inp["w_down"], inp["w13_s"],
                  inp["w_down_s"], inp["logit_offset"], inp["sel_bias"],
                  inp["sentinel_mask"])
    layer.backward(inp["dy"])
    assert moe_check_status() == 0
    return layer, inp


def host(t):
    return t.detach().float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()


def gpu_routed_oracle(cfg, layer, R):
    """The GPU's selection checked against the oracle's (bit-exact except on
    near-tie tokens, fp32 margin < 1e-5), then the oracle's dispatch of the
    GPU's own selection: the permutation every later output depends on.
    Returns (flipped tokens, oracle Dispatch of the GPU's idx)."""
    idx = layer.topk_idx.cpu().numpy()
    diff = np.nonzero((idx != R.idx).any(axis=1))[0]
    assert np.all(R.margin[diff] < O.NEAR_TIE), ("non-near-tie routing mismatch", diff[:10])
    mask = W.make_input(cfg, "sentinel_mask").numpy() if cfg.sentinel_frac else None
    Dp = O.dispatch(idx, cfg.E, cfg.capacity_factor, cfg.min_capacity, mask)
    return diff, Dp


def check_dispatch(cfg, layer, R, Dp=None):
    """Bit-exact routing and permutation.  The selection matches the oracle's
    except on near-tie tokens; the dispatch (counts, kept, drops, sentinels,
    every slot's expert and rank) matches the oracle's counting sort of the
    GPU's own selection exactly.  Returns (number of flipped tokens, that
    oracle Dispatch)."""
    diff, Dg = gpu_routed_oracle(cfg, layer, R)
    if diff.size == 0 and Dp is not None:
        assert np.array_equal(Dg.rank, Dp.rank) and np.array_equal(Dg.expert, Dp.expert)
    E, K, T = cfg.E, cfg.K, cfg.T
    counts, kept = host(layer.counts), host(layer.kept)
    offsets, stats = host(layer.offsets), host(layer.stats)
    slot_row, row_slot = host(layer.slot_row), host(layer.row_slot)
    tile_e = host(layer.tile_expert)
    n_rows = int(stats[2])
    assert n_rows % 128 == 0 and stats[3] * 128 == n_rows
    # permutation in the GPU's padded row space -> (expert, rank) per slot
    ex = np.full(T * K, -1)
    rk = np.full(T * K, -1)
    kept_slots = np.nonzero(slot_row >= 0)[0]
    rows = slot_row[kept_slots]
    assert np.all(rows < n_rows)
    ex[kept_slots] = tile_e[rows // 128]
    rk[kept_slots] = rows - offsets[ex[kept_slots]]
    assert np.all(row_slot[rows] == kept_slots)                    # inverse map
    assert np.all(ex[kept_slots] < E)
    align = int(layer.sizes.row_align)                             # padded layout
    assert align in (128, 256)
    for e in range(E):
        assert offsets[e] % align == 0
        assert offsets[e + 1] - offsets[e] == -(-kept[e] // align) * align
    pad_rows = np.ones(n_rows, dtype=bool)
    pad_rows[rows] = False
    if cfg.n_shared:
        pad_rows[offsets[E]:offsets[E] + T] = False
    assert np.all(row_slot[:n_rows][pad_rows] == -1)
    if layer.x_perm is not None:
        assert np.all(host(layer.x_perm)[:n_rows][pad_rows] == 0)
        # every gathered row is its token's row of x, bit for bit
        dev = layer.x_perm.device
        xg = W.make_input(cfg, "x", dev)
        rt = torch.from_numpy(rows.astype(np.int64)).to(dev)
        tt = torch.from_numpy((kept_slots // K).astype(np.int64)).to(dev)
        assert torch.equal(layer.x_perm[rt], xg[tt])
        if cfg.n_shared:
            s0 = int(offsets[E])
            assert torch.equal(layer.x_perm[s0:s0 + T], xg)
    assert np.array_equal(counts, Dg.counts)
    assert np.array_equal(kept, Dg.kept)
    assert int(stats[0]) == Dg.n_drop
    assert int(stats[1]) == Dg.n_sentinel
    assert np.array_equal(ex, np.where(Dg.rank >= 0, Dg.expert, -1))
    assert np.array_equal(rk, Dg.rank)
    assert np.all(slot_row[Dg.sentinel] == -2) and np.all(slot_row[Dg.dropped] == -1)
    return diff.size, Dg


def oracle_on_gpu_routing(cfg, layer, L=None):
    """Oracle forward + backward on the GPU's own top-K selection (identical
    to the oracle's own except on near-tie tokens, which route_layer checks
    and counts).  Returns (fw, bw, flips)."""
    L = L or oracle_layer(cfg)
    o = O.opts_of(cfg)
    R_own = O.route_layer(L, o)
    flips, _ = check_dispatch(cfg, layer, R_own)
    fw = O.forward(L, o, idx_given=layer.topk_idx.cpu().numpy())
    bw = O.backward(L, o, fw, W.make_input(cfg, "dy").double().numpy())
    return fw, bw, flips


@pytest.mark.parametrize("name", [n for n, c in W.REDUCED.items() if not c.expert_choice])
def test_parity_reduced(name):
    check_layer_parity(name, W.REDUCED[name])


@pytest.mark.parametrize("name", list(W.EDGE))
def test_parity_edge_shapes(name):
    """One token, a few tokens, select-all, padding experts in the router's
    split, the general routing kernel, K = 1 in the fused router, sigmoid
    without a bias, 512 experts with groups: the same bar as the reduced
    configs."""
    check_layer_parity(name, W.EDGE[name])


def check_layer_parity(name, cfg):
    layer, inp = run_gpu(cfg)
    fw, bw, flips = oracle_on_gpu_routing(cfg, layer)
    R = fw["R"]
    tl = tol(cfg)
    # router (fp32 on both sides)
    assert rel_l2(host(layer.logits), R.logits) < 1e-5
    assert rel_l2(host(layer.probs), R.p) < 1e-5
    assert rel_l2(host(layer.lse), R.lse) < 1e-5
    assert rel_l2(host(layer.topk_w), R.g) < 1e-5
    # forward output and losses
    assert rel_l2(host(layer.y), fw["y"]) < tl
    if cfg.aux_alpha:
        assert abs(float(layer.losses[0]) - fw["aux"]) <= 1e-5 * abs(fw["aux"])
    if cfg.z_lambda:
        assert abs(float(layer.losses[1]) - fw["z"]) <= 1e-5 * abs(fw["z"])
    # gradients
    assert rel_l2(host(layer.dg), bw["dg"]) < tl
    assert rel_l2(host(layer.dlogits), bw["ds"]) < tl
    assert rel_l2(host(layer.dw_r), bw["dw_r"]) < tl
    assert rel_l2(host(layer.dx), bw["dx"]) < tl
    dw13 = np.stack([bw["dw13"][e] for e in range(cfg.E)])
    dwd = np.stack([bw["dwd"][e] for e in range(cfg.E)])
    assert rel_l2(host(layer.dw13), dw13) < tl
    assert rel_l2(host(layer.dw_down), dwd) < tl
    if cfg.n_shared:
        assert rel_l2(host(layer.dw13_s), bw["dw13_s"]) < tl
        assert rel_l2(host(layer.dw_down_s), bw["dwd_s"]) < tl
    # sentinel and dropped slots: zero gate gradient, exactly
    masked = (host(layer.slot_row) < 0).reshape(cfg.T, cfg.K)
    assert np.all(host(layer.dg)[masked] == 0.0)
    if cfg.K == 1 and not cfg.n_shared:
        # a token whose only slot has no row: y_t = 0 exactly (written by the
        # down projection's epilogue when it does the combine)
        assert np.all(host(layer.y)[masked[:, 0]] == 0.0)
    print("%s: near-tie flips %d, GPU near-tie count %d, drops %d, sentinels %d" % (
        name, flips, int(layer.near_ties[0]), int(layer.stats[0]), int(layer.stats[1])))


@pytest.mark.parametrize("name", ["mm_a", "olmoe", "mix", "ds3", "mm_pair", "mix_pair"])
def test_tensor_core_path_matches_simt_path(name):
    """The tcgen05 GEMMs against the CUDA-core GEMMs on the same inputs."""
    cfg = W.REDUCED[name]
    tc, inp = run_gpu(cfg, gemm_impl=0)
    simt, _ = run_gpu(cfg, gemm_impl=1, inp=inp)
    # both paths compute fp32-accurate logits (tensor cores on three-way
    # bf16 splits for E >= 8, CUDA cores otherwise), in different orders
    assert rel_l2(host(tc.logits), host(simt.logits).astype(np.float64)) < 2e-6
    # a token may pick differently only where the exact logits nearly tie
    flip = (tc.topk_idx != simt.topk_idx).any(dim=1).cpu().numpy()
    if flip.any():
        R = O.forward(oracle_layer(cfg), O.opts_of(cfg))["R"]
        assert np.all(R.margin[flip] < O.NEAR_TIE), np.nonzero(flip)[0][:10]
    keep = torch.from_numpy(~flip).to(tc.y.device)
    for attr in ("y", "dx", "dg"):
        a, b = getattr(tc, attr).float()[keep], getattr(simt, attr).float()[keep]
        assert (a - b).norm() / b.norm() < 1e-2, attr
    for attr in ("dw13", "dw_down", "dw_r"):
        a, b = getattr(tc, attr).float(), getattr(simt, attr).float()
        assert (a - b).norm() / b.norm() < (1e-2 if not flip.any() else 5e-2), attr
    # the two paths may align expert segments differently (CTA-pair tiles
    # use 256-row segments): compare every slot's expert and rank instead
    # (each path's permutation is also checked against the oracle's
    # counting sort of its own selection in test_parity_reduced)
    def expert_rank(L):
        sr = L.slot_row.long()
        kept = sr >= 0
        e = torch.full_like(sr, -1)
        r = torch.full_like(sr, -1)
        e[kept] = L.tile_expert.long()[sr[kept] // 128]
        r[kept] = sr[kept] - L.offsets.long()[e[kept]]
        return e, r
    if not flip.any():
        for a, b in zip(expert_rank(tc), expert_rank(simt)):
            assert torch.equal(a, b)
    print("%s: tensor-core vs SIMT selection flips %d" % (name, int(flip.sum())))


def test_k1_variant_b_router_grad_is_exactly_aux_only():
    """MiniMind-shaped K=1: variant B's router gradient does not depend on
    the upstream gradient at all (only the aux loss reaches the router);
    variant A's does (STA324 §8.3; MiniMind issue §2)."""
    for name, zero in (("mm_b", True), ("mm_a", False)):
        cfg = W.REDUCED[name]
        layer, inp = run_gpu(cfg)
        d1, w1 = layer.dlogits.clone(), layer.dw_r.clone()
        layer.backward(inp["dy"] * -3.0)
        torch.cuda.synchronize()
        same = torch.equal(d1, layer.dlogits) and torch.equal(w1, layer.dw_r)
        assert same == zero, name
        if zero:
            assert float(layer.dw_r.abs().sum()) > 0     # the aux gradient is there


def test_generator_identical_on_gpu_and_cpu():
    cfg = W.REDUCED["ds3"]
    for n in ("x", "w13", "w_r", "sel_bias"):
        assert torch.equal(W.make_input(cfg, n, "cuda").cpu(), W.make_input(cfg, n))


def test_device_error_word_on_bad_expert_id():
    """An expert id outside [-1, E) is reported through the error word and
    the slot is treated as a sentinel (host-planted; no GPU fault)."""
    from mixture_experts_routing_fp32_b200 import MoELayer, config_from, api, MoEError
    cfg = W.REDUCED["mm_a"]
    layer = MoELayer(config_from(cfg))
    x = W.make_input(cfg, "x", "cuda")
    idx = torch.zeros(cfg.T, cfg.K, dtype=torch.int32, device="cuda")
    idx[5, 0] = cfg.E + 3
    api.moe_dispatch(layer.cfg, idx, None, x, layer.counts, layer.kept, layer.offsets,
                     layer.slot_row, layer.row_slot, layer.tile_expert, layer.stats,
                     layer.x_perm, layer.ws)
    with pytest.raises(MoEError):
        api.moe_check_status()
    assert int(layer.stats[1]) == 1 and int(layer.slot_row[5 * cfg.K]) == -2
    assert api.moe_check_status() == 0          # the word was cleared


def test_bias_update_matches_oracle():
    """The selection-bias step on the GPU's own counts, bit for bit: each
    side subtracts or adds the same fp32 gamma once."""
    from oracle import balance as B
    cfg = W.REDUCED["ds3"]
    layer, inp = run_gpu(cfg)
    bias = inp["sel_bias"].clone()
    gamma = 1e-3
    layer.update_bias(bias, gamma)
    torch.cuda.synchronize()
    exp = B.bias_update(layer.counts.cpu().numpy(), inp["sel_bias"].cpu().double().numpy(),
                        float(np.float32(gamma))).astype(np.float32)
    np.testing.assert_array_equal(bias.cpu().numpy(), exp)
    n = layer.counts.cpu().numpy()
    moved = bias.cpu().numpy() - inp["sel_bias"].cpu().numpy()
    assert np.all(moved[n * cfg.E > n.sum()] < 0) and np.all(moved[n * cfg.E < n.sum()] > 0)


def test_sentinel_slots_are_marked_minus_two():
    cfg = W.REDUCED["olmoe"]
    layer, _ = run_gpu(cfg)
    mask = W.make_input(cfg, "sentinel_mask").numpy().astype(bool)
    sr = layer.slot_row.cpu().numpy()
    assert np.all(sr[mask] == -2)
    assert np.all(sr[~mask] >= -1)


def ec_oracle_on_gpu_choice(cfg, layer):
    """Expert-choice oracle on the GPU's own picks: each expert's C picks
    bit-exact against the oracle's except experts whose C-th and (C+1)-th
    fp32 scores nearly tie (counted); then the oracle's forward and backward
    with the GPU's picks.  Returns (Lc, o, fw, bw, R, n_flipped_experts)."""
    from oracle import expert_choice as X
    L = oracle_layer(cfg)
    R, chosen_own, C = X.route(L, cfg.capacity_factor, cfg.min_capacity)
    T, E = cfg.T, cfg.E
    chosen = layer.ec_mask.cpu().numpy().reshape(T, E) == 0
    assert np.all(chosen.sum(axis=0) == C)
    flip = (chosen != chosen_own).any(axis=0)
    assert np.all(X.ec_margin(R.p, C)[flip] < O.NEAR_TIE), np.nonzero(flip)[0]
    Lc = X.layer_for(L, chosen)
    o = X.opts_for(E, cfg.z_lambda)
    fw = O.forward_routed(Lc, o, R)
    fw["chosen"], fw["C"] = chosen, C
    bw = O.backward(Lc, o, fw, W.make_input(cfg, "dy").double().numpy())
    return Lc, o, fw, bw, R, int(flip.sum())


@pytest.mark.parametrize("name", ["ec8", "olmoe_ec"])
def test_expert_choice_parity(name):
    """Expert choice against its oracle: every expert's picks bit-exact
    (except experts whose C-th and (C+1)-th fp32 scores nearly tie, where the
    oracle then runs on the GPU's picks), exactly C rows per expert, outputs
    and all gradients within the bf16 tolerance."""
    cfg = W.REDUCED[name]
    layer, inp = run_gpu(cfg)
    Lc, o, fw, bw, R, flips = ec_oracle_on_gpu_choice(cfg, layer)
    E, C = cfg.E, fw["C"]
    assert rel_l2(host(layer.logits), R.logits) < 1e-5
    assert rel_l2(host(layer.probs), R.p) < 1e-5
    assert np.array_equal(host(layer.counts), np.full(E, C))
    Dp = fw["Dp"]
    assert np.array_equal(host(layer.slot_row) >= 0, Dp.rank >= 0)
    assert rel_l2(host(layer.y), fw["y"]) < tol(cfg)
    for attr, ref in (("dx", bw["dx"]), ("dw_r", bw["dw_r"]), ("dg", bw["dg"]),
                      ("dlogits", bw["ds"])):
        assert rel_l2(host(getattr(layer, attr)), ref) < tol(cfg), attr
    assert rel_l2(host(layer.dw13), np.stack([bw["dw13"][e] for e in range(E)])) < tol(cfg)
    assert rel_l2(host(layer.dw_down), np.stack([bw["dwd"][e] for e in range(E)])) < tol(cfg)
    if cfg.z_lambda:
        assert abs(float(layer.losses[1]) - fw["z"]) <= 1e-5 * abs(fw["z"])
    print("%s: expert-choice near-tie flips %d (experts), GPU near-ties %d" % (
        name, flips, int(layer.near_ties[0])))


def padding_rows(layer, cfg):
    """Rows in use that hold neither a routed slot nor a shared-expert token."""
    n = int(layer.stats[2])
    rs = layer.row_slot[:n].long()
    r = torch.arange(n, device=rs.device)
    s0 = int(layer.offsets[cfg.E])
    shared = (r >= s0) & (r < s0 + cfg.T) if cfg.n_shared else torch.zeros_like(rs, dtype=torch.bool)
    return (rs < 0) & ~shared


GRAD_ATTRS = ("y", "dx", "dw13", "dw_down", "dw_r", "dg", "dlogits")


def assert_gather_identical(cfg, ref, fused):
    """Same operands in shared memory, same MMAs: bit-identical results."""
    assert fused.x_perm is None
    n = int(ref.stats[2])
    assert torch.equal(ref.row_slot[:n], fused.row_slot[:n])
    for attr in ("a13", "h", "o"):
        assert torch.equal(getattr(fused, attr)[:n], getattr(ref, attr)[:n]), attr
    attrs = GRAD_ATTRS + (("dw13_s", "dw_down_s") if cfg.n_shared else ())
    for attr in attrs:
        assert torch.equal(getattr(fused, attr), getattr(ref, attr)), attr
    # padding rows were gathered from outside x: zeros, like the permuted copy
    pad = padding_rows(fused, cfg)
    assert torch.count_nonzero(fused.a13[:n][pad]) == 0
    assert torch.count_nonzero(fused.h[:n][pad]) == 0


@pytest.mark.parametrize("name", ["mm_b", "olmoe", "mix", "ds3", "mm_pair", "mix_pair", "ec8",
                                  "olmoe_ec"])
def test_fused_gather_matches_permuted_copy(name):
    """gate/up A rows (forward) and gate/up weight-gradient B rows (backward)
    copied from the token rows of x by the GEMMs' producer warp (cp.async)
    (single CTAs and CTA pairs, shared expert, expert choice, capacity
    drops, sentinels) against the same GEMMs on the dispatch's permuted copy
    of x, and against the oracle."""
    cfg = W.REDUCED[name]
    ref, inp = run_gpu(cfg)
    fused, _ = run_gpu(cfg, inp=inp, gather=True)
    assert_gather_identical(cfg, ref, fused)
    if cfg.expert_choice:
        _, _, fw, bw, _, flips = ec_oracle_on_gpu_choice(cfg, fused)
    else:
        fw, bw, flips = oracle_on_gpu_routing(cfg, fused)
    assert rel_l2(host(fused.y), fw["y"]) < tol(cfg)
    assert rel_l2(host(fused.dx), bw["dx"]) < tol(cfg)
    assert rel_l2(host(fused.dw13), np.stack([bw["dw13"][e] for e in range(cfg.E)])) < tol(cfg)
    assert rel_l2(host(fused.dw_down), np.stack([bw["dwd"][e] for e in range(cfg.E)])) < tol(cfg)
    assert rel_l2(host(fused.dw_r), bw["dw_r"]) < tol(cfg)
    print("%s fused gather: near-tie flips %d" % (name, flips))


@pytest.mark.parametrize("name", ["mm_b", "mm_mask", "mm_pair"])
def test_token_order_epilogues_match_separate_kernels(name):
    """One slot per token: y written by the down GEMM's epilogue (scaled by g
    from the fp32 accumulator) against moe_expert_ffn + moe_combine on the
    same layer buffers; o itself is bit-identical."""
    from mixture_experts_routing_fp32_b200 import api
    cfg = W.REDUCED[name]
    layer, inp = run_gpu(cfg)
    c = layer.cfg
    y_fused, o_fused = layer.y.clone(), layer.o.clone()
    api.moe_expert_ffn(c, layer.x_perm, layer.offsets, layer.tile_expert, layer.stats,
                       inp["w13"], inp["w_down"], None, None, layer.a13, layer.h, layer.o,
                       layer.ws)
    api.moe_combine(c, layer.o, layer.slot_row, layer.topk_w, layer.offsets, layer.y)
    torch.cuda.synchronize()
    n = int(layer.stats[2])
    assert torch.equal(o_fused[:n], layer.o[:n])
    a, b = y_fused.float(), layer.y.float()
    # the separate path rounds o to bf16 before scaling: the two differ by
    # at most two bf16 roundings, |a - b| <= 2^-7 |b| elementwise
    assert torch.all((a - b).abs() <= (2.0 ** -7) * b.abs())
    assert torch.equal(a == 0, b == 0)
