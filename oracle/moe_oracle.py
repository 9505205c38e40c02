"""Plain CPU oracle for the token-choice MoE layer, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only
tests/, the smoke check in __graft_entry__.py and the CPU-baseline leg of
bench.py may call it.  It shares no code with the CUDA path.

Everything is float64 numpy with library matmuls as the only primitive,
written step by step in the order the pages give them.  The one deliberate
exception is the router logit: the pages keep the router in fp32 ("8-MoE"
lecture notes, Switch Transformers, mixed-precision strategy; STA324 notes
"08 MoE", §8.6), so the logit s = x W_r^T (+ offset) is formed exactly and
rounded once to float32, and every routing decision (top-k, group limit) is
taken on values derived from those float32 logits.

Pages cited (by title and section):
  [STA324]   "08 MoE：容量、路由、梯度、均衡和系统实现" (STA324 notes), §8.1-§8.9
  [TRAIN]    "MoE 训练：稀疏计算背后的路由与通信" (MoE training course page)
  [8MOE]     "8-MoE" lecture notes (Router / Gating Network, KeepTopK,
             Expert Capacity, GShard, Switch Transformers, ST-MoE,
             MoE 高效推理 / token grouping & permutation)
  [HF48687]  "Wrong router gradient with experts_implementation=batched_mm
             under expert parallelism" (transformers issue summary)
  [MM858]    "[Bug] num_experts_per_tok=1 时 MoE 路由器收不到梯度" (MiniMind issue)

Pins: every function here is pinned by tests in tests/test_oracle_*.py
against worked examples printed on the pages, closed forms, brute force,
special cases that reduce to library routines, and finite differences.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, Optional

import numpy as np

from . import balance

SOFTMAX, SIGMOID = 0, 1
GROUP_MAX, GROUP_TOP2SUM = 0, 1
NEAR_TIE = 1e-5          # fp32-margin below which a top-k decision is a near-tie
SIGMOID_EPS = 1e-20      # added to the sum of selected sigmoid affinities


def f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------
def router_logits(x, w_r, logit_offset=None, round_fp32=True) -> np.ndarray:
    """s_{t,e} = sum_d x_{t,d} W_r[e,d] (+ offset_e), rounded to float32.

    [STA324] §8.2: the router is one linear map from the token to E logits;
    [8MOE] GShard routing network (linear layer then softmax) and Switch
    Transformers (the router stays in full precision).  W_r is stored [E, D]
    like nn.Linear(D, E).
    """
    s = f64(x) @ f64(w_r).T
    if logit_offset is not None:
        s = s + f64(logit_offset)[None, :]
    # round_fp32=False keeps float64 logits (finite-difference checks only)
    return s.astype(np.float32) if round_fp32 else s


def softmax_rows(s) -> np.ndarray:
    s = f64(s)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=1, keepdims=True)


def logsumexp_rows(s) -> np.ndarray:
    s = f64(s)
    m = s.max(axis=1)
    return m + np.log(np.exp(s - m[:, None]).sum(axis=1))


def sigmoid(s) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-f64(s)))


@dataclass
class Routing:
    logits: np.ndarray      # [T,E] float32
    p: np.ndarray           # [T,E] scores: softmax probs or sigmoid affinities
    lse: np.ndarray         # [T]   logsumexp of the logits (z-loss)
    idx: np.ndarray         # [T,K] int, selected experts, best first
    g: np.ndarray           # [T,K] gate weights (after route_scale)
    margin: np.ndarray      # [T]   min gap among the top K+1 scores and at the group boundary


def route(logits, K, *, score_fn=SOFTMAX, renorm=1, n_groups=1,
          topk_groups=1, group_score=GROUP_MAX, route_scale=1.0,
          sel_bias=None, idx_given=None) -> Routing:
    """Scores, group-limited top-K selection and gate weights.

    Score function ([STA324] §8.2, §8.6):
      softmax: p = softmax(s); the selection score is the logit s itself
               (§8.2 applies TopK to the logits), which orders experts
               exactly as p does.
      sigmoid: p = sigmoid(s) (affinity); selection uses p + b_e, while the
               gate weights use the raw affinity p without b (§8.6: the bias
               steers the choice only, the mixing weights come from the
               unbiased affinity).
    Group limit ([STA324] §8.2 and [TRAIN] name "group-limited routing"
    without defining the group score): experts form n_groups contiguous
    groups; a group's score is the max of its selection scores (GROUP_MAX,
    the plainest reading) or the sum of its two largest (GROUP_TOP2SUM); the
    topk_groups best groups are kept and all other experts are excluded.
    Top-K: descending selection score; equal scores go to the lower index.
    Gate weights ([STA324] §8.2, worked example [.50,.30,.15,.05]):
      A (renorm=0): g_k = p_{idx_k}, no renormalisation, sum < 1
      B (renorm=1), softmax: g_k = exp(s_k) / sum_{j in T} exp(s_j)
      B (renorm=1), sigmoid: g_k = p_k / (sum_{j in T} p_j + 1e-20)
    then g *= route_scale ([TRAIN]: implementations may add a scaling).
    idx_given (tests only): a [T,K] selection to use instead of this
    function's own top-K (another implementation's choices on near-tie
    tokens); scores, margins and the gate-weight formulas are unchanged.
    """
    s32 = np.asarray(logits)
    s = f64(s32)
    T, E = s.shape
    lse = logsumexp_rows(s)
    if score_fn == SOFTMAX:
        p = softmax_rows(s)
        u = s.copy()
    else:
        p = sigmoid(s)
        u = p + (f64(sel_bias)[None, :] if sel_bias is not None else 0.0)

    margin = np.full(T, np.inf)
    if n_groups > 1:
        gs = E // n_groups
        ug = u.reshape(T, n_groups, gs)
        if group_score == GROUP_MAX:
            gscore = ug.max(axis=2)
        else:
            srt = -np.sort(-ug, axis=2)
            gscore = srt[:, :, 0] + srt[:, :, 1]
        gorder = np.argsort(-gscore, axis=1, kind="stable")
        keep = gorder[:, :topk_groups]
        if topk_groups < n_groups:
            gsorted = np.take_along_axis(gscore, gorder, axis=1)
            margin = np.minimum(margin, gsorted[:, topk_groups - 1]
                                - gsorted[:, topk_groups])
        allowed = np.zeros((T, n_groups), dtype=bool)
        np.put_along_axis(allowed, keep, True, axis=1)
        u = np.where(np.repeat(allowed, gs, axis=1), u, -np.inf)

    order = np.argsort(-u, axis=1, kind="stable")
    idx = order[:, :K].copy()
    if idx_given is not None:
        idx = np.asarray(idx_given).astype(np.int64).reshape(T, K)
    usorted = np.take_along_axis(u, order, axis=1)
    # smallest gap between consecutive selection scores among the top K+1:
    # both which experts are chosen and their slot order hang on these
    top = usorted[:, :min(K + 1, E)]
    if top.shape[1] > 1:
        gaps = top[:, :-1] - top[:, 1:]
        gaps = np.where(np.isfinite(top[:, 1:]), gaps, np.inf)
        margin = np.minimum(margin, gaps.min(axis=1))

    if score_fn == SOFTMAX:
        if renorm:
            sel = np.take_along_axis(s, idx, axis=1)
            m = sel.max(axis=1, keepdims=True)
            e = np.exp(sel - m)
            g = e / e.sum(axis=1, keepdims=True)
        else:
            g = np.take_along_axis(p, idx, axis=1)
    else:
        sel = np.take_along_axis(p, idx, axis=1)
        g = sel / (sel.sum(axis=1, keepdims=True) + SIGMOID_EPS) if renorm else sel
    g = g * route_scale
    return Routing(logits=s32, p=p, lse=lse, idx=idx.astype(np.int64), g=g,
                   margin=margin)


# ---------------------------------------------------------------------------
# Capacity and dispatch
# ---------------------------------------------------------------------------
def capacity(T, K, E, capacity_factor, min_capacity=0) -> Optional[int]:
    """C = max(ceil(c*T*K/E), min_capacity); None (no limit) when c <= 0.

    [STA324] §8.5 gives ceil(c*T*K/E); [TRAIN] (capacity, dropless and group
    routing trade-offs) gives about c*T*k/E; [8MOE] Switch Transformers gives
    tokens per batch / experts x capacity factor.  T*K is the nominal slot
    count.
    """
    if capacity_factor is None or capacity_factor <= 0:
        return None
    c = math.ceil(float(capacity_factor) * float(T * K) / float(E))
    return max(int(c), int(min_capacity))


@dataclass
class Dispatch:
    counts: np.ndarray      # [E] valid (non-sentinel) slots per expert, before drops
    kept: np.ndarray        # [E] min(counts, C)
    offsets: np.ndarray     # [E+1] exclusive scan of kept (compact rows)
    expert: np.ndarray      # [T*K] expert of each slot, -1 for sentinel slots
    rank: np.ndarray        # [T*K] position within its expert, -1 if dropped/sentinel
    dropped: np.ndarray     # [T*K] bool: valid slot beyond capacity
    sentinel: np.ndarray    # [T*K] bool
    C: Optional[int]

    @property
    def n_drop(self) -> int:
        return int(self.dropped.sum())

    @property
    def n_sentinel(self) -> int:
        return int(self.sentinel.sum())

    def row(self) -> np.ndarray:
        """Compact row of each slot (offsets[e] + rank), -1 when not kept."""
        r = np.full(self.rank.shape, -1, dtype=np.int64)
        k = self.rank >= 0
        r[k] = self.offsets[self.expert[k]] + self.rank[k]
        return r


def dispatch(idx, E, capacity_factor=0.0, min_capacity=0,
             sentinel_mask=None) -> Dispatch:
    """Counting-sort dispatch with capacity drop and sentinel slots.

    Slots are the (t,k) pairs in flat order j = t*K + k.  Walking them in that
    order, each valid slot of expert e takes rank n_e and n_e grows by one
    ([8MOE] MoE 高效推理: sort tokens by expert id so an expert's tokens are
    contiguous; [STA324] §8.8 gather tokens per expert).  A slot whose rank
    reaches the capacity C is dropped ([8MOE] Expert Capacity / GShard drop
    tokens; [TRAIN]: a dropped assignment loses one branch, the token may keep
    its other one).  Sentinel slots (expert id -1, or flagged in
    sentinel_mask) have no local expert: they take no rank, are not counted,
    and contribute nothing ([HF48687] cause analysis; [STA324] §8.5 padding
    must not pollute load statistics).  Counts are taken before drops: f in
    the aux loss is the actual selection frequency ([TRAIN]).
    """
    idx = np.asarray(idx)
    T, K = idx.shape
    expert = idx.reshape(-1).astype(np.int64).copy()
    if sentinel_mask is not None:
        expert[np.asarray(sentinel_mask).reshape(-1).astype(bool)] = -1
    sentinel = expert < 0
    C = capacity(T, K, E, capacity_factor, min_capacity)
    counts = np.zeros(E, dtype=np.int64)
    rank = np.full(T * K, -1, dtype=np.int64)
    dropped = np.zeros(T * K, dtype=bool)
    for j in range(T * K):
        e = expert[j]
        if e < 0:
            continue
        r = counts[e]
        counts[e] += 1
        if C is None or r < C:
            rank[j] = r
        else:
            dropped[j] = True
    kept = counts.copy() if C is None else np.minimum(counts, C)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    return Dispatch(counts=counts, kept=kept, offsets=offsets, expert=expert,
                    rank=rank, dropped=dropped, sentinel=sentinel, C=C)


# ---------------------------------------------------------------------------
# Expert FFN (SwiGLU)
# ---------------------------------------------------------------------------
def silu(a):
    return a / (1.0 + np.exp(-a))


def swiglu_forward(xr, w13, wd):
    """One SwiGLU expert on the rows xr.

    [STA324] §8.1: each SwiGLU expert has about 3DF parameters: a gate and an
    up projection D->F and a down projection F->D.  Plain reading: h =
    silu(x W_gate^T) * (x W_up^T), o = h W_down^T, with W13 = [W_gate; W_up]
    stored [2F, D] and W_down stored [D, F].
    """
    xr, w13, wd = f64(xr), f64(w13), f64(wd)
    F = wd.shape[1]
    a = xr @ w13[:F].T
    b = xr @ w13[F:].T
    h = silu(a) * b
    o = h @ wd.T
    return a, b, h, o


def swiglu_backward(xr, a, b, h, do, w13, wd):
    """Chain rule through o = (silu(a)*b) W_down^T, a|b = x W13^T."""
    xr, w13, wd = f64(xr), f64(w13), f64(wd)
    dh = do @ wd                                   # [rows, F]
    dwd = do.T @ h                                 # [D, F]
    sa = 1.0 / (1.0 + np.exp(-a))
    dsilu = sa * (1.0 + a * (1.0 - sa))
    da = dh * b * dsilu
    db = dh * silu(a)
    da13 = np.concatenate([da, db], axis=1)        # [rows, 2F]
    dw13 = da13.T @ xr                             # [2F, D]
    dxr = da13 @ w13                               # [rows, D]
    return dxr, dw13, dwd


# ---------------------------------------------------------------------------
# Losses
# ---------------------------------------------------------------------------
def aux_loss(counts, p, alpha, E):
    """Switch-style load-balance loss L = alpha * E * sum_e f_e P_e.

    f_e = n_e / sum_e n_e (hard, pre-drop, valid slots; constant for the
    gradient), P_e = mean_t p_{t,e}.  [TRAIN] (why load balance matters)
    gives the form E * sum_e f_e p_e; [STA324] §8.5: uniform routing gives
    alpha, full collapse about alpha*E, and its example E=2, f=[.75,.25],
    P=[.6,.4], alpha=.01 gives .011.
    Reading: the slot-count denominator sum_e n_e equals T*K without
    sentinels and keeps the uniform value at alpha for any K ([STA324] §8.5
    warns the TopK form's denominator varies).
    """
    counts = f64(counts)
    tot = counts.sum()
    f = counts / tot if tot > 0 else np.zeros_like(counts)
    P = f64(p).mean(axis=0)
    return float(alpha * E * np.dot(f, P)), f, P


def aux_loss_from_stats(counts, p_sum, n_tokens, alpha, E):
    """aux_loss() from pooled statistics of a batch split into parts (for
    example data-parallel ranks): counts summed over the parts, p_sum[e] =
    sum over all the batch's tokens of p_{t,e}, n_tokens = its token count,
    so P_e = p_sum_e / n_tokens.  [STA324] §8.5: the balance statistic may
    be taken over the whole batch or over all devices.
    """
    counts = f64(counts)
    tot = counts.sum()
    f = counts / tot if tot > 0 else np.zeros_like(counts)
    P = f64(p_sum) / float(n_tokens)
    return float(alpha * E * np.dot(f, P))


def z_loss(lse, lam):
    """Router z-loss lambda * mean_t (logsumexp_e s_{t,e})^2.

    [8MOE] ST-MoE router z-loss; [STA324] §8.6 (batch mean of the squared
    log-sum-exp).
    """
    return float(lam * np.mean(f64(lse) ** 2))


# ---------------------------------------------------------------------------
# Full layer
# ---------------------------------------------------------------------------
@dataclass
class Layer:
    """Inputs of one layer as arrays / on-demand expert weights."""
    x: np.ndarray                   # [T, D]
    w_r: np.ndarray                 # [E, D]
    w13: Callable[[int], np.ndarray]   # e -> [2F, D]
    wd: Callable[[int], np.ndarray]    # e -> [D, F]
    w13_s: Optional[np.ndarray] = None  # [2F, D] shared expert
    wd_s: Optional[np.ndarray] = None   # [D, F]
    logit_offset: Optional[np.ndarray] = None
    sel_bias: Optional[np.ndarray] = None
    sentinel_mask: Optional[np.ndarray] = None


@dataclass
class Opts:
    K: int
    score_fn: int = SOFTMAX
    renorm: int = 1
    n_groups: int = 1
    topk_groups: int = 1
    group_score: int = GROUP_MAX
    capacity_factor: float = 0.0
    min_capacity: int = 0
    route_scale: float = 1.0
    aux_alpha: float = 0.0
    z_lambda: float = 0.0
    seq_len: int = 0             # > 0: the aux loss is sequence-wise (oracle/balance.py)
    logits_fp32: bool = True     # False only for finite-difference checks


def opts_of(cfg) -> Opts:
    """Opts from any object carrying the layer option fields."""
    return Opts(K=cfg.K, score_fn=cfg.score_fn, renorm=cfg.renorm,
                n_groups=cfg.n_groups, topk_groups=cfg.topk_groups,
                group_score=cfg.group_score,
                capacity_factor=cfg.capacity_factor,
                min_capacity=cfg.min_capacity, route_scale=cfg.route_scale,
                aux_alpha=cfg.aux_alpha, z_lambda=cfg.z_lambda,
                seq_len=getattr(cfg, "seq_len", 0))


def route_layer(L: Layer, o: Opts, idx_given=None) -> Routing:
    s = router_logits(L.x, L.w_r, L.logit_offset, o.logits_fp32)
    return route(s, o.K, score_fn=o.score_fn, renorm=o.renorm,
                 n_groups=o.n_groups, topk_groups=o.topk_groups,
                 group_score=o.group_score, route_scale=o.route_scale,
                 sel_bias=L.sel_bias, idx_given=idx_given)


def forward(L: Layer, o: Opts, idx_given=None):
    """y_t = sum_{k kept} g_{t,k} E_{idx_k}(x_t) (+ shared(x_t)), plus losses.

    [8MOE] Router / Gating Network: y = sum_i G(x)_i E_i(x); [STA324] §8.8:
    a token appears K times, so outputs accumulate; §8.7: the shared expert
    runs on every token, unweighted, and takes no top-K slot.
    Returns a dict with routing, dispatch, per-slot SwiGLU values and y.
    idx_given (tests only): see route().
    """
    return forward_routed(L, o, route_layer(L, o, idx_given))


def forward_routed(L: Layer, o: Opts, R: Routing):
    """forward() from a given routing (token choice, or the slot form of
    expert choice in oracle/expert_choice.py)."""
    x = f64(L.x)
    T, D = x.shape
    E = L.w_r.shape[0]
    Dp = dispatch(R.idx, E, o.capacity_factor, o.min_capacity,
                  L.sentinel_mask)
    K = o.K
    slot_o = {}
    slot_act = {}
    for e in range(E):
        slots = np.nonzero(Dp.expert == e)[0]
        slots = slots[Dp.rank[slots] >= 0]
        if slots.size == 0:
            continue
        slots = slots[np.argsort(Dp.rank[slots])]
        toks = slots // K
        a, b, h, oo = swiglu_forward(x[toks], L.w13(e), L.wd(e))
        slot_act[e] = (slots, toks, a, b, h, oo)
    y = np.zeros((T, D))
    gflat = R.g.reshape(-1)
    o_slot = np.zeros((T * K, D))
    for e, (slots, toks, a, b, h, oo) in slot_act.items():
        o_slot[slots] = oo
    for k in range(K):
        j = np.arange(T) * K + k
        kept = Dp.rank[j] >= 0
        y[kept] += gflat[j[kept], None] * o_slot[j[kept]]
    shared = None
    if L.w13_s is not None:
        shared = swiglu_forward(x, L.w13_s, L.wd_s)
        y += shared[3]
    if o.aux_alpha and o.seq_len:
        laux, f, P = balance.seq_aux_loss(R.p, Dp.expert, K, o.aux_alpha, o.seq_len, o.score_fn)
    elif o.aux_alpha:
        laux, f, P = aux_loss(Dp.counts, R.p, o.aux_alpha, E)
    else:
        laux, f, P = 0.0, None, None
    lz = z_loss(R.lse, o.z_lambda) if o.z_lambda else 0.0
    return dict(R=R, Dp=Dp, slot_act=slot_act, o_slot=o_slot, y=y,
                shared=shared, aux=laux, z=lz, f=f, P=P)


def gate_grad(o_slot, dy, Dp: Dispatch, K, sentinel_unmasked=None):
    """dL/dg_{t,k} = <proj_out_{t,k}, dy_t>, zero on sentinel / dropped slots.

    [HF48687] cause analysis: the gradient of the sample weight is the expert
    output proj_out, so slots with no local expert must have proj_out zeroed
    (as grouped_mm does) or they leak gradient into the router.
    `sentinel_unmasked` (tests only) is the negative control: a [T*K, D]
    array of expert-0 outputs used for sentinel slots, i.e. the batched_mm
    behaviour that clamps the id and does not zero proj_out.
    """
    T = dy.shape[0]
    dyr = np.repeat(f64(dy), K, axis=0)            # [T*K, D], row j = dy_{j//K}
    dg = np.einsum("jd,jd->j", o_slot, dyr)
    dg[Dp.rank < 0] = 0.0
    if sentinel_unmasked is not None:
        sj = Dp.sentinel
        dg[sj] = np.einsum("jd,jd->j", sentinel_unmasked[sj], dyr[sj])
    return dg.reshape(T, K)


def router_backward(R: Routing, dg, o: Opts, counts=None, T_total=None, seq_f=None):
    """dL/dlogits from the gate path, the aux loss and the z-loss.

    Gate path ([STA324] §8.3: with the selected set fixed, g is differentiable
    in the logits; [MM858] §2 root cause):
      A softmax: dp_{idx_k} += route_scale * dg_k, then through p = softmax(s)
      B softmax: g = softmax over the selected logits, so
                 ds_sel = gn * (dgn - <gn, dgn>) with gn = g/route_scale,
                 dgn = route_scale*dg; for K=1 gn = 1 and ds is exactly 0
      B sigmoid: g_k = rs*p_k/S, S = sum_sel p + eps:
                 dp_k = rs/S * (dg_k - sum_j dg_j g_j / rs), ds = dp p (1-p)
      A sigmoid: dp_k = rs * dg_k, ds = dp p (1-p)
    Aux ([STA324] §8.5): dL/dp_{t,e} = alpha E f_e / T, f held constant;
    sequence-wise aux (o.seq_len > 0, per-sequence f in seq_f): see
    oracle/balance.py.
    z ([8MOE] ST-MoE): dL/ds_{t,e} = 2 lambda lse_t softmax(s_t)_e / T.
    The hot-spot offset and the selection bias receive no gradient.
    """
    s = f64(R.logits)
    T, E = s.shape
    Tn = T if T_total is None else T_total
    K = R.idx.shape[1]
    rs = o.route_scale
    dg = f64(dg)
    ds = np.zeros((T, E))
    rows = np.arange(T)[:, None]
    valid = R.idx >= 0
    idx = np.where(valid, R.idx, 0)
    dgv = np.where(valid, dg, 0.0)
    if o.score_fn == SOFTMAX:
        p = R.p
        dp = np.zeros((T, E))
        if not o.renorm:
            np.add.at(dp, (np.repeat(rows, K, axis=1), idx), rs * dgv)
        if o.aux_alpha and o.seq_len:
            dp += balance.seq_aux_grad_scores(p, seq_f, o.aux_alpha, o.seq_len, SOFTMAX)
        elif o.aux_alpha:
            cnt = f64(counts)
            f = cnt / cnt.sum() if cnt.sum() > 0 else np.zeros(E)
            dp += o.aux_alpha * E * f[None, :] / Tn
        ds += p * (dp - (p * dp).sum(axis=1, keepdims=True))
        if o.renorm:
            gn = R.g / rs
            dgn = rs * dgv
            inner = (gn * dgn).sum(axis=1, keepdims=True)
            np.add.at(ds, (np.repeat(rows, K, axis=1), idx),
                      np.where(valid, gn * (dgn - inner), 0.0))
    else:
        sel = np.take_along_axis(R.p, idx, axis=1)
        if o.renorm:
            S = sel.sum(axis=1, keepdims=True) + SIGMOID_EPS
            inner = (dgv * R.g).sum(axis=1, keepdims=True) / rs
            dpk = rs / S * (dgv - inner)
        else:
            dpk = rs * dgv
        dsk = np.where(valid, dpk * sel * (1.0 - sel), 0.0)
        np.add.at(ds, (np.repeat(rows, K, axis=1), idx), dsk)
        if o.aux_alpha and o.seq_len:
            ds += balance.seq_aux_grad_scores(R.p, seq_f, o.aux_alpha, o.seq_len, SIGMOID)
        elif o.aux_alpha:
            raise ValueError("the batch aux loss is defined for softmax scores only")
    if o.z_lambda:
        ds += 2.0 * o.z_lambda * R.lse[:, None] * softmax_rows(s) / Tn
    return ds


def backward(L: Layer, o: Opts, fw, dy, sentinel_unmasked=None):
    """All gradients of <y, dy> + L_aux + L_z.

    Returns dx [T,D], dw_r [E,D], dw13 {e: [2F,D]}, dwd {e: [D,F]},
    dw13_s, dwd_s, dg [T,K], ds [T,E].
    """
    x = f64(L.x)
    dy = f64(dy)
    T, D = x.shape
    E = L.w_r.shape[0]
    K = o.K
    R, Dp = fw["R"], fw["Dp"]
    dg = gate_grad(fw["o_slot"], dy, Dp, K, sentinel_unmasked)
    gflat = R.g.reshape(-1)
    dx = np.zeros((T, D))
    dw13, dwd = {}, {}
    for e in range(E):
        if e not in fw["slot_act"]:
            w13 = L.w13(e)
            dw13[e] = np.zeros(w13.shape)
            dwd[e] = np.zeros(L.wd(e).shape)
            continue
        slots, toks, a, b, h, oo = fw["slot_act"][e]
        do = gflat[slots, None] * dy[toks]
        dxr, dw13[e], dwd[e] = swiglu_backward(x[toks], a, b, h, do,
                                               L.w13(e), L.wd(e))
        np.add.at(dx, toks, dxr)
    dw13_s = dwd_s = None
    if fw["shared"] is not None:
        a, b, h, _ = fw["shared"]
        dxs, dw13_s, dwd_s = swiglu_backward(x, a, b, h, dy, L.w13_s, L.wd_s)
        dx += dxs
    ds = router_backward(R, dg, o, Dp.counts, seq_f=fw["f"] if o.seq_len else None)
    dw_r = ds.T @ x
    dx += ds @ f64(L.w_r)
    return dict(dx=dx, dw_r=dw_r, dw13=dw13, dwd=dwd, dw13_s=dw13_s,
                dwd_s=dwd_s, dg=dg, ds=ds)


# ---------------------------------------------------------------------------
# Per-token / per-column pieces for sampled checks of full-size layers
# ---------------------------------------------------------------------------
def token_slots(Dp: Dispatch, t, K):
    """(k, expert) of token t's kept slots, in k order."""
    out = []
    for k in range(K):
        j = t * K + k
        if Dp.rank[j] >= 0:
            out.append((k, int(Dp.expert[j])))
    return out


def token_forward_backward(L: Layer, o: Opts, R: Routing, Dp: Dispatch, t,
                           dy_t, counts_total_T=None):
    """y_t, dg_t, ds_t and dx_t of one token (exact; needs only its experts).

    The aux term of ds uses the global counts (Dp.counts) and T.
    """
    x_t = f64(L.x[t:t + 1])
    dy_t = f64(dy_t).reshape(1, -1)
    K = o.K
    T = L.x.shape[0]
    y = np.zeros((1, x_t.shape[1]))
    dg = np.zeros(K)
    dx = np.zeros_like(x_t)
    g = R.g[t]
    for k, e in token_slots(Dp, t, K):
        w13, wd = L.w13(e), L.wd(e)
        a, b, h, oo = swiglu_forward(x_t, w13, wd)
        y += g[k] * oo
        dg[k] = float((oo * dy_t).sum())
        dxr, _, _ = swiglu_backward(x_t, a, b, h, g[k] * dy_t, w13, wd)
        dx += dxr
    if L.w13_s is not None:
        a, b, h, oo = swiglu_forward(x_t, L.w13_s, L.wd_s)
        y += oo
        dxr, _, _ = swiglu_backward(x_t, a, b, h, dy_t, L.w13_s, L.wd_s)
        dx += dxr
    Rt = Routing(logits=R.logits[t:t + 1], p=R.p[t:t + 1], lse=R.lse[t:t + 1],
                 idx=R.idx[t:t + 1], g=R.g[t:t + 1], margin=R.margin[t:t + 1])
    ds = router_backward(Rt, dg[None, :], o, Dp.counts, T_total=T)[0]
    dx += ds[None, :] @ f64(L.w_r)
    return dict(y=y[0], dg=dg, ds=ds, dx=dx[0])


def tokens_forward_backward(L: Layer, o: Opts, R: Routing, Dp: Dispatch, toks,
                            dy_toks):
    """y, dg, ds and dx of the tokens `toks` (exact), as token_forward_backward
    on each of them, but expert by expert: every expert's weights are fetched
    once for all the sampled slots it serves (full-size layers regenerate
    them on demand).  Returns arrays with one row per entry of `toks`.
    """
    toks = np.asarray(toks, dtype=np.int64)
    n = toks.size
    K = o.K
    T = L.x.shape[0]
    xt = f64(L.x[toks])
    dyt = f64(dy_toks).reshape(n, -1)
    D = xt.shape[1]
    y = np.zeros((n, D))
    dg = np.zeros((n, K))
    dx = np.zeros((n, D))
    by_e = {}
    for i, t in enumerate(toks):
        for k, e in token_slots(Dp, int(t), K):
            by_e.setdefault(e, []).append((i, k))
    # per token, its slots' terms are added in k order
    contrib = {}
    for e in sorted(by_e):
        ik = np.array(by_e[e])
        ii, kk = ik[:, 0], ik[:, 1]
        w13, wd = L.w13(e), L.wd(e)
        a, b, h, oo = swiglu_forward(xt[ii], w13, wd)
        g = R.g[toks[ii], kk]
        dg[ii, kk] = (oo * dyt[ii]).sum(axis=1)
        dxr, _, _ = swiglu_backward(xt[ii], a, b, h, g[:, None] * dyt[ii], w13, wd)
        for r in range(ii.size):
            contrib[(int(ii[r]), int(kk[r]))] = (g[r] * oo[r], dxr[r])
    for (i, k) in sorted(contrib):
        y[i] += contrib[(i, k)][0]
        dx[i] += contrib[(i, k)][1]
    if L.w13_s is not None:
        a, b, h, oo = swiglu_forward(xt, L.w13_s, L.wd_s)
        y += oo
        dxr, _, _ = swiglu_backward(xt, a, b, h, dyt, L.w13_s, L.wd_s)
        dx += dxr
    Rt = Routing(logits=R.logits[toks], p=R.p[toks], lse=R.lse[toks],
                 idx=R.idx[toks], g=R.g[toks], margin=R.margin[toks])
    ds = router_backward(Rt, dg, o, Dp.counts, T_total=T)
    dx += ds @ f64(L.w_r)
    return dict(y=y, dg=dg, ds=ds, dx=dx)


def expert_column_grads(L: Layer, o: Opts, R: Routing, Dp: Dispatch, e, j,
                        dy_rows):
    """dW13[e][j,:], dW13[e][F+j,:] and dW_down[e][:,j] from the expert's rows.

    dy_rows(tokens) -> [n, D] upstream gradient rows.  Needs only rows j and
    F+j of W13[e] and column j of W_down[e] (passed by the callables
    w13_rows(e, rows) / wd_col(e, j) when present on L, else sliced).
    j may be a list of columns: each result then has one row per column.
    """
    js = np.atleast_1d(np.asarray(j, dtype=np.int64))
    K = o.K
    slots = np.nonzero((Dp.expert == e) & (Dp.rank >= 0))[0]
    slots = slots[np.argsort(Dp.rank[slots])]
    toks = slots // K
    if hasattr(L, "w13_rows"):
        F = L.F
        wg = f64(L.w13_rows(e, np.concatenate([js, F + js])))
        wdj = np.stack([f64(L.wd_col(e, int(c))) for c in js], axis=1)   # [D, n_j]
    else:
        w13 = f64(L.w13(e))
        F = w13.shape[0] // 2
        wg = w13[np.concatenate([js, F + js])]
        wdj = f64(L.wd(e))[:, js]
    D = wg.shape[1]
    nj = js.size
    if slots.size == 0:
        z = np.zeros((nj, D))
        out = (z, z.copy(), z.copy())
    else:
        xr = f64(L.x[toks])
        a = xr @ wg[:nj].T                     # [rows, n_j]
        b = xr @ wg[nj:].T
        do = R.g.reshape(-1)[slots, None] * f64(dy_rows(toks))
        dh = do @ wdj
        sa = 1.0 / (1.0 + np.exp(-a))
        da = dh * b * sa * (1.0 + a * (1.0 - sa))
        db = dh * silu(a)
        h = silu(a) * b
        out = (da.T @ xr, db.T @ xr, (do.T @ h).T)
    if np.ndim(j) == 0:
        return tuple(v[0] for v in out)
    return out
