"""Benchmark of the token-choice MoE layer step (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config mix]
                    [--impl reference]

One step = the whole hot path over one batch: router, dispatch, aux/z loss,
grouped SwiGLU experts, combine, and the full backward (gate-weight
gradient, expert dgrad/wgrad, router gradient, dx).  The default workload
is the largest of the five layer shapes, the Mixtral-shaped layer (T=32768,
D=4096, E=8, K=2, F=14336, bf16, variant B, capacity factor 1.25 with +2.0
on expert 0's logit, so the hot expert overflows and drops).  Multi-GPU
(torchrun): data-parallel replicas,
each rank runs its own batch (weak scaling, no data-path collective);
timing is the max over ranks.

Rank 0 prints one JSON line.  `value` is tokens/s from CUDA events around
CUDA-graph replays of the step with inputs resident in HBM (L2 flushed
between steps); `e2e` is the same metric through the Python API with the
step's inputs copied from pinned host memory and y, dx read back; the
roofline entry times the dominant kernel's launches with CUDA events on its
launching stream inside the timed region.  `--impl reference` times the
CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "MoE layer fwd+bwd tokens/s at 1 B200; grouped-GEMM % bf16 peak; HBM GB/s"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
SHAPE_NAMES = {"tiny": "tiny fp32", "mm": "MiniMind-shaped", "olmoe": "OLMoE-shaped",
               "mix": "Mixtral-shaped", "ds3": "DeepSeek-V3-shaped"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="mix", choices=sorted(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--gather", type=int, default=0, choices=[0, 1],
                    help="1: the gate/up GEMMs' producer warp copies token rows of x "
                         "(cp.async; no permuted copy of x); 0: the dispatch writes x_perm")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="sequence-wise aux loss over groups of this many tokens")
    ap.add_argument("--aux-alpha", type=float, default=None)
    ap.add_argument("--bias-gamma", type=float, default=0.0,
                    help="selection-bias update step after each forward (sigmoid routing)")
    ap.add_argument("--timeline", action="store_true",
                    help="print one profiled step's launch timeline to stderr")
    ap.add_argument("--cpu-sample-s", type=float, default=10.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the config's token count (small cases for profiling)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the config's expert count (small cases for profiling)")
    ap.add_argument("--only", default="", choices=["", "router"],
                    help="router: time moe_router alone on the config's shape (one JSON line, "
                         "GB/s of the router kernel; for profiling captures)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_init(n_gpus, backend="nccl"):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t[0])


def rank_config(cfg: W.LayerConfig, rank: int) -> W.LayerConfig:
    """Each data-parallel rank draws its own tokens (weights are shared)."""
    return cfg if rank == 0 else cfg.replace(seed=cfg.seed + 1000 * rank)


# ---------------------------------------------------------------------------
# work accounting (algorithmic, per step)
# ---------------------------------------------------------------------------
def expert_rows(cfg, kept_total):
    return kept_total + (cfg.T if cfg.n_shared else 0)


def gemm_flops(cfg, kept_total):
    """Algorithmic FLOPs of each tensor-core GEMM family for one step."""
    M = expert_rows(cfg, kept_total)
    D, F = cfg.D, cfg.F
    return {
        "tc_gate_up_swiglu": 2 * M * D * 2 * F,
        "tc_down": 2 * M * F * D,
        "tc_dgrad_down_swiglu_bwd": 2 * M * D * F,
        "tc_wgrad_down": 2 * M * D * F,
        "tc_dgrad_gate_up": 2 * M * 2 * F * D,
        "tc_wgrad_gate_up": 2 * M * 2 * F * D,
        # one slot per token: combine / unpermute-sum in the epilogue
        "tc_down_combine": 2 * M * F * D,
        "tc_dgrad_gate_up_dx": 2 * M * 2 * F * D,
    }


def gemm_bytes(cfg, kept_total):
    """Algorithmic DRAM bytes of each expert GEMM for one step: operands,
    the fused epilogue's extra input (a13 in the SwiGLU backward) and its
    outputs, each read or written once."""
    a = 2 if cfg.dtype == "bf16" else 4
    M = expert_rows(cfg, kept_total)
    D, F, E = cfg.D, cfg.F, cfg.E + (1 if cfg.n_shared else 0)
    w13, wd = E * 2 * F * D * a, E * D * F * a
    return {
        "tc_gate_up_swiglu": M * D * a + w13 + M * 3 * F * a,
        "tc_down": M * F * a + wd + M * D * a,
        "tc_dgrad_down_swiglu_bwd": M * D * a + wd + 2 * M * 2 * F * a,
        "tc_dgrad_gate_up": M * 2 * F * a + w13 + M * D * a,
        "tc_wgrad_down": M * D * a + M * F * a + wd,
        "tc_wgrad_gate_up": M * 2 * F * a + M * D * a + w13,
        # + y rows and gate weights / dx rows written in token order from the
        # fp32 accumulator, ds and W_r read (no dX_perm round trip)
        "tc_down_combine": M * F * a + wd + M * D * a + cfg.T * D * a + cfg.T * 4,
        "tc_dgrad_gate_up_dx": (M * 2 * F * a + w13 + cfg.T * D * a + cfg.T * cfg.E * 4
                                + cfg.E * D * 4),
    }


def hbm_bytes(cfg, kept_total, rows_used):
    """Algorithmic DRAM bytes of each memory-bound kernel for one step: every
    distinct operand element read once (a token row gathered K times counts
    once) and every result written once (activations in the layer dtype,
    router tensors fp32)."""
    a = 2 if cfg.dtype == "bf16" else 4
    T, D, E, K = cfg.T, cfg.D, cfg.E, cfg.K
    M = expert_rows(cfg, kept_total)
    router = T * D * a + E * D * 4 + 2 * T * E * 4 + T * 4 + T * K * 8
    return {
        "router_fused": router, "router_tc": router, "router_logits": T * D * a + E * D * 4 + T * E * 4,
        "router_route": 3 * T * E * 4 + T * 4 + T * K * 8,
        "dispatch_gather": T * D * a + rows_used * D * a,
        "combine": M * D * a + T * D * a + T * K * 8,
        "bwd_gate_grad_rows": M * D * a + T * D * a + rows_used * D * a + T * K * 8,
        "dx_unpermute_router": M * D * a + T * D * a + T * E * 4 + E * D * 4,
        "dx_unpermute_sum": M * D * a + T * D * 4 + T * D * a,
    }


def source_hash(files=None):
    """Hash of the kernel sources (all of csrc/, or the named files)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "mixture_experts_routing_fp32_b200", "csrc")
    for n in sorted(files or os.listdir(d)):
        with open(os.path.join(d, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j.get("hbm_gbs", 6545.0), j.get("bf16_tflops", 1652.8), \
            j.get("bf16_tflops_sustained", 1386.2), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def recorded_traffic(kernel, workload, tokens, experts):
    """DRAM bytes per launch from a committed ncu summary, if it was captured
    on this workload's shape and the files that define that kernel still
    hash to what they were then (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != source_hash(e.get("files")):
        return None
    if e.get("T", tokens) != tokens or e.get("E", experts) != experts:
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5], f[6], f[7], f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        load = [r for r in rows if r[0] > 0.5 * r[1]] or rows
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for n, v in zip(names, r[2:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in load),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args):
    from mixture_experts_routing_fp32_b200 import (MoELayer, config_from, moe_check_status,
                                                   moe_launch_count, moe_set_side_streams)
    from mixture_experts_routing_fp32_b200.api import LaunchProfile
    from mixture_experts_routing_fp32_b200.build import build

    rank, world, local = dist_init(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        build()
    barrier(world)
    base = W.CONFIGS[args.config]
    if args.tokens:
        base = base.replace(T=args.tokens)
    if args.experts:
        base = base.replace(E=args.experts)
    if args.seq_len:
        base = base.replace(seq_len=args.seq_len)
    if args.aux_alpha is not None:
        base = base.replace(aux_alpha=args.aux_alpha)
    cfg = rank_config(base, rank)
    names = ("x", "w_r", "w13", "w_down", "dy")
    inp = {n: W.make_input(cfg if n in ("x", "dy") else base, n, dev) for n in names}
    opt = {
        "w13_s": W.make_input(base, "w13_s", dev) if base.n_shared else None,
        "w_down_s": W.make_input(base, "w_down_s", dev) if base.n_shared else None,
        "logit_offset": W.make_input(base, "logit_offset", dev) if base.hot_expert_offset else None,
        "sel_bias": W.make_input(base, "sel_bias", dev) if base.sel_bias_range else None,
        "sentinel_mask": W.make_input(cfg, "sentinel_mask", dev) if base.sentinel_frac else None,
    }
    layer = MoELayer(config_from(base), device=dev, gather=bool(args.gather))
    weights = dict(w_r=inp["w_r"], w13=inp["w13"], w_down=inp["w_down"], **opt)
    x, dy = inp["x"], inp["dy"]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.forward(x, **weights)
        if args.bias_gamma and weights.get("sel_bias") is not None:
            layer.update_bias(weights["sel_bias"], args.bias_gamma)
        layer.backward(dy)

    # warm-up (eager), then capture one step in a CUDA graph with per-launch events
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    moe_check_status()
    moe_launch_count(reset=True)
    step()
    torch.cuda.synchronize(dev)
    launches_per_step = moe_launch_count(reset=True)

    # e2e through the public API, pipelined over steps: every step copies its
    # inputs in from pinned host memory (copy-in stream), computes (the
    # caller's stream, after an L2 flush: the layer's forward + backward
    # calls, captured once per input buffer set into a CUDA graph), and
    # copies y and dx out to pinned host memory (copy-out stream); step i's
    # copy-in overlaps step i-1's compute and its copy-out overlaps step
    # i+1's.  Timed from the first copy-in to the last copy-out, divided by
    # the number of steps.
    NB = 2
    hx = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    hdy = torch.empty(dy.shape, dtype=dy.dtype, pin_memory=True)
    hx.copy_(x)
    hdy.copy_(dy)
    din = [(torch.empty_like(x), torch.empty_like(dy)) for _ in range(NB)]
    dout = [(torch.empty_like(layer.y), torch.empty_like(x)) for _ in range(NB)]
    hout = [(torch.empty(layer.y.shape, dtype=layer.y.dtype, pin_memory=True),
             torch.empty(x.shape, dtype=x.dtype, pin_memory=True)) for _ in range(NB)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    e2e_flush = torch.empty(192 << 20, dtype=torch.uint8, device=dev)
    h2d = hx.numel() * hx.element_size() + hdy.numel() * hdy.element_size()
    d2h = sum(t.numel() * t.element_size() for t in hout[0])

    def e2e_compute(b):
        layer.forward(din[b][0], **weights)
        if args.bias_gamma and weights.get("sel_bias") is not None:
            layer.update_bias(weights["sel_bias"], args.bias_gamma)
        layer.backward(din[b][1])
        dout[b][0].copy_(layer.y)
        dout[b][1].copy_(layer.dx)

    def capture_fn(fn):
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                fn()
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        return g

    for b in range(NB):                 # inputs for the eager warm-up and capture
        din[b][0].copy_(x)
        din[b][1].copy_(dy)
        e2e_compute(b)
    torch.cuda.synchronize(dev)
    e2e_graphs = None if args.no_graph else [capture_fn(lambda b=b: e2e_compute(b))
                                             for b in range(NB)]

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_comp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n):
            b = i % NB
            with torch.cuda.stream(s_in):
                if i >= NB:
                    s_in.wait_event(ev_comp[i - NB])     # step i-NB no longer reads din[b]
                din[b][0].copy_(hx, non_blocking=True)
                din[b][1].copy_(hdy, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= NB:
                stream.wait_event(ev_out[i - NB])        # dout[b] copied out
            e2e_flush.fill_(i & 0xFF)
            if e2e_graphs is not None:
                e2e_graphs[b].replay()
            else:
                e2e_compute(b)
            ev_comp[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                hout[b][0].copy_(dout[b][0], non_blocking=True)
                hout[b][1].copy_(dout[b][1], non_blocking=True)
                ev_out[i].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1) / n

    e2e_run(3)
    e2e = max_over_ranks(e2e_run(args.steps), world, dev)
    moe_check_status()
    assert torch.equal(hout[(args.steps - 1) % NB][1].to(dev), layer.dx)


    def capture():
        return capture_fn(step)

    # `value` comes from a graph with no measurement nodes in it; the
    # per-launch timing comes from a second graph captured with the
    # library's begin/end events around every launch and with the side
    # streams folded into the caller's stream, so that every launch has the
    # GPU to itself while it is timed; it is replayed in its own loop below.
    graph = None if args.no_graph else capture()
    prof = LaunchProfile(128)
    prof.reset()
    moe_set_side_streams(False)
    layer.side_streams = False
    graph_prof = None if args.no_graph else capture()
    if graph is not None:
        moe_set_side_streams(True)
        layer.side_streams = True

    def replay(g):
        if g is not None:
            g.replay()
        else:
            prof.reset()
            step()

    for g in (graph, graph_prof):
        for _ in range(max(args.warmup, 3)):
            flush.fill_(1)
            replay(g)
    torch.cuda.synchronize(dev)
    moe_check_status()

    kept_total = int(layer.kept.sum())
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    per_launch = []
    prof_ok = True
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit() else local
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_index) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)          # L2 flush between timed steps (untimed)
            ev0[i].record(stream)
            replay(graph)
            ev1[i].record(stream)
        barrier(world)
        torch.cuda.synchronize(dev)
        # per-launch durations: the profiled graph, same flushes
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            replay(graph_prof)
            torch.cuda.synchronize(dev)
            if prof_ok:
                try:
                    per_launch.append(prof.read())
                except Exception:
                    prof_ok = False
    if args.timeline and rank == 0:
        flush.fill_(7)
        replay(graph_prof)
        torch.cuda.synchronize(dev)
        for (name, t, on_side), t0 in zip(prof.read(), prof.starts()):
            print("%9.2f us  %8.2f us  %s%s" % (t0 * 1e3, t * 1e3, name,
                                                 " [side]" if on_side else ""),
                  file=sys.stderr)
    step_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    ms = statistics.mean(step_ms)
    timing_src = ("begin/end events around each launch inside replays of the step graph "
                  "captured with the backward's side streams folded into the caller's stream "
                  "(each launch has the GPU to itself)")
    if not prof_ok or not per_launch or not per_launch[0]:
        # events recorded by graph nodes unreadable: time the same launches
        # eagerly (L2 flushed between steps) in a separate pass
        timing_src = "separate eager pass"
        per_launch = []
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            prof.reset()
            step()
            torch.cuda.synchronize(dev)
            per_launch.append(prof.read())
    ms_max = max_over_ranks(ms, world, dev)
    moe_check_status()

    # per-kernel totals per step (side-stream launches, if any were timed
    # concurrently, are marked: their event times include GPU sharing)
    fam, side = {}, set()
    for launches in per_launch:
        for name, t, on_side in launches:
            fam.setdefault(name, []).append(t)
            if on_side:
                side.add(name)
    tot = {k: sum(v) / len(per_launch) for k, v in fam.items()}
    hbm, bf16, bf16_sus, peak_src = measured_peaks()
    clocks = clk.summary()
    # tensor peak: the sustained figure when the power cap engaged during the
    # timed region (the GPU ran long enough to settle at its capped clock),
    # else the burst figure (each launch is timed on its own at full clock)
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    tc_peak = bf16_sus if capped else bf16
    tc_kind = ("sustained: sw_power_cap was active during the timed region" if capped else
               "burst: no power cap during the timed region, each launch timed alone")
    flops = gemm_flops(base, kept_total)
    rows_used = int(layer.stats[2])
    hbm_b = hbm_bytes(base, kept_total, rows_used)
    # dominant kernel: the largest share of the step among launches timed alone
    main = {k: v for k, v in tot.items() if k not in side} or tot
    dom = max(main, key=main.get)
    n_dom = len(fam[dom]) / len(per_launch)
    dom_ms = statistics.mean(fam[dom])
    gbytes = gemm_bytes(base, kept_total)
    if dom in flops:
        # a fused GEMM is bound by the slower of its tensor work and its
        # DRAM traffic at the measured peaks; report against that bound
        t_tensor = flops[dom] / (tc_peak * 1e12)
        t_hbm = gbytes[dom] / (hbm * 1e9)
        if t_tensor >= t_hbm:
            achieved = flops[dom] / n_dom / (dom_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": round(achieved, 2),
                    "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": round(achieved / tc_peak, 4),
                    "peak_source": "%s bf16 dense, %s" % (peak_src, tc_kind)}
        else:
            achieved = gbytes[dom] / n_dom / (dom_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4),
                    "peak_source": "%s copy bandwidth (the kernel's DRAM traffic outweighs its "
                                   "tensor work at the measured peaks)" % peak_src}
        roof["tensor_TFLOPs"] = round(flops[dom] / n_dom / (dom_ms * 1e-3) / 1e12, 2)
        roof["algorithmic_bytes"] = gbytes[dom] // int(max(1, n_dom))
        roof["algorithmic_flops"] = flops[dom] // int(max(1, n_dom))
    else:
        gbs = hbm_b[dom] / n_dom / (dom_ms * 1e-3) / 1e9 if dom in hbm_b else None
        roof = {"bound": "hbm", "achieved": round(gbs, 1) if gbs else None, "peak": hbm,
                "unit": "GB/s", "frac": round(gbs / hbm, 4) if gbs else None,
                "peak_source": "%s copy bandwidth" % peak_src}
    roof.update({"kernel": dom, "launch_ms": round(dom_ms, 5), "timing": timing_src,
                 "launches_per_step": n_dom,
                 "traffic": recorded_traffic(dom, base.name, base.T, base.E)})
    gemm_names = sorted(k for k in flops if k in tot)
    gemm_total_ms = sum(tot[k] for k in gemm_names)
    gemm_tflops = (sum(flops[k] for k in gemm_names) / (gemm_total_ms * 1e-3) / 1e12
                   if gemm_total_ms else None)

    # memory-bound kernels: algorithmic bytes / launch time vs HBM peak
    hbm_table = {}
    for k, b in hbm_b.items():
        if k in tot and tot[k] > 0:
            gbs = b / (tot[k] * 1e-3) / 1e9
            hbm_table[k] = {"bytes": b, "ms": round(tot[k], 5), "GB/s": round(gbs, 1),
                            "frac_of_hbm": round(gbs / hbm, 4),
                            "side_stream": k in side}
    cpu = cpu_baseline(base, args.cpu_sample_s) if (rank == 0 and world == 1 and not args.no_cpu) else None
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(base.T * world / (ms_max * 1e-3), 1),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_max, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if base.dtype == "bf16" else "f32",
            "data": "synthetic (seeded counter-hash normals, bf16-rounded; shapes of the %s "
                    "layer)" % SHAPE_NAMES.get(base.name.split("_")[0], base.name),
            "config": {"workload": "%s: T=%d D=%d E=%d K=%d F=%d %s variant %s aux %.0e%s%s" % (
                base.name, base.T, base.D, base.E, base.K, base.F, base.dtype,
                "B" if base.renorm else "A", base.aux_alpha,
                " sequence-wise over %d tokens" % base.seq_len if base.seq_len else "",
                " bias update gamma %g" % args.bias_gamma if args.bias_gamma else ""),
                "global_batch_tokens": base.T * world, "parallelism": "dp%d (replicas)" % world,
                "l2": "flushed between timed steps (256 MiB write)",
                "cuda_graph": graph is not None,
                "row_gather": ("inside the gate/up GEMMs (producer-warp cp.async copies of "
                               "x rows)" if args.gather else "dispatch kernel writes x_perm"),
                "programmatic_dependent_launch": os.environ.get("MOE_PDL", "1") != "0"},
            "e2e": {"value": round(base.T * world / (e2e * 1e-3), 1), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e, 4),
                    "path": "Python API (MoELayer.forward/backward) captured once per input "
                            "buffer set into a CUDA graph; pinned-host copies pipelined over "
                            "steps (copy-in of step i and copy-out of step i-1 overlap "
                            "compute); L2 flushed (192 MiB write) before each step's compute"},
            "gpu_launches": launches_per_step * args.steps,
            "roofline": roof,
            "expert_gemms": {
                "per_kernel": {k: {"ms": round(tot[k], 5),
                                   "TFLOP/s": round(flops[k] / (tot[k] * 1e-3) / 1e12, 1),
                                   "frac_of_tensor": round(flops[k] / (tot[k] * 1e-3) / 1e12
                                                           / tc_peak, 3),
                                   "GB/s": round(gbytes[k] / (tot[k] * 1e-3) / 1e9, 1),
                                   "frac_of_hbm": round(gbytes[k] / (tot[k] * 1e-3) / 1e9 / hbm,
                                                        3)}
                               for k in gemm_names},
                "tflops": round(gemm_tflops, 2) if gemm_tflops else None,
                "frac_of_sustained": round(gemm_tflops / bf16_sus, 4) if gemm_tflops else None,
                "frac_of_burst": round(gemm_tflops / bf16, 4) if gemm_tflops else None,
                "frac_of_peak": round(gemm_tflops / tc_peak, 4) if gemm_tflops else None,
                "peak": tc_peak, "peak_kind": tc_kind,
                "ms_per_step": round(gemm_total_ms, 5), "kernels": gemm_names,
                "timing": "sum of the expert GEMM launches timed one by one"},
            "kernels_ms_per_step": {k + (" [side stream]" if k in side else ""): round(v, 5)
                                    for k, v in sorted(tot.items(), key=lambda kv: -kv[1])},
            "hbm_kernels": hbm_table,
            "kept_rows": kept_total,
            "routing": {"near_ties": int(layer.near_ties[0]), "n_drop": int(layer.stats[0]),
                        "n_sentinel": int(layer.stats[1]),
                        "capacity": int(layer.sizes.capacity),
                        "expert_counts": [int(v) for v in layer.counts.cpu()],
                        "note": "near_ties: tokens whose selection margin among the top K+1 "
                                "fp32 scores is below 1e-5 (the GPU's count); n_drop: "
                                "assignments beyond capacity"},
            "clocks": clocks,
            "cpu_baseline": cpu,
            "source_hash": source_hash(),
        }
        print(json.dumps(line), flush=True)
    prof.close()
    graph = graph_prof = e2e_graphs = None
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# the CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------
CPU_SAMPLE_FLOP = 0.3e12          # expert FLOPs of one oracle sample step (seconds)
CPU_WEIGHT_BYTES = 16 << 30       # host bytes of the sample's expert weights


def cpu_sample_tokens(cfg):
    """Tokens of one CPU-oracle sample: a power of two up to 512 whose expert
    work (18*D*F FLOPs per kept slot, shared expert included) stays under
    CPU_SAMPLE_FLOP, so one sample takes seconds on the host cores."""
    per_tok = 18.0 * cfg.D * cfg.F * (cfg.K + cfg.n_shared)
    T_s = 512
    while T_s > 16 and T_s * per_tok > CPU_SAMPLE_FLOP:
        T_s //= 2
    return min(cfg.T, T_s)


class OracleSample:
    """The oracle's inputs for the first T_s tokens of cfg, built before any
    clock starts.  Only the experts those tokens route to are materialised,
    held as float32 (the bf16 weights exactly; the oracle widens what it is
    given to float64 as its first step); if they would exceed
    CPU_WEIGHT_BYTES the sample shrinks until they fit."""

    def __init__(self, cfg, T_s):
        import numpy as np
        from oracle import moe_oracle as O
        f32 = lambda t: t.float().numpy()
        while True:
            x = f32(W.make_input(cfg, "x", rows=np.arange(T_s)))
            w_r = f32(W.make_input(cfg, "w_r"))
            self.L = O.Layer(x=x, w_r=w_r, w13=self._w13, wd=self._wd)
            if cfg.n_shared:
                self.L.w13_s, self.L.wd_s = f32(W.make_input(cfg, "w13_s")), \
                    f32(W.make_input(cfg, "w_down_s"))
            if cfg.hot_expert_offset:
                self.L.logit_offset = f32(W.make_input(cfg, "logit_offset"))
            if cfg.sel_bias_range:
                self.L.sel_bias = f32(W.make_input(cfg, "sel_bias"))
            if cfg.expert_choice:
                hit = range(cfg.E)
            else:
                sub = cfg.replace(T=T_s)
                R = O.route_layer(self.L, O.opts_of(sub))
                hit = sorted(set(int(e) for e in R.idx.reshape(-1)))
            per_e = 3 * cfg.D * cfg.F * 4
            if len(hit) * per_e <= CPU_WEIGHT_BYTES or T_s <= 8:
                break
            T_s //= 2
        self.T_s, self.hit = T_s, list(hit)
        self.w13 = {e: f32(W.make_input(cfg, "w13", expert=e)) for e in hit}
        self.wd = {e: f32(W.make_input(cfg, "w_down", expert=e)) for e in hit}
        self.dy = f32(W.make_input(cfg, "dy", rows=np.arange(T_s)))
        self.cfg = cfg

    def _w13(self, e):
        return self.w13[e]

    def _wd(self, e):
        return self.wd[e]

    def describe(self):
        return ("first %d of %d tokens, full forward+backward in the float64 numpy oracle "
                "(%d of %d experts routed to, their weights materialised before timing)"
                % (self.T_s, self.cfg.T, len(self.hit), self.cfg.E))

    def step(self):
        """One forward + backward of the oracle on the sample; seconds."""
        from oracle import moe_oracle as O
        cfg = self.cfg
        t0 = time.perf_counter()
        if cfg.expert_choice:
            # expert choice picks across the batch: the sample is its own batch
            # (each expert picks ceil(c * T_s / E) of its tokens)
            from oracle import expert_choice as X
            Lc, o, fw = X.forward(self.L, cfg.capacity_factor, cfg.min_capacity,
                                  z_lambda=cfg.z_lambda)
            O.backward(Lc, o, fw, self.dy)
        else:
            o = O.opts_of(cfg.replace(T=self.T_s))
            fw = O.forward(self.L, o)
            O.backward(self.L, o, fw, self.dy)
        return time.perf_counter() - t0


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(cfg, budget_s):
    smp = OracleSample(cfg, cpu_sample_tokens(cfg))
    times = []
    t_end = time.perf_counter() + budget_s
    while True:
        times.append(smp.step())
        if time.perf_counter() > t_end or len(times) >= 20:
            break
    s = statistics.mean(times)
    return {"value": round(smp.T_s / s, 2), "unit": UNIT, "cores": cpu_threads(),
            "kind": "oracle",
            "sample": "%s, mean of %d runs (%.2f s each)" % (smp.describe(), len(times), s)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = W.CONFIGS[args.config]
    smp = OracleSample(cfg, cpu_sample_tokens(cfg))
    for _ in range(args.warmup):
        smp.step()
    times = [smp.step() for _ in range(args.steps)]
    s = statistics.mean(times)
    v = round(smp.T_s / s, 2)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "%s (oracle on the first %d tokens per step)" % (cfg.name,
                                                                                 smp.T_s)},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": smp.describe() + " per step"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_router_only(args):
    """moe_router alone on the config's shape: L2 flushed before each call,
    CUDA-event time of each library launch (LaunchProfile)."""
    from mixture_experts_routing_fp32_b200 import api, config_from, moe_check_status
    from mixture_experts_routing_fp32_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    base = W.CONFIGS[args.config]
    if args.tokens:
        base = base.replace(T=args.tokens)
    if args.experts:
        base = base.replace(E=args.experts)
    cfg = config_from(base)
    T, E, K = base.T, base.E, base.K
    x = W.make_input(base, "x", dev)
    w_r = W.make_input(base, "w_r", dev)
    off = W.make_input(base, "logit_offset", dev) if base.hot_expert_offset else None
    bias = W.make_input(base, "sel_bias", dev) if base.sel_bias_range else None
    f32 = dict(dtype=torch.float32, device=dev)
    logits, probs = torch.empty(T, E, **f32), torch.empty(T, E, **f32)
    lse, w = torch.empty(T, **f32), torch.empty(T, K, **f32)
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    ties = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(api.moe_get_sizes(cfg).ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    prof = api.LaunchProfile(16)
    per = {}
    for i in range(max(args.warmup, 3) + args.steps):
        flush.fill_(i & 255)
        prof.reset()
        api.moe_router(cfg, x, w_r, off, bias, logits, probs, lse, idx, w, ties, ws)
        torch.cuda.synchronize(dev)
        if i >= max(args.warmup, 3):
            for n, ms, _ in prof.read():
                per.setdefault(n, []).append(ms)
    moe_check_status()
    med = {n: sorted(v)[len(v) // 2] for n, v in per.items()}
    a = 2 if base.dtype == "bf16" else 4
    nbytes = T * base.D * a + E * base.D * 4 + 2 * T * E * 4 + T * 4 + T * K * 8
    kern = "router_tc" if "router_tc" in med else max(med, key=med.get)
    hbm, _, _, src = measured_peaks()
    gbs = nbytes / (med[kern] * 1e-3) / 1e9
    print(json.dumps({
        "metric": "router kernel GB/s (algorithmic bytes / CUDA-event time, L2 flushed)",
        "value": round(gbs, 1), "unit": "GB/s", "kernel": kern,
        "frac_of_hbm": round(gbs / hbm, 4), "peak_source": src, "bytes": nbytes,
        "kernels_ms": {n: round(v, 5) for n, v in med.items()}, "steps": args.steps,
        "config": {"workload": "%s: T=%d D=%d E=%d K=%d" % (base.name, T, base.D, E, K)},
        "near_ties": int(ties.item())}))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.only == "router":
        run_router_only(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
