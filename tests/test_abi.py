"""The C-ABI library: builds, loads, exports every declared symbol, and
validates configurations on the host (no CUDA calls, no GPU needed)."""
from __future__ import annotations

import ctypes
import math
import os
import re

import pytest

from mixture_experts_routing_fp32_b200 import _lib as C
from mixture_experts_routing_fp32_b200 import api
from mixture_experts_routing_fp32_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return C.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|int64_t|const char\*)\s+(moe_\w+)\s*\(",
                                 src, flags=re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(C.EXPORTS) == names


def test_config_struct_layout_matches_header():
    # 12 int32 fields, then float, int32, 3 floats, 6 int32 = 23 x 4 bytes
    assert ctypes.sizeof(C.MoeConfig) == 23 * 4
    assert ctypes.sizeof(C.MoeSizes) == 40


def _rows_max(T, K, E, C_, n_shared, align):
    kept_total = T * K if C_ is None else min(T * K, E * C_)
    pad = (align - 1) * min(E, kept_total)
    r = -(-(kept_total + pad) // align) * align
    return r + (-(-T // align) * align if n_shared else 0)


@pytest.mark.parametrize("T,D,E,K,F,c,ns", [
    (4096, 768, 4, 1, 2048, 0.0, 0),
    (32768, 4096, 8, 2, 14336, 1.25, 0),
    (8192, 7168, 256, 8, 2048, 0.0, 1),
    (256, 64, 4, 2, 64, 1.1, 0),
])
def test_sizes(lib, T, D, E, K, F, c, ns):
    cfg = api.make_config(T, D, E, K, F, capacity_factor=c, n_shared=ns,
                          score_fn=1 if ns else 0)
    s = api.moe_get_sizes(cfg)
    Cap = None if c <= 0 else max(math.ceil(c * T * K / E), 0)
    assert s.capacity == (-1 if Cap is None else Cap)
    align = 256 if (K * T if Cap is None else min(K * T, E * Cap)) // E >= 1536 else 128
    assert s.row_align == align
    assert s.rows_max == _rows_max(T, K, E, Cap, ns, align)
    assert s.tiles_max * 128 == s.rows_max
    assert s.ws_bytes > 0
    if T == 256:
        assert s.capacity == 141        # the course page's lab: ceil(1.1*256*2/4)


@pytest.mark.parametrize("bad", [
    dict(K=5),                        # K > E
    dict(K=17, E=32),                 # K > 16
    dict(D=30),                       # D % 8
    dict(E=513, K=2),                 # E > 512
    dict(n_groups=3),                 # E % n_groups
    dict(n_groups=2, topk_groups=1, K=3),   # topk_groups * E/n_groups < K
    dict(aux_alpha=0.01, score_fn=1),       # batch aux needs softmax scores
    dict(seq_len=48),                 # seq_len must divide T
    dict(seq_len=-1),
    dict(expert_choice=1),            # expert choice needs K = E and a capacity
    dict(expert_choice=1, K=4, capacity_factor=1.0, renorm=1),   # ... and variant A
    dict(expert_choice=1, K=4, capacity_factor=1.0, renorm=0, aux_alpha=0.01),
    dict(dtype="fp16"),               # maps to fp32 -> still valid; replaced below
    dict(loss_tokens=32),             # global loss token count below T
    dict(loss_tokens=-1),
    dict(loss_tokens=128, seq_len=32),    # global scope is for the batch losses only
])
def test_invalid_configs_rejected(lib, bad):
    kw = dict(T=64, D=32, E=4, K=2, F=64)
    kw.update(bad)
    if kw.get("dtype") == "fp16":
        cfg = api.make_config(**{k: v for k, v in kw.items() if k != "dtype"})
        cfg.dtype = 7
    else:
        cfg = api.make_config(**kw)
    out = C.MoeSizes()
    assert lib.moe_get_sizes(ctypes.byref(cfg), ctypes.byref(out)) == C.MOE_ERR_ARG


def test_null_pointers_rejected_before_any_launch(lib):
    cfg = api.make_config(64, 32, 4, 2, 64, dtype="fp32")
    args = [None] * 12
    assert lib.moe_router(ctypes.byref(cfg), *args) == C.MOE_ERR_ARG
    assert lib.moe_dispatch(ctypes.byref(cfg), *([None] * 13)) == C.MOE_ERR_ARG
    assert lib.moe_backward(ctypes.byref(cfg), *([None] * 33)) == C.MOE_ERR_ARG
    assert lib.moe_status_string(C.MOE_ERR_ARG).startswith(b"invalid")
    with pytest.raises(C.MoEError):
        C.check(C.MOE_ERR_ARG, "x")


def test_fused_paths_rejected_where_unsupported(lib):
    """The gathered expert FFN and a NULL x_perm in the backward exist only on
    the tensor-core path: fp32 layers are refused on the host, before any
    pointer is used (the dummy addresses below are never dereferenced)."""
    cfg = api.make_config(64, 32, 4, 2, 64, dtype="fp32")
    dummy = ctypes.c_void_p(256)
    assert lib.moe_expert_ffn_gather(ctypes.byref(cfg), *([dummy] * 13), None) == C.MOE_ERR_ARG
    args = [dummy] * 33
    args[14] = None                      # x_perm
    args[-1] = None                      # stream
    assert lib.moe_backward(ctypes.byref(cfg), *args) == C.MOE_ERR_ARG
    # fused FFN + combine: y is required; with x_perm NULL also x and the
    # tensor-core path
    bf = api.make_config(4096, 768, 4, 1, 2048)
    a = [dummy] * 18
    a[15] = None                         # y
    a[17] = None                         # stream
    assert lib.moe_expert_ffn_combine(ctypes.byref(bf), *a) == C.MOE_ERR_ARG
    a = [dummy] * 18
    a[1] = None                          # x_perm
    a[17] = None
    assert lib.moe_expert_ffn_combine(ctypes.byref(cfg), *a) == C.MOE_ERR_ARG


def test_misaligned_x_or_router_weight_rejected_before_any_launch(lib):
    """x and W_r are read with 16-byte vector loads: a pointer off that
    boundary is refused on the host (the dummy addresses are never
    dereferenced)."""
    cfg = api.make_config(64, 32, 4, 2, 64, dtype="fp32")
    ok, off = ctypes.c_void_p(256), ctypes.c_void_p(260)
    for i in (0, 1):                     # x, w_r
        args = [ok] * 12
        args[i] = off
        args[-1] = None                  # stream
        assert lib.moe_router(ctypes.byref(cfg), *args) == C.MOE_ERR_ARG
        args = [ok] * 33
        args[i] = off
        args[-1] = None
        assert lib.moe_backward(ctypes.byref(cfg), *args) == C.MOE_ERR_ARG


def test_package_has_no_cpu_fallback():
    # the product path never imports the oracle
    pkg = os.path.join(ROOT, "mixture_experts_routing_fp32_b200")
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            src = open(os.path.join(pkg, name)).read()
            assert "oracle" not in src.replace("never imports the oracle", ""), name


def test_global_loss_entry_points_validate_on_host(lib):
    """moe_aux_stats / moe_aux_loss_global refuse NULL buffers and the
    sequence-wise configuration before any launch; a loss token count of at
    least T is accepted."""
    ok = api.make_config(64, 32, 4, 2, 64, dtype="fp32", aux_alpha=0.01, loss_tokens=256)
    out = C.MoeSizes()
    assert lib.moe_get_sizes(ctypes.byref(ok), ctypes.byref(out)) == C.MOE_OK
    assert lib.moe_aux_stats(ctypes.byref(ok), None, None, None, None, None) == C.MOE_ERR_ARG
    assert lib.moe_aux_loss_global(ctypes.byref(ok), None, None, None, None) == C.MOE_ERR_ARG
    seq = api.make_config(64, 32, 4, 2, 64, dtype="fp32", aux_alpha=0.01, seq_len=32)
    dummy = ctypes.c_void_p(256)
    assert lib.moe_aux_stats(ctypes.byref(seq), dummy, dummy, dummy, dummy, None) == C.MOE_ERR_ARG
    assert lib.moe_set_backward_streams(None) == C.MOE_OK


def test_shard_configs_refused_on_the_host(lib):
    """Shards need the tensor-core path, token choice, no shared expert and
    a range inside [0, E); refused before any launch."""
    L = lib
    out = C.MoeSizes()
    ok = api.make_config(256, 128, 8, 2, 128, expert_base=4, n_local_experts=4)
    assert L.moe_get_sizes(ctypes.byref(ok), ctypes.byref(out)) == C.MOE_OK
    for bad in (dict(expert_base=6, n_local_experts=4), dict(expert_base=2),
                dict(n_local_experts=4, n_shared=1), dict(n_local_experts=4, dtype="fp32"),
                dict(n_local_experts=4, D=96)):
        kw = dict(T=256, D=128, E=8, K=2, F=128)
        kw.update(bad)
        c = api.make_config(**kw)
        assert L.moe_get_sizes(ctypes.byref(c), ctypes.byref(out)) == C.MOE_ERR_ARG, bad
