"""The seeded input generator: identical values on every path and slice."""
import numpy as np
import torch

import workloads as W
from workloads import gen


def test_c_and_torch_paths_bit_identical():
    shape = (3, 1000, 77)
    a = gen.normal(shape, 0, 3, 0.02, use_c=True)
    b = gen.normal(shape, 0, 3, 0.02, use_c=False)
    assert torch.equal(a, b)
    # indices beyond 2**32 (DeepSeek-V3-sized expert weights)
    idx = torch.tensor([0, 7, 2**32 + 1, 2**33 + 99, 3 * 2**31 - 1])
    assert torch.equal(gen.normal_at((3, 2**31), idx, 0, 3, 0.02),
                       gen._normal_torch(idx, 0, 3, 0.02, "cpu"))


def test_slices_match_full_tensor():
    cfg = W.CONFIGS["olmoe"].replace(T=300, D=64, E=6, F=32)
    x = W.make_input(cfg, "x")
    rows = torch.tensor([299, 0, 17])
    assert torch.equal(W.make_input(cfg, "x", rows=rows), x[rows])
    w = W.make_input(cfg, "w13")
    assert torch.equal(W.make_input(cfg, "w13", expert=4), w[4])
    assert x.dtype == torch.bfloat16 and W.make_input(cfg, "w_r").dtype == torch.float32


def test_distributions_and_recipe():
    cfg = W.CONFIGS["olmoe"]
    x = W.make_input(cfg.replace(T=2048), "x").float()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    w = W.make_input(cfg, "w_r")
    assert abs(w.std() - 0.02) < 0.001
    m = W.make_input(cfg, "sentinel_mask")
    assert int(m.sum()) == round(0.1 * cfg.T * cfg.K) == 13107
    b = W.make_input(W.CONFIGS["ds3"], "sel_bias")
    assert b.abs().max() < 0.1
    off = W.make_input(W.CONFIGS["mix"], "logit_offset")
    assert off[0] == 2.0 and torch.all(off[1:] == 0)
