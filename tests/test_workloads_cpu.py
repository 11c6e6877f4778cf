"""The seeded input recipe (CPU): every machine draws the same tensors, in the
stated order and rounding, and the FLOP counts the benchmark reports follow
the stated formulas.  The module that holds the recipe does no attention
arithmetic; these checks restate the recipe, not the method."""

import math

import numpy as np
import torch

from exact_io_aware_49_b200 import workloads as wl


def test_five_workloads_and_their_shapes():
    got = [(w.B, w.H, w.N, w.d, w.causal, w.p_drop, w.seed) for w in wl.WORKLOADS]
    assert got == [(1, 1, 128, 64, False, 0.0, 0), (2, 8, 1024, 64, True, 0.0, 1), (4, 16, 4096, 128, True, 0.1, 2),
                   (2, 32, 16384, 64, True, 0.0, 3), (1, 32, 32768, 128, True, 0.1, 4)]
    assert [w.qk_std for w in wl.WORKLOADS] == [1.0, 1.0, 1.0, 4.0, 1.0]
    assert set(wl.BY_NAME) == {w.name for w in wl.WORKLOADS}


def test_draw_order_rounding_and_determinism():
    w = wl.Workload("t", 2, 3, 40, 64, True, 0.0, 17)
    q, k, v, do = wl.draw_inputs(w)
    g = torch.Generator(device="cpu").manual_seed(17)
    ref = [torch.randn((2, 3, 40, 64), generator=g, dtype=torch.float32) for _ in range(4)]
    for got, want in zip((q, k, v, do), ref):
        assert got.dtype == torch.bfloat16 and tuple(got.shape) == (2, 3, 40, 64)
        assert torch.equal(got, want.to(torch.bfloat16))  # round-to-nearest-even of the fp32 draw
    again = wl.draw_inputs(w)
    assert all(torch.equal(a, b) for a, b in zip((q, k, v, do), again))
    f16 = wl.draw_inputs(w, dtype=torch.float16)
    assert all(x.dtype == torch.float16 for x in f16)
    assert torch.equal(f16[2], ref[2].to(torch.float16))


def test_wide_logit_scaling_touches_only_q_and_k():
    base = wl.Workload("a", 1, 2, 64, 64, True, 0.0, 5)
    wide = wl.Workload("b", 1, 2, 64, 64, True, 0.0, 5, qk_std=4.0)
    x, y = wl.draw_inputs(base), wl.draw_inputs(wide)
    g = torch.Generator(device="cpu").manual_seed(5)
    ref = [torch.randn((1, 2, 64, 64), generator=g, dtype=torch.float32) for _ in range(4)]
    assert torch.equal(y[0], (ref[0] * 4.0).to(torch.bfloat16))
    assert torch.equal(y[1], (ref[1] * 4.0).to(torch.bfloat16))
    assert torch.equal(x[2], y[2]) and torch.equal(x[3], y[3])


def test_reduced_draws_use_the_same_recipe():
    w = wl.BY_NAME["causal_dropout_N32768_d128"]
    q = wl.draw_inputs(w, B=1, H=1, N=8)[0]
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    assert torch.equal(q, torch.randn((1, 1, 8, 128), generator=g, dtype=torch.float32).to(torch.bfloat16))


def test_sampled_rows_are_seeded_distinct_and_sorted():
    w = wl.BY_NAME["causal_dropout_N32768_d128"]
    rows = wl.sample_rows(w, B=1, H=3, N=5000)
    assert len(rows) == 1 and len(rows[0]) == 3
    for idx in rows[0]:
        a = idx.numpy()
        assert len(a) == 256 and len(np.unique(a)) == 256
        assert (np.diff(a) > 0).all() and a.min() >= 0 and a.max() < 5000
    again = wl.sample_rows(w, B=1, H=3, N=5000)
    assert all(torch.equal(a, b) for a, b in zip(rows[0], again[0]))
    assert not torch.equal(rows[0][0], rows[0][1])  # each head draws its own rows


def test_flop_counts():
    w = wl.BY_NAME["causal_dropout_N32768_d128"]
    assert math.isclose(w.fwd_flops(), 4 * 32 * 32768 ** 2 * 128 / 2)
    assert math.isclose(w.bwd_flops(), 2.5 * w.fwd_flops())
    nc = wl.BY_NAME["single_tile_N128_d64"]
    assert math.isclose(nc.fwd_flops(), 4 * 128 ** 2 * 64)
    assert math.isclose(w.scale, 128 ** -0.5)
