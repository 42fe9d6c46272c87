"""The benchmark's FLOP count against the FLOP formula and figures printed on
"Muon 优化器完全拆解…", section "收益与代价" (tests/golden/flop_overhead.txt)."""

import os

import pytest

import bench
from tests.conftest import read_golden


def test_metric_flops_is_the_printed_formula():
    # one step on an n x m matrix with m <= n costs 2 (2 n m^2 + m^3); the
    # benchmark counts 10 steps, with r = min and c = max
    for n, m in [(1024, 1024), (4096, 14336), (14336, 4096), (256, 512), (7, 3)]:
        r, c = min(n, m), max(n, m)
        assert bench.metric_flops([(n, m)], ns_steps=1) == 2 * (2 * c * r * r + r ** 3)
        assert bench.metric_flops([(n, m)]) == 10 * bench.metric_flops([(n, m)], ns_steps=1)
        # "at most 6 n m^2 for a square matrix"
        assert bench.metric_flops([(n, m)], ns_steps=1) <= 6 * c * r * r


def test_printed_overhead_figures(golden_dir):
    rows = read_golden(os.path.join(golden_dir, "flop_overhead.txt"))
    for label, T, m, B, pct in rows:
        T, m, B, pct = int(T), int(m), int(B), float(pct)
        # overhead relative to forward + backward (6 n m B) for a square layer
        n = m
        overhead = T * bench.metric_flops([(n, m)], ns_steps=1) / (6.0 * n * m * B)
        assert overhead == pytest.approx(T * m / B)
        assert round(100 * overhead, 1) == pct, label


def _plan_flops(shapes, prec):
    import ctypes

    from muon_step_b200 import _lib
    from muon_step_b200._lib import MUON_OK, MuonParam

    lib = _lib.load()
    arr = (MuonParam * len(shapes))(*[MuonParam(0x10000, 0x20000, 0x30000, None, n, m)
                                      for n, m in shapes])
    plan = ctypes.c_void_p()
    assert lib.muon_plan_create(arr, len(shapes), prec, None, ctypes.byref(plan)) == MUON_OK
    g, p, a = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    assert lib.muon_plan_flops(plan, ctypes.byref(g), ctypes.byref(p), ctypes.byref(a)) == MUON_OK
    cnt = ctypes.c_int()
    kinds = (ctypes.c_int * 128)()
    assert lib.muon_plan_launches(plan, ctypes.byref(cnt), kinds, 128) == MUON_OK
    lib.muon_plan_destroy(plan)
    return (g.value, p.value, a.value), set(kinds[:cnt.value])


@pytest.mark.parametrize("prec,precision", [(0, "bf16"), (1, "fp32")])
def test_executed_stage_flops_match_the_planner(prec, precision):
    """The roofline's per-launch FLOPs of each grouped stage equal the
    planner's own count of the tiles it runs (one execute = 10 launches)."""
    shapes = [(4096, 4096), (4096, 14336), (14336, 4096), (1000, 300), (257, 1029), (2048, 7168)]
    (g, p, a), _ = _plan_flops(shapes, prec)
    for kind, total in ((1, g), (2, p), (3, a)):
        assert 10 * bench.executed_stage_flops(kind, shapes, precision) == pytest.approx(total, rel=1e-12)
    assert bench.executed_stage_flops(4, shapes, precision) == bench.executed_stage_flops(3, shapes, precision)
    if precision == "bf16":
        # the symmetric stages skip the upper blocks: about half of the dense product
        for r, c in [(4096, 14336), (2048, 2048)]:
            ratio = bench.executed_stage_flops(1, [(r, c)]) / (2.0 * r * r * c)
            assert 0.5 < ratio < 0.55


def test_one_cta_kinds_follow_the_planner():
    for shape in [(1, 1), (64, 64), (1, 4096), (65, 64), (128, 128), (129, 64), (128, 512),
                  (1, 4097), (129, 129), (300, 400)]:
        _, kinds = _plan_flops([shape], 0)
        want = bench.one_cta_kind(*shape)
        if want is None:
            assert kinds == {0, 10, 4} and not kinds & {5, 8, 9}, shape
        else:
            assert kinds == {0, want}, shape
        _, kinds32 = _plan_flops([shape], 1)
        assert bench.one_cta_kind(*shape, precision="fp32") is None and not kinds32 & {5, 8, 9}


def test_dominant_roofline_picks_the_longest_kernel_and_its_bound():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    shapes = [(4096, 14336)] * 2
    # Apply launches take the most time: tensor-bound at r = 4096 (about r / 4 flop per byte)
    per = {0: [1.0], 1: [0.5] * 10, 2: [0.2] * 10, 3: [1.0] * 9, 4: [1.2]}
    roof = bench.dominant_roofline([], per, shapes, peaks)
    assert roof["kind"] == 3 and roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    flops = 2 * 2.0 * 4096 * 4096 * 14336
    assert roof["achieved"] == pytest.approx(flops / 1e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1400.0)
    # the elementwise kernel dominating: HBM-bound at 16 bytes per element
    per = {0: [5.0], 3: [0.1] * 9}
    roof = bench.dominant_roofline([], per, shapes, peaks)
    assert roof["kind"] == 0 and roof["bound"] == "hbm"
    assert roof["achieved"] == pytest.approx(16.0 * 2 * 4096 * 14336 / 5e-3 / 1e9)
    # the small-matrix kernel on 128 x 128 matrices: all ten steps on chip, so
    # 60 r^3 FLOPs per 12 r^2 bytes put it on the tensor side of the ridge
    per = {0: [0.1], 5: [2.0]}
    roof = bench.dominant_roofline([], per, [(128, 128)] * 1000, peaks)
    assert roof["kind"] == 5 and roof["bound"] == "tensor"
    assert roof["bytes_per_launch"] == 12.0 * 128 * 128 * 1000
    assert roof["flops_per_launch"] == 1000 * 10 * 6.0 * 128 ** 3
