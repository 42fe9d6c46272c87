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
