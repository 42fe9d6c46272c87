"""Properties of the library's step that the pages fix, on the GPU.

* The worked example ("Ch 06 · Muon", §5 "完整算法", box "具体例子 · 抹平
  shape 依赖"): after Newton-Schulz ||O'||_F = sqrt(min(n, m)), and scaling
  by sqrt(max(n, m)) brings a 1024 x 1024 and a 256 x 4096 layer to the same
  ||O||_F = 1024 (gamma = 1). The composed quintics end in [1.0000, 1.0020]
  on well-conditioned inputs ("Muon 优化器完全拆解…", section "小结"), so
  ||O'||_F / sqrt(min) lies in [1, 1.0021]: checked in fp32, and within the
  2e-2 parity bound around it in bf16.
* NaN and Inf are not checked and propagate as in the plain definition: a
  NaN in one gradient element makes that element of M NaN, the norm NaN and
  so every element of that matrix's W NaN, and leaves the other matrices
  alone.
"""

import math

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _step(wl, precision, **hyper):
    import muon_step_b200 as ms

    plan = ms.MuonPlan([(wl.W[k], wl.G[k], wl.M[k]) for k in range(wl.count)], precision=precision)
    plan.execute(**hyper)
    torch.cuda.synchronize()
    assert ms.sync_status() == 0


@pytest.mark.parametrize("precision,band", [("fp32", (1.0, 1.0021)),
                                            ("bf16", (1.0 - 2e-2, 1.0021 + 2e-2))])
def test_worked_example(precision, band):
    shapes = [(1024, 1024), (256, 4096), (4096, 256)]
    wl = workloads.make_random(shapes, device="cuda", seed=41, spectrum="flat")
    for k in range(wl.count):
        wl.W[k].zero_()
        wl.M[k].zero_()
    # momentum 0 gives N = G; lr 1, no decay, gamma 1: W = -sqrt(max(n, m)) O'
    _step(wl, precision, lr=1.0, momentum=0.0, weight_decay=0.0, gamma=1.0)
    for (n, m), W in zip(shapes, wl.W):
        fro = float(W.double().norm())
        o_ratio = fro / math.sqrt(max(n, m)) / math.sqrt(min(n, m))
        assert band[0] <= o_ratio <= band[1], (precision, n, m, o_ratio)
        assert 1024.0 * band[0] <= fro <= 1024.0 * band[1], (precision, n, m, fro)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_nan_in_one_gradient_propagates_to_that_matrix_only(precision):
    # grouped path (300 x 520), one-CTA paths (64 x 64, 100 x 300)
    shapes = [(300, 520), (64, 64), (100, 300), (300, 520)]
    wl = workloads.make_random(shapes, device="cuda", seed=42)
    for k in (0, 1, 2):
        wl.G[k][7, 11] = float("nan")
    _step(wl, precision, lr=0.02, momentum=0.95, weight_decay=0.1, gamma=0.2)
    for k in (0, 1, 2):
        M = wl.M[k]
        assert torch.isnan(M[7, 11])
        mask = torch.ones_like(M, dtype=torch.bool)
        mask[7, 11] = False
        assert torch.isfinite(M[mask]).all()
        assert torch.isnan(wl.W[k]).all()
    assert torch.isfinite(wl.W[3]).all() and torch.isfinite(wl.M[3]).all()
