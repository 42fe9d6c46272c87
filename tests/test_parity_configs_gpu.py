"""Parity on the full-size workloads, in the launch configuration the
benchmark times (one grouped plan over every matrix of the workload).

Sampled matrices are compared with the float64 oracle where it finishes in
about a minute. On the two largest sweep bases (8192 and 16384) one oracle
step on a whole matrix takes minutes to hours, so those points run with
inputs of the form P blockdiag(B_1 .. B_k) Q (random row and column
permutations, full-rank blocks of 512 rows): every Newton-Schulz step
multiplies by a polynomial in X X^T ("Ch 06 · Muon" §3), so the exact
iteration acts block by block under the whole matrix's normalisation and
leaves zeros off the blocks. Every element of O' is then compared with the
oracle, at full size, in the launch configuration the benchmark times.
"""

import math

import numpy as np
import pytest
import torch

import workloads
from tests.parity import TOL_ELEMENTWISE, TOL_O, blockwise_oracle, check_step, rel

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _check(wl, sample):
    worst = check_step(wl, "bf16", sample=sample)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE and worst["W_given_O"] <= TOL_ELEMENTWISE, worst
    return worst


def test_dense_d4096_sampled():
    """16-layer d = 4096 stack, 112 matrices; one Q, one gate and one down
    (14336 x 4096, the transposed path) checked."""
    wl = workloads.make("dense_d4096", device="cuda")
    _check(wl, sample=[0, 4, 7 * 9 + 6])
    del wl
    _free()


def test_moe_64x3_sampled():
    """64-expert bank, 192 matrices with expert scales over three decades."""
    wl = workloads.make("moe_64x3", device="cuda")
    _check(wl, sample=[0, 2, 3 * 40 + 1, 3 * 63 + 2])
    del wl
    _free()


SMALL_SWEEP = [(b, a) for b in (128, 512, 2048) for a in ("1x1", "1x4", "4x1")]
LARGE_SWEEP = [(b, a) for b in (8192, 16384) for a in ("1x1", "1x4", "4x1")]


@pytest.mark.parametrize("base,aspect", SMALL_SWEEP)
def test_sweep_sampled(base, aspect):
    wl = workloads.make(f"sweep_{base}_{aspect}", device="cuda")
    _check(wl, sample=[0, wl.count - 1])
    del wl
    _free()


@pytest.mark.parametrize("base,aspect", LARGE_SWEEP)
def test_sweep_large_blockwise(base, aspect):
    """The two largest sweep bases at full size (the sweep point's batch, one
    grouped plan, as the benchmark launches it), with G and M_prev of the form
    P blockdiag(B_1 .. B_k) Q: O' compared element by element with the float64
    oracle's blockwise iteration (relative Frobenius error per matrix <= 2e-2),
    exact zeros off the blocks, and the momentum and the update (given the
    library's O') <= 1e-6, for every matrix of the batch."""
    import muon_step_b200 as ms

    wl, supports = workloads.make_sweep_blocks(base, aspect, device="cuda")
    h = wl.hyper
    M0 = [m.clone() for m in wl.M]
    W0 = [w.clone() for w in wl.W]
    O = [torch.empty_like(w) for w in wl.W]
    plan = ms.MuonPlan([(wl.W[i], wl.G[i], wl.M[i], O[i]) for i in range(wl.count)])
    plan.execute(lr=h["lr"], momentum=h["mu"], weight_decay=h["wd"], gamma=h["gamma"],
                 nesterov=h["nesterov"])
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    n, m = wl.shapes[0]
    c = max(n, m)
    worst = 0.0
    for i in range(wl.count):
        # momentum and the update given the library's O', elementwise in float64
        M_ref = h["mu"] * M0[i].double() + wl.G[i].double()
        assert (torch.linalg.norm(wl.M[i].double() - M_ref) / torch.linalg.norm(M_ref)).item() \
            <= TOL_ELEMENTWISE
        del M_ref
        W_ref = W0[i].double() * (1 - h["lr"] * h["wd"]) - h["lr"] * h["gamma"] * math.sqrt(c) * O[i].double()
        assert (torch.linalg.norm(wl.W[i].double() - W_ref) / torch.linalg.norm(W_ref)).item() \
            <= TOL_ELEMENTWISE
        del W_ref
        # exact zeros off the blocks
        rows, cols = supports[i]
        Z = O[i].clone()
        Z[rows[:, :, None], cols[:, None, :]] = 0.0
        assert torch.count_nonzero(Z).item() == 0, (i, torch.count_nonzero(Z).item())
        del Z
        # the blocks against the oracle
        idx = (rows[:, :, None], cols[:, None, :])
        ref = blockwise_oracle(wl.G[i][idx].double().cpu().numpy(),
                               M0[i][idx].double().cpu().numpy(), h)
        got = O[i][idx].double().cpu().numpy()
        err = rel(got, ref)
        worst = max(worst, err)
        assert err <= TOL_O["bf16"], (i, err)
    print(f"sweep {base} {aspect}: {wl.count} matrices, worst O' error {worst:.3e}")
    del wl, plan, O, M0, W0
    _free()
