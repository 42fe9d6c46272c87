"""Helpers shared by the GPU parity tests: run the library on a workload and
compare every (or a sampled) matrix with the float64 oracle."""

from __future__ import annotations

import math

import numpy as np
import torch

from oracle import muon_oracle

# tolerances (relative Frobenius error per matrix)
TOL_O = {"bf16": 2e-2, "fp32": 1e-4}   # O' against the oracle
TOL_ELEMENTWISE = 1e-6                  # momentum, and the update given the GPU's own O'

# Matrices with fewer elements than this are too small for the bf16 rounding
# of the iterate operand to average out over the Frobenius norm: a CPU
# emulation of the kernels' rounding (bf16 X, A, B; fp32 master iterate) on
# 12,000 random Gaussian matrices of 2 to 64 elements reached 3.8e-2; with the
# split bf16 high + low iterate, 3.0e-2 on 12,600 such matrices.
TINY_ELEMENTS = 256
TOL_O_TINY_BF16 = 5e-2


def tol_o(precision, shape):
    n, m = shape
    if precision == "bf16" and n * m < TINY_ELEMENTS:
        return TOL_O_TINY_BF16
    return TOL_O[precision]


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    if nb == 0.0:
        return float(np.linalg.norm(a))
    return float(np.linalg.norm(a - b) / nb)


def run_step(wl, precision="bf16", hyper=None, schedule=None, sample=None, steps=1,
             scale_mode="shape"):
    """Snapshot the sampled inputs, run `steps` Muon steps through the library
    (plan API) capturing O', and return per-sample records."""
    import muon_step_b200 as ms

    hyper = dict(wl.hyper if hyper is None else hyper)
    idx = list(range(wl.count)) if sample is None else list(sample)
    before = {k: (wl.W[k].double().cpu().numpy(), wl.G[k].double().cpu().numpy(),
                  wl.M[k].double().cpu().numpy()) for k in idx}
    O = {k: torch.empty_like(wl.W[k]) for k in idx}
    params = [(wl.W[k], wl.G[k], wl.M[k], O.get(k)) for k in range(wl.count)]
    plan = ms.MuonPlan(params, precision=precision, schedule=schedule, scale_mode=scale_mode)
    ws = plan.alloc_workspace()
    history = []
    for _ in range(steps):
        plan.execute(ws, lr=hyper["lr"], momentum=hyper["mu"], weight_decay=hyper["wd"],
                     gamma=hyper["gamma"], nesterov=hyper["nesterov"])
        history.append({k: O[k].double().cpu().numpy() for k in idx})
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    after = {k: (wl.W[k].double().cpu().numpy(), wl.M[k].double().cpu().numpy()) for k in idx}
    return before, after, history, hyper


def check_step(wl, precision="bf16", hyper=None, schedule=None, sample=None, steps=1,
               scale_mode="shape"):
    """Compare the library's step(s) with the oracle; return worst errors."""
    before, after, history, hyper = run_step(wl, precision, hyper, schedule, sample, steps,
                                             scale_mode)
    sched = muon_oracle.HYBRID_SCHEDULE if schedule is None else schedule
    worst = {"O": 0.0, "O_over_tol": 0.0, "M": 0.0, "W_given_O": 0.0, "W": 0.0}
    for k, (W, G, M) in before.items():
        n, m = W.shape
        for s in range(steps):
            W, M, O_ref = muon_oracle.muon_step(W, G, M, lr=hyper["lr"], mu=hyper["mu"],
                                                wd=hyper["wd"], gamma=hyper["gamma"],
                                                nesterov_on=hyper["nesterov"], schedule=sched,
                                                scale_mode=scale_mode)
            e = rel(history[s][k], O_ref)
            worst["O"] = max(worst["O"], e)
            worst["O_over_tol"] = max(worst["O_over_tol"], e / tol_o(precision, (n, m)))
        W_gpu, M_gpu = after[k]
        worst["M"] = max(worst["M"], rel(M_gpu, M))
        worst["W"] = max(worst["W"], rel(W_gpu, W))
        if steps == 1:
            # the update arithmetic, given the library's own O'
            W0 = before[k][0]
            O_gpu = history[0][k]
            if scale_mode == "shape":
                O_sc = muon_oracle.rescale(O_gpu, n, m, hyper["gamma"])
            elif scale_mode == "unit_rms":
                O_sc = muon_oracle.rescale_unit_rms(O_gpu, hyper["gamma"])
            else:
                O_sc = muon_oracle.rescale_none(O_gpu, hyper["gamma"])
            W_from_O = muon_oracle.decay_and_update(W0, O_sc, hyper["lr"], hyper["wd"])
            worst["W_given_O"] = max(worst["W_given_O"], rel(W_gpu, W_from_O))
    return worst


def check_ns(xs, precision="bf16", schedule=None, eps=1e-7):
    import muon_step_b200 as ms

    sched = muon_oracle.HYBRID_SCHEDULE if schedule is None else schedule
    outs = ms.ns_orthogonalize(xs, precision=precision, schedule=schedule, eps=None if eps == 1e-7 else eps)
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    errs = []
    for x, o in zip(xs, outs):
        ref = muon_oracle.ns_orthogonalize(x.double().cpu().numpy(), sched, eps)
        errs.append((tuple(x.shape), rel(o.double().cpu().numpy(), ref), tol_o(precision, tuple(x.shape))))
    return errs


def all_within(errs):
    return all(e <= t for _, e, t in errs)
