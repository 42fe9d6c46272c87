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



def tol_o(precision, shape):
    """The O' bound for one matrix: 2e-2 in the bf16 precision, 1e-4 in fp32,
    at every size."""
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


def blockwise_oracle(Gb, Mb, hyper, schedule=None):
    """O' of a permuted block-diagonal matrix P blockdiag(B_1 .. B_k) Q from
    the float64 oracle, block by block: the blocks of G and M_prev are given
    as [k, rows, cols] stacks (the same support). Every Newton-Schulz step
    multiplies X by a polynomial in X X^T, which is block-diagonal under the
    same row permutation when X is, and permutations commute with the
    iteration; so O' is the oracle's iteration of each block divided by the
    WHOLE matrix's norm, and zero off the blocks (pinned against the oracle's
    whole-matrix step in tests/test_oracle_pins.py). Returns the blocks of O'
    in the caller's orientation."""
    sched = muon_oracle.HYBRID_SCHEDULE if schedule is None else schedule
    mu = hyper["mu"]
    Mt = muon_oracle.momentum(Mb, Gb, mu)
    N = muon_oracle.nesterov(Mt, Gb, mu) if hyper["nesterov"] else Mt
    fro = math.sqrt(float(np.sum(N * N)))
    out = []
    for Nj in N:
        X, transposed = muon_oracle.orient(Nj)
        O = muon_oracle.hybrid_newton_schulz(X / (fro + muon_oracle.DEFAULT_EPS), sched)
        out.append(O.T if transposed else O)
    return np.stack(out)
