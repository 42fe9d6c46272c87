"""Pins of the AdamW companion oracle and of the Muon diagnostics oracle.

The AdamW oracle is tied to (a) torch.optim.AdamW run in float64 on the CPU, a
library routine written independently of it, (b) closed forms of the first
step and of a constant gradient, and (c) the pure-decay special case. The
diagnostics are tied to the Nesterov identity and to the update-RMS lemma of
[V4-breakdown] section "更新尺度：让 Muon 借用 AdamW 的超参". Every planted
mistake below must trip at least one pin.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import companion_oracle as co
from oracle import muon_oracle


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


HYPERS = [
    dict(lr=0.02, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.1),
    dict(lr=1e-3, beta1=0.8, beta2=0.95, eps=1e-6, wd=0.0),
    dict(lr=0.3, beta1=0.5, beta2=0.7, eps=1e-3, wd=0.5),
]


def test_matches_torch_adamw_float64():
    """Ten steps with changing random gradients against torch.optim.AdamW."""
    rng = np.random.default_rng(5)
    for h in HYPERS:
        p0 = rng.standard_normal(257)
        grads = [rng.standard_normal(257) * 10.0 ** rng.uniform(-4, 1) for _ in range(10)]
        tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
        opt = torch.optim.AdamW([tp], lr=h["lr"], betas=(h["beta1"], h["beta2"]), eps=h["eps"],
                                weight_decay=h["wd"])
        p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
        for t, g in enumerate(grads, start=1):
            tp.grad = torch.tensor(g, dtype=torch.float64)
            opt.step()
            p, m, v = co.adamw_step(p, g, m, v, t, **h)
            assert rel(p, tp.detach().numpy()) < 1e-13
            st = opt.state[tp]
            assert rel(m, st["exp_avg"].numpy()) < 1e-13
            assert rel(v, st["exp_avg_sq"].numpy()) < 1e-13


def test_first_step_closed_form():
    """From zero moments, m_hat = g and v_hat = g^2: the move is g / (|g| + eps)."""
    rng = np.random.default_rng(6)
    for h in HYPERS:
        p = rng.standard_normal(64)
        g = rng.standard_normal(64) * 1e-3
        want = p * (1 - h["lr"] * h["wd"]) - h["lr"] * g / (np.abs(g) + h["eps"])
        got, m, v = co.adamw_step(p, g, np.zeros(64), np.zeros(64), 1, **h)
        assert rel(got, want) < 1e-14
        assert rel(m, (1 - h["beta1"]) * g) < 1e-15
        assert rel(v, (1 - h["beta2"]) * g * g) < 1e-15


def test_constant_gradient_keeps_the_first_move():
    """With a constant gradient the bias corrections undo the averages exactly:
    m_hat = g and v_hat = g^2 at every step."""
    h = HYPERS[0]
    g = np.array([0.5, -2.0, 1e-4, -3e-6])
    p = np.array([1.0, -1.0, 0.25, 4.0])
    m = np.zeros(4)
    v = np.zeros(4)
    for t in range(1, 30):
        want = p * (1 - h["lr"] * h["wd"]) - h["lr"] * g / (np.abs(g) + h["eps"])
        p, m, v = co.adamw_step(p, g, m, v, t, **h)
        assert rel(p, want) < 1e-12


def test_zero_gradient_is_pure_decay():
    p = np.linspace(-1, 1, 9)
    got, m, v = co.adamw_step(p, np.zeros(9), np.zeros(9), np.zeros(9), 1, lr=0.02, wd=0.1)
    assert np.array_equal(got, p * (1 - 0.02 * 0.1))
    assert not np.any(m) and not np.any(v)


def test_step_zero_is_rejected():
    with pytest.raises(ValueError):
        co.adamw_step(np.ones(2), np.ones(2), np.zeros(2), np.zeros(2), 0)


# ----------------------------------------------------------------------------
# diagnostics
# ----------------------------------------------------------------------------

def _orthogonal(rng, n):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


def test_diagnostic_norm_is_the_nesterov_input():
    """||N||_F with N = (1 + mu) G + mu^2 M_prev (the Nesterov expansion)."""
    rng = np.random.default_rng(7)
    G = rng.standard_normal((12, 20))
    Mp = rng.standard_normal((12, 20))
    mu = 0.95
    norm, _ = co.muon_step_diagnostics(G, Mp, 12, 20, mu=mu)
    assert abs(norm - np.linalg.norm((1 + mu) * G + mu * mu * Mp)) < 1e-12 * norm
    norm_plain, _ = co.muon_step_diagnostics(G, Mp, 12, 20, mu=mu, nesterov_on=False)
    assert abs(norm_plain - np.linalg.norm(mu * Mp + G)) < 1e-12 * norm_plain


@pytest.mark.parametrize("n,m", [(16, 16), (12, 40), (40, 12)])
def test_diagnostic_rms_follows_the_lemma(n, m):
    """Well-conditioned full-rank N: O' ~ U V^T with singular values in the
    band [1.0000, 1.0020], so RMS(O') = sqrt(1/max(n, m)) up to that band, the
    shape rule brings RMS(O) to gamma, unit-RMS gives gamma exactly and no
    rescale leaves gamma sqrt(1/max(n, m))."""
    rng = np.random.default_rng(n * 100 + m)
    r = min(n, m)
    U = _orthogonal(rng, n)[:, :r]
    V = _orthogonal(rng, m)[:, :r]
    N = U @ np.diag(rng.uniform(0.8, 1.2, r)) @ V.T
    gamma = 0.2
    zero = np.zeros((n, m))
    _, shape = co.muon_step_diagnostics(N, zero, n, m, mu=0.0, gamma=gamma)
    assert gamma * (1 - 1e-6) <= shape <= gamma * 1.0021
    _, unit = co.muon_step_diagnostics(N, zero, n, m, mu=0.0, gamma=gamma, scale_mode="unit_rms")
    assert abs(unit - gamma) < 1e-12
    _, none = co.muon_step_diagnostics(N, zero, n, m, mu=0.0, gamma=gamma, scale_mode="none")
    base = gamma / math.sqrt(max(n, m))
    assert base * (1 - 1e-6) <= none <= base * 1.0021


def test_diagnostics_of_a_zero_gradient():
    norm, r = co.muon_step_diagnostics(np.zeros((4, 6)), np.zeros((4, 6)), 4, 6)
    assert norm == 0.0 and r == 0.0


# ----------------------------------------------------------------------------
# planted mistakes
# ----------------------------------------------------------------------------

def _pins():
    failed = []
    for name, fn in {
        "torch": test_matches_torch_adamw_float64,
        "first_step": test_first_step_closed_form,
        "constant": test_constant_gradient_keeps_the_first_move,
        "zero": test_zero_gradient_is_pure_decay,
        "norm": test_diagnostic_norm_is_the_nesterov_input,
        "rms_square": lambda: test_diagnostic_rms_follows_the_lemma(16, 16),
        "rms_wide": lambda: test_diagnostic_rms_follows_the_lemma(12, 40),
    }.items():
        try:
            with np.errstate(all="ignore"):
                fn()
        except Exception:
            failed.append(name)
    return failed


def _no_bias_correction(m, v, step, beta1, beta2, eps):
    return m / (np.sqrt(v) + eps)


def _eps_inside(m, v, step, beta1, beta2, eps):
    return (m / (1 - beta1 ** step)) / np.sqrt(v / (1 - beta2 ** step) + eps)


def _coupled_decay(p, g, m, v, step, lr=0.02, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.1):
    g = np.asarray(g, np.float64) + wd * np.asarray(p, np.float64)
    m_new, v_new = co.adamw_moments(m, v, g, beta1, beta2)
    return np.asarray(p, np.float64) - lr * co.adamw_update(m_new, v_new, step, beta1, beta2, eps), m_new, v_new


def _decay_after_move(p, g, m, v, step, lr=0.02, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.1):
    m_new, v_new = co.adamw_moments(m, v, g, beta1, beta2)
    u = co.adamw_update(m_new, v_new, step, beta1, beta2, eps)
    return (np.asarray(p, np.float64) - lr * u) * (1 - lr * wd), m_new, v_new


def _swapped_betas(m, v, g, beta1, beta2):
    g = np.asarray(g, np.float64)
    return beta2 * m + (1 - beta2) * g, beta1 * v + (1 - beta1) * g * g


def _abs_not_square(m, v, g, beta1, beta2):
    g = np.asarray(g, np.float64)
    return beta1 * m + (1 - beta1) * g, beta2 * v + (1 - beta2) * np.abs(g)


def _rms_over_rows(O):
    O = np.asarray(O, np.float64)
    return float(np.sqrt(np.sum(O * O) / O.shape[0]))


def _norm_squared(N):
    return float(np.sum(np.asarray(N, np.float64) ** 2))


MUTATIONS = {
    "no_bias_correction": ("adamw_update", _no_bias_correction),
    "eps_inside_sqrt": ("adamw_update", _eps_inside),
    "coupled_decay": ("adamw_step", _coupled_decay),
    "decay_after_move": ("adamw_step", _decay_after_move),
    "swapped_betas": ("adamw_moments", _swapped_betas),
    "abs_not_square": ("adamw_moments", _abs_not_square),
    "rms_over_rows": ("rms", _rms_over_rows),
    "norm_squared": ("frobenius_norm", _norm_squared),
}


def test_pins_pass_on_the_oracle():
    assert _pins() == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(monkeypatch, name):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(co, attr, fn)
    assert _pins(), f"planted mistake {name!r} passed every pin"


def test_muon_pieces_are_the_muon_oracle():
    """The diagnostics reuse the pinned Muon oracle, not a copy of it."""
    assert co.muon_oracle is muon_oracle
