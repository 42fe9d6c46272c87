"""Float64 CPU oracle for the AdamW companion step and the Muon diagnostics.

TEST INFRASTRUCTURE ONLY, like muon_oracle.py: only the test suite,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it; the library never does, and this module imports nothing from it.

Sources (cited by page title and section):

* [V4-breakdown] "Muon 优化器完全拆解：矩阵级正交化更新如何撑起万亿 MoE 训练".
  - Section "AdamW 到底哪里”不协调”": AdamW moves each element by its
    bias-corrected first-moment average over the square root of its
    bias-corrected second-moment average, with a small constant eps against
    division by zero.
  - Algorithm 1, step five: the decoupled weight decay, written as a
    multiplication by (1 - lr * wd), is the form AdamW introduced; the Muon
    group and the AdamW group share lr and wd = 0.1.
  - Section "为什么嵌入层、输出头、bias、RMSNorm 还在用 AdamW": embeddings,
    the prediction head, biases, gates and all RMSNorm weights stay on AdamW;
    every other (matrix) parameter goes to Muon.
  - Section "更新尺度：让 Muon 借用 AdamW 的超参": the update-RMS lemma, which
    the diagnostics measure (RMS of O' near sqrt(1 / max(n, m)); RMS of the
    rescaled update near gamma).

Readings where the pages leave a point open:

* The moments are the usual exponential averages, m = b1 m + (1 - b1) g and
  v = b2 v + (1 - b2) g^2, with bias corrections 1 - b1^t and 1 - b2^t at step
  t = 1, 2, ...; eps is added to the square root of the corrected v.
  [V4-breakdown] prints neither b1, b2 nor eps; the defaults here are the customary 0.9, 0.999
  and 1e-8, and all three are parameters.
* The decay multiplies the parameter before the Adam move:
  p <- p (1 - lr wd) - lr m_hat / (sqrt(v_hat) + eps).
"""

from __future__ import annotations

import numpy as np

from . import muon_oracle

DEFAULT_BETAS = (0.9, 0.999)
DEFAULT_EPS = 1e-8


def adamw_moments(m: np.ndarray, v: np.ndarray, g: np.ndarray, beta1: float, beta2: float):
    """Exponential averages of the gradient and of its square."""
    g = np.asarray(g, np.float64)
    m_new = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v_new = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    return m_new, v_new


def adamw_update(m: np.ndarray, v: np.ndarray, step: int, beta1: float, beta2: float,
                 eps: float) -> np.ndarray:
    """The Adam move m_hat / (sqrt(v_hat) + eps) with bias-corrected moments."""
    if step < 1:
        raise ValueError("AdamW steps count from 1")
    m_hat = m / (1.0 - beta1 ** step)
    v_hat = v / (1.0 - beta2 ** step)
    return m_hat / (np.sqrt(v_hat) + eps)


def adamw_step(p, g, m, v, step: int, lr: float = 0.02, beta1: float = DEFAULT_BETAS[0],
               beta2: float = DEFAULT_BETAS[1], eps: float = DEFAULT_EPS, wd: float = 0.1):
    """One AdamW step on one tensor: returns (p', m', v') in float64."""
    m_new, v_new = adamw_moments(m, v, g, beta1, beta2)
    u = adamw_update(m_new, v_new, step, beta1, beta2, eps)
    p_new = np.asarray(p, np.float64) * (1.0 - lr * wd) - lr * u
    return p_new, m_new, v_new


def frobenius_norm(N: np.ndarray) -> float:
    """||N||_F, the quantity the Muon step divides by (plus eps)."""
    N = np.asarray(N, np.float64)
    return float(np.sqrt(np.sum(N * N)))


def rms(O: np.ndarray) -> float:
    """Root mean square over the elements: ||O||_F / sqrt(number of elements)."""
    O = np.asarray(O, np.float64)
    return float(np.sqrt(np.mean(O * O))) if O.size else 0.0


def muon_step_diagnostics(G, M_prev, n: int, m: int, mu: float = 0.95, gamma: float = 0.2,
                          nesterov_on: bool = True, schedule=muon_oracle.HYBRID_SCHEDULE,
                          eps: float = muon_oracle.DEFAULT_EPS, scale_mode: str = "shape"):
    """(||N||_F, RMS(O)) of one Muon step: the norm of the orthogonaliser's
    input and the RMS of the scaled update O that multiplies lr."""
    M = muon_oracle.momentum(np.asarray(M_prev, np.float64), np.asarray(G, np.float64), mu)
    N = muon_oracle.nesterov(M, np.asarray(G, np.float64), mu) if nesterov_on else M
    O_prime = muon_oracle.ns_orthogonalize(N, schedule, eps)
    if scale_mode == "shape":
        O = muon_oracle.rescale(O_prime, n, m, gamma)
    elif scale_mode == "unit_rms":
        O = muon_oracle.rescale_unit_rms(O_prime, gamma)
    elif scale_mode == "none":
        O = muon_oracle.rescale_none(O_prime, gamma)
    else:
        raise ValueError(scale_mode)
    return frobenius_norm(N), rms(O)
