"""Float64 CPU oracle for the Muon optimizer step on 2-D weight matrices.

TEST INFRASTRUCTURE ONLY. This module states, as plainly as possible, what the
GPU library computes, so that the GPU results can be checked against it. Only
the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it. The library's product path never imports, links or
calls anything here, and this module imports nothing from the library.

Sources (web pages on the method; cited by page title and section):

* [V4-breakdown] "Muon 优化器完全拆解：矩阵级正交化更新如何撑起万亿 MoE 训练"
  (pinghaoyang.com.cn/aigc/posts/muon-optimizer-deepseek-v4/).
  Section "V4 的完整更新公式，逐行拆解" (the update formula and its terms),
  section "更新尺度：让 Muon 借用 AdamW 的超参" (the RMS rescale).
* [V4-book] "Ch 06 · Muon — 矩阵参数的指南针" (DeepSeek-V4-book, chapter 6).
  §3 "Newton–Schulz：用 5 次 matmul 近似 polar" (the iteration),
  §4 "为什么 V4 要做 Hybrid 两段式 10 步" (the 8 + 2 schedule),
  §5 "完整算法" (the expanded Algorithm 1 "Muon Optimizer (V4 Hybrid)").

Each function below is the plain mathematical definition of one term of the
update, in float64 and in the pages' notation; ``muon_step`` composes them.
Matrix products use numpy's ``@`` (a library matmul) and nothing else: no
blocking, fusion or reordering.

Readings where the pages leave a point open (each also listed in the design
notes of the repository):

* The normalisation adds eps = 1e-7 to the Frobenius norm, outside the square
  root: X0 = N / (||N||_F + eps). The pages divide by ||N||_F alone.
* A matrix with more rows than columns is orthogonalised in its transposed
  form (rows <= cols) and transposed back. In exact arithmetic the iteration
  commutes with transposition, so this changes only rounding.
* The momentum has no (1 - mu) dampening: the formula M = mu*M + G rules over
  the word "EMA" in the surrounding text.
* gamma defaults to 0.2 (Moonlight's value); DeepSeek-V4 uses 0.18. It is a
  parameter.

Parity pins (tests/test_oracle_pins.py) tie this module to facts fixed by the
pages and by mathematics, not to itself:

* closed form: on small inputs the iteration equals U p(S) V^T with p the
  composition of the scalar quintics and U, S, V from LAPACK's SVD;
* the printed singular-value band of the hybrid schedule;
* the printed coefficient table;
* the worked shape example (Frobenius norms 32, 16 and 1024);
* the update-RMS lemma, the Nesterov identity, the polar factor, and the
  special cases (zero, rank-1, semi-orthogonal, padding, transpose, scale).
"""

from __future__ import annotations

import numpy as np

# [V4-book] §4 and §5 Algorithm 1; [V4-breakdown] section
# "另一条路：开源生态干脆不分片" (the Megatron-Bridge "deepseekv4" coefficient entry): eight aggressive
# steps, then two standard Newton-Schulz steps.
AGGRESSIVE_ABC = (3.4445, -4.7750, 2.0315)
STANDARD_ABC = (2.0, -1.5, 0.5)
HYBRID_SCHEDULE = (AGGRESSIVE_ABC,) * 8 + (STANDARD_ABC,) * 2

DEFAULT_EPS = 1e-7


def momentum(M_prev: np.ndarray, G: np.ndarray, mu: float) -> np.ndarray:
    """Momentum accumulation M_t = mu * M_{t-1} + G_t (no dampening).

    [V4-breakdown] section "V4 的完整更新公式，逐行拆解"; [V4-book] §5.
    """
    return mu * M_prev + G


def nesterov(M: np.ndarray, G: np.ndarray, mu: float) -> np.ndarray:
    """Nesterov look-ahead N_t = mu * M_t + G_t (the input to orthogonalisation).

    [V4-breakdown] section "V4 的完整更新公式，逐行拆解"; [V4-book] §5.
    """
    return mu * M + G


def orient(N: np.ndarray) -> tuple[np.ndarray, bool]:
    """Return (X, transposed): X = N^T when N has more rows than columns."""
    if N.shape[0] > N.shape[1]:
        return N.T.copy(), True
    return N.copy(), False


def frobenius_normalise(N: np.ndarray, eps: float = DEFAULT_EPS) -> np.ndarray:
    """X = N / (||N||_F + eps), which puts every singular value in [0, 1).

    [V4-book] §5: N is scaled into the region where the iteration of §3
    converges.
    """
    fro = np.sqrt(np.sum(N * N))
    return N / (fro + eps)


def ns_step(X: np.ndarray, a: float, b: float, c: float) -> np.ndarray:
    """One Newton-Schulz step X <- a X + b (X X^T) X + c (X X^T)^2 X.

    The quintic as [V4-book] §3 writes it: three terms, each a product with
    the Gram matrix X X^T.
    """
    A = X @ X.T
    return a * X + b * (A @ X) + c * ((A @ A) @ X)


def hybrid_newton_schulz(X0: np.ndarray, schedule=HYBRID_SCHEDULE) -> np.ndarray:
    """Compose the schedule's quintic steps, first to last ([V4-book] §4:
    eight aggressive steps, then two standard ones, by default)."""
    X = X0
    for a, b, c in schedule:
        X = ns_step(X, a, b, c)
    return X


def rescale(O_prime: np.ndarray, n: int, m: int, gamma: float) -> np.ndarray:
    """O = O' * sqrt(max(n, m)) * gamma.

    [V4-breakdown] section "更新尺度：让 Muon 借用 AdamW 的超参"; [V4-book] §5.
    """
    return O_prime * (np.sqrt(float(max(n, m))) * gamma)


def rescale_unit_rms(O_prime: np.ndarray, gamma: float) -> np.ndarray:
    """O = gamma * O' / RMS(O'): the update normalised to unit RMS, then scaled.

    [V4-breakdown] section "另一条路：开源生态干脆不分片", the Megatron-Bridge
    recipe's muon_scale_mode "unit_rms_norm" with muon_extra_scale_factor
    gamma: the update is brought to unit RMS, then multiplied by the extra
    factor (0.2 in that recipe). A zero O' stays zero.
    """
    rms = np.sqrt(np.mean(O_prime * O_prime))
    return O_prime * (gamma / rms) if rms > 0.0 else np.zeros_like(O_prime)


def rescale_none(O_prime: np.ndarray, gamma: float) -> np.ndarray:
    """O = gamma * O': no shape-dependent rescale, as in the original Muon
    ([V4-breakdown] section "V4 的完整更新公式，逐行拆解": the original Muon
    had neither weight decay nor the RMS rescale; gamma = 1 reproduces it)."""
    return O_prime * gamma


SCALE_MODES = ("shape", "unit_rms", "none")


def decay_and_update(W: np.ndarray, O: np.ndarray, lr: float, wd: float) -> np.ndarray:
    """Decoupled weight decay and step: W_t = W_{t-1} (1 - lr*wd) - lr * O_t.

    [V4-breakdown] section "V4 的完整更新公式，逐行拆解"; [V4-book] §5.
    """
    return W * (1.0 - lr * wd) - lr * O


def ns_orthogonalize(X: np.ndarray, schedule=HYBRID_SCHEDULE,
                     eps: float = DEFAULT_EPS) -> np.ndarray:
    """O' = HybridNewtonSchulz(X / (||X||_F + eps)), in X's own orientation."""
    X = np.asarray(X, dtype=np.float64)
    Xo, transposed = orient(X)
    O = hybrid_newton_schulz(frobenius_normalise(Xo, eps), schedule)
    return O.T.copy() if transposed else O


def muon_step(W, G, M_prev, lr=0.02, mu=0.95, wd=0.1, gamma=0.2,
              nesterov_on=True, schedule=HYBRID_SCHEDULE, eps=DEFAULT_EPS, scale_mode="shape"):
    """One Muon step for one n x m matrix, all in float64:

        M_t = mu M_{t-1} + G_t,   N_t = mu M_t + G_t,
        O'_t = NS(N_t / (||N_t||_F + eps)),
        W_t = W_{t-1} (1 - lr wd) - lr * scale(O'_t),

    the composition of the definitions above. Returns (W_t, M_t, O'_t) where
    O'_t is the orthogonalised direction before the RMS rescale, in W's
    orientation. With ``nesterov_on`` false the orthogonaliser's input is M_t
    itself (the original Muon). ``scale_mode``
    picks the update's scale: "shape" (sqrt(max(n, m)) gamma, the default),
    "unit_rms" (gamma / RMS(O')) or "none" (gamma).
    """
    W = np.asarray(W, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M_prev = np.asarray(M_prev, dtype=np.float64)
    n, m = W.shape
    M = momentum(M_prev, G, mu)
    N = nesterov(M, G, mu) if nesterov_on else M
    O_prime = ns_orthogonalize(N, schedule, eps)
    if scale_mode == "shape":
        O = rescale(O_prime, n, m, gamma)
    elif scale_mode == "unit_rms":
        O = rescale_unit_rms(O_prime, gamma)
    elif scale_mode == "none":
        O = rescale_none(O_prime, gamma)
    else:
        raise ValueError(scale_mode)
    W_new = decay_and_update(W, O, lr, wd)
    return W_new, M, O_prime
