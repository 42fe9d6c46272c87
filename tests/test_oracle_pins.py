"""Pins for the float64 oracle: facts fixed by the pages and by mathematics.

Each test ties the oracle to something other than itself: numbers the pages
print (tests/golden/, each file citing its page and section), closed forms that
use LAPACK's SVD in place of the iteration, and exact special cases. The last
test plants plausible mistakes in the oracle and checks that some pin fails for
every one of them.
"""

import math
import os

import numpy as np
import pytest

from oracle import muon_oracle
from oracle import muon_oracle as oracle
from tests.conftest import read_golden

EPS = 1e-7


# ----------------------------------------------------------------------------
# helpers written from the pages' scalar view, independent of the oracle
# ----------------------------------------------------------------------------

def golden_schedule(golden_dir):
    rows = read_golden(os.path.join(golden_dir, "hybrid_schedule.txt"))
    return [tuple(float(v) for v in r[1:4]) for r in rows]


def p_scalar(sigma, schedule):
    """Composition of the scalar quintics p(s) = a s + b s^3 + c s^5.

    "Ch 06 · Muon" §3: in the singular basis every NS step maps each singular
    value through the same odd quintic while U and V stay fixed.
    """
    s = np.asarray(sigma, dtype=np.float64)
    for a, b, c in schedule:
        s = a * s + b * s**3 + c * s**5
    return s


def random_orthogonal(rng, n, k):
    """n x k with orthonormal columns (QR of a Gaussian, sign-fixed)."""
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))


def matrix_with_spectrum(rng, n, m, sigmas):
    k = len(sigmas)
    U = random_orthogonal(rng, n, k)
    V = random_orthogonal(rng, m, k)
    return (U * np.asarray(sigmas)) @ V.T


def closed_form(N, schedule, eps=EPS):
    """U p(S / (||S||_2 + eps)) V^T from LAPACK's SVD (||N||_F = ||S||_2)."""
    U, S, Vt = np.linalg.svd(N, full_matrices=False)
    s0 = S / (math.sqrt(float(np.sum(S * S))) + eps)
    return (U * p_scalar(s0, schedule)) @ Vt


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ----------------------------------------------------------------------------
# printed numbers
# ----------------------------------------------------------------------------

def test_schedule_is_the_printed_table(golden_dir):
    sched = golden_schedule(golden_dir)
    assert len(sched) == 10
    assert [tuple(x) for x in oracle.HYBRID_SCHEDULE] == sched


def test_band_of_the_hybrid_schedule(golden_dir):
    lo_in, hi_in, lo_out, hi_out = (float(v) for v in
                                    read_golden(os.path.join(golden_dir, "band.txt"))[0])
    s = np.linspace(lo_in, hi_in, 20001)
    out = p_scalar(s, golden_schedule(golden_dir))
    # printed to 4 decimals: [1.0000, 1.0020]
    assert out.min() >= lo_out - 5e-5
    assert out.max() <= hi_out + 5e-5


def test_band_through_the_oracle(golden_dir):
    """Matrices whose normalised singular values fill the printed input band."""
    lo_in, hi_in, lo_out, hi_out = (float(v) for v in
                                    read_golden(os.path.join(golden_dir, "band.txt"))[0])
    rng = np.random.default_rng(11)
    r, c = 48, 80
    # choose raw singular values so that S / ||S||_2 spans [lo_in, hi_in]
    t = np.linspace(lo_in, hi_in, r)
    X0 = matrix_with_spectrum(rng, r, c, t)
    X0 /= np.linalg.norm(X0)  # oracle normalises again; scale the band after
    S_target = np.linspace(lo_in, hi_in, r)
    U, _, Vt = np.linalg.svd(X0, full_matrices=False)
    X0 = (U * S_target) @ Vt
    O = oracle.hybrid_newton_schulz(X0)
    sv = np.linalg.svd(O, compute_uv=False)
    assert sv.min() >= lo_out - 5e-5 and sv.max() <= hi_out + 5e-5


def test_worked_example_norms(golden_dir):
    rng = np.random.default_rng(3)
    for n, m, fro_ns, fro_scaled in read_golden(os.path.join(golden_dir, "worked_example.txt")):
        n, m, fro_ns, fro_scaled = int(n), int(m), float(fro_ns), float(fro_scaled)
        r = min(n, m)
        N = matrix_with_spectrum(rng, n, m, rng.uniform(1.0, 2.0, r))
        O_prime = oracle.ns_orthogonalize(N)
        ratio = np.linalg.norm(O_prime) / fro_ns
        assert 1.0 - 1e-6 <= ratio <= 1.0021
        # the step with gamma = 1, lr = 1, wd = 0 on W = 0 gives W' = -O
        W_new, _, _ = oracle.muon_step(np.zeros((n, m)), N, np.zeros((n, m)), lr=1.0,
                                       mu=0.0, wd=0.0, gamma=1.0)
        assert 1.0 - 1e-6 <= np.linalg.norm(W_new) / fro_scaled <= 1.0021


def test_update_rms_lemma():
    """RMS(U V^T) = sqrt(r / (n m)); after sqrt(max) * gamma the RMS is gamma.

    "Muon 优化器完全拆解…", section "更新尺度": the lemma and the 0.2 alignment.
    """
    rng = np.random.default_rng(5)
    gamma = 0.2
    for n, m in [(96, 96), (64, 192), (192, 64)]:
        N = matrix_with_spectrum(rng, n, m, rng.uniform(0.5, 1.0, min(n, m)))
        O_prime = oracle.ns_orthogonalize(N)
        rms = np.sqrt(np.mean(O_prime**2))
        assert abs(rms / math.sqrt(1.0 / max(n, m)) - 1) < 2.1e-3
        O = oracle.rescale(O_prime, n, m, gamma)
        assert abs(np.sqrt(np.mean(O**2)) / gamma - 1) < 2.1e-3


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------

SHAPES = [(1, 1), (1, 7), (7, 1), (8, 8), (5, 12), (12, 5), (33, 47), (47, 33), (64, 64)]


@pytest.mark.parametrize("n,m", SHAPES)
@pytest.mark.parametrize("spectrum", ["flat", "geometric"])
def test_closed_form_via_svd(golden_dir, n, m, spectrum):
    rng = np.random.default_rng(n * 1000 + m)
    r = min(n, m)
    if spectrum == "flat":
        sig = rng.uniform(0.5, 1.5, r)
    else:
        sig = np.geomspace(1.0, 1e-3, r) if r > 1 else np.array([1.0])
    N = matrix_with_spectrum(rng, n, m, sig) * 3e-2
    got = oracle.ns_orthogonalize(N)
    want = closed_form(N, golden_schedule(golden_dir))
    assert rel(got, want) <= 1e-12


def test_singular_vectors_preserved():
    """"Ch 06 · Muon" §3: U and V do not change; U^T O' V is diagonal."""
    rng = np.random.default_rng(9)
    N = matrix_with_spectrum(rng, 40, 56, np.geomspace(1, 1e-2, 40))
    U, S, Vt = np.linalg.svd(N, full_matrices=False)
    D = U.T @ oracle.ns_orthogonalize(N) @ Vt.T
    off = D - np.diag(np.diag(D))
    assert np.abs(off).max() < 1e-12


def test_polar_factor_and_shampoo_identity():
    """Well-conditioned input: O' is within the band's 2e-3 of U V^T, computed
    two independent ways: SVD, and (N N^T)^{-1/4} N (N^T N)^{-1/4} by eigh
    ("Muon 优化器完全拆解…", section "Muon 的定义": the Shampoo identity)."""
    rng = np.random.default_rng(21)
    n, m = 40, 72
    N = matrix_with_spectrum(rng, n, m, rng.uniform(0.7, 1.2, n))
    U, _, Vt = np.linalg.svd(N, full_matrices=False)
    polar = U @ Vt

    def inv_quarter(S):
        w, Q = np.linalg.eigh(S)
        w = np.where(w > 1e-12 * w.max(), w, np.inf)
        return (Q * w**-0.25) @ Q.T

    shampoo = inv_quarter(N @ N.T) @ N @ inv_quarter(N.T @ N)
    assert rel(shampoo, polar) < 1e-10
    assert rel(oracle.ns_orthogonalize(N), polar) <= 2.0e-3


# ----------------------------------------------------------------------------
# exact special cases
# ----------------------------------------------------------------------------

def test_nesterov_expansion():
    """N = mu M_t + G = (1 + mu) G + mu^2 M_{t-1}
    ("Muon 优化器完全拆解…", Algorithm 1 explanation, "第二步：Nesterov 技巧")."""
    rng = np.random.default_rng(1)
    G = rng.standard_normal((17, 23))
    Mp = rng.standard_normal((17, 23))
    for mu in (0.0, 0.5, 0.95):
        M = oracle.momentum(Mp, G, mu)
        N = oracle.nesterov(M, G, mu)
        assert np.allclose(N, (1 + mu) * G + mu * mu * Mp, rtol=1e-14, atol=1e-14)
        assert np.allclose(M, mu * Mp + G, rtol=1e-14, atol=1e-14)


def test_zero_gradient_gives_pure_decay():
    rng = np.random.default_rng(2)
    W = rng.standard_normal((24, 40))
    Z = np.zeros_like(W)
    lr, wd = 0.02, 0.1
    W_new, M_new, O_prime = oracle.muon_step(W, Z, Z, lr=lr, wd=wd)
    assert not np.any(O_prime)
    assert not np.any(M_new)
    assert np.array_equal(W_new, W * (1 - lr * wd))


def test_rank_one(golden_dir):
    rng = np.random.default_rng(4)
    u = rng.standard_normal(30)
    v = rng.standard_normal(50)
    for scale in (1e-3, 1.0, 1e3):
        N = scale * np.outer(u, v)
        fro = np.linalg.norm(N)
        s0 = fro / (fro + EPS)
        want = p_scalar(s0, golden_schedule(golden_dir)) * np.outer(u / np.linalg.norm(u),
                                                                    v / np.linalg.norm(v))
        # the null directions hold float64 rounding (~1e-16); the composed
        # map's slope at 0 is a^8 * 2^2 ~ 7.9e4, which amplifies it
        assert rel(oracle.ns_orthogonalize(N), want) < 1e-16 * 7.9e4 * 30


def test_semi_orthogonal_input(golden_dir):
    rng = np.random.default_rng(6)
    for r, c in [(16, 16), (16, 64), (64, 16)]:
        Q = random_orthogonal(rng, max(r, c), min(r, c))
        Q = Q.T if r < c else Q  # r x c with orthonormal rows or columns
        k = min(r, c)
        s0 = 1.0 / (math.sqrt(k) + EPS)
        want = p_scalar(s0, golden_schedule(golden_dir)) * Q
        assert rel(oracle.ns_orthogonalize(Q), want) < 1e-13


def test_zero_padding_leaves_block_unchanged():
    rng = np.random.default_rng(8)
    N = matrix_with_spectrum(rng, 20, 36, np.geomspace(1, 1e-2, 20))
    P = np.zeros((29, 45))
    P[:20, :36] = N
    O = oracle.ns_orthogonalize(N)
    OP = oracle.ns_orthogonalize(P)
    assert rel(OP[:20, :36], O) < 1e-12
    assert np.abs(OP[20:, :]).max() == 0 and np.abs(OP[:, 36:]).max() == 0


def test_orientation_and_scale():
    rng = np.random.default_rng(10)
    N = matrix_with_spectrum(rng, 52, 20, np.geomspace(1, 1e-2, 20))  # tall
    O = oracle.ns_orthogonalize(N)
    # iterating on the tall matrix directly (X X^T is 52 x 52) gives the same map
    direct = oracle.hybrid_newton_schulz(N / (np.linalg.norm(N) + EPS))
    assert rel(O, direct) < 1e-12
    assert rel(oracle.ns_orthogonalize(N.T), O.T) < 1e-15
    # scale invariance up to the eps term
    assert rel(oracle.ns_orthogonalize(1e4 * N), O) < 1e-9


# ----------------------------------------------------------------------------
# planted mistakes: every one must trip at least one pin
# ----------------------------------------------------------------------------

def _pins(golden_dir):
    """Run a compact set of pins; return the names of those that fail."""
    failed = []
    checks = {
        "closed_form_wide": lambda: test_closed_form_via_svd(golden_dir, 12, 20, "geometric"),
        "closed_form_tall": lambda: test_closed_form_via_svd(golden_dir, 20, 12, "flat"),
        "schedule": lambda: test_schedule_is_the_printed_table(golden_dir),
        "worked_example": lambda: test_worked_example_norms_small(golden_dir),
        "nesterov": test_nesterov_expansion,
        "zero": test_zero_gradient_gives_pure_decay,
        "step_closed_form": lambda: test_step_against_closed_form(golden_dir),
    }
    for name, fn in checks.items():
        try:
            with np.errstate(all="ignore"):
                fn()
        except Exception:  # AssertionError, shape errors, NaN comparisons
            failed.append(name)
    return failed


def test_worked_example_norms_small(golden_dir):
    """Scaled-down worked example (same shape ratio), used by the mutation check."""
    rng = np.random.default_rng(12)
    for n, m in [(32, 32), (8, 128)]:
        N = matrix_with_spectrum(rng, n, m, rng.uniform(1.0, 2.0, min(n, m)))
        W_new, _, O_prime = oracle.muon_step(np.zeros((n, m)), N, np.zeros((n, m)), lr=1.0,
                                             mu=0.0, wd=0.0, gamma=1.0)
        assert 1 - 1e-6 <= np.linalg.norm(O_prime) / math.sqrt(min(n, m)) <= 1.0021
        assert 1 - 1e-6 <= np.linalg.norm(W_new) / math.sqrt(n * m) <= 1.0021


def test_step_against_closed_form(golden_dir):
    """Whole step: W' = W (1 - lr wd) - lr gamma sqrt(max) U p(S0) V^T with
    N = (1 + mu) G + mu^2 M_prev; all from the pages' closed forms."""
    rng = np.random.default_rng(13)
    n, m = 18, 10
    W = rng.standard_normal((n, m))
    G = rng.standard_normal((n, m))
    Mp = rng.standard_normal((n, m))
    lr, mu, wd, gamma = 0.02, 0.95, 0.1, 0.2
    N = (1 + mu) * G + mu * mu * Mp
    want = W * (1 - lr * wd) - lr * gamma * math.sqrt(max(n, m)) * closed_form(
        N, golden_schedule(golden_dir))
    W_new, M_new, _ = oracle.muon_step(W, G, Mp, lr=lr, mu=mu, wd=wd, gamma=gamma)
    assert rel(W_new, want) < 1e-12
    assert rel(M_new, mu * Mp + G) < 1e-15


MUTATIONS = {
    "b_sign": ("ns_step", lambda X, a, b, c: _ns(X, a, -b, c)),
    "drop_c": ("ns_step", lambda X, a, b, c: _ns(X, a, b, 0.0)),
    "product_on_wrong_side": ("ns_step", lambda X, a, b, c: _ns_wrong_side(X, a, b, c)),
    "c_times_A_not_A2": ("ns_step", lambda X, a, b, c: _ns_c_linear(X, a, b, c)),
    "no_eps": ("frobenius_normalise", lambda N, eps=EPS: N / np.sqrt(np.sum(N * N))),
    "fro_squared": ("frobenius_normalise", lambda N, eps=EPS: N / (np.sum(N * N) + eps)),
    "nesterov_uses_g_only": ("nesterov", lambda M, G, mu: G),
    "momentum_dampened": ("momentum", lambda Mp, G, mu: mu * Mp + (1 - mu) * G),
    "rescale_min": ("rescale", lambda O, n, m, g: O * math.sqrt(min(n, m)) * g),
    "decay_subtract": ("decay_and_update", lambda W, O, lr, wd: W - lr * wd - lr * O),
    "no_transpose_back": ("orient", lambda N: (N.T.copy(), N.shape[0] > N.shape[1])),
}


def _ns(X, a, b, c):
    A = X @ X.T
    return a * X + b * (A @ X) + c * ((A @ A) @ X)


def _ns_wrong_side(X, a, b, c):
    # X (X X^T) in place of (X X^T) X: a shape error unless X is square
    A = X @ X.T
    return a * X + b * (X @ A) + c * ((X @ A) @ A)


def _ns_c_linear(X, a, b, c):
    A = X @ X.T
    return a * X + b * (A @ X) + c * (A @ X)


def test_pins_pass_on_the_oracle(golden_dir):
    assert _pins(golden_dir) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(golden_dir, monkeypatch, name):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(muon_oracle, attr, fn)
    assert _pins(golden_dir), f"planted mistake {name!r} passed every pin"


def test_planted_schedule_mistakes_are_caught(golden_dir, monkeypatch):
    bad = [
        muon_oracle.HYBRID_SCHEDULE[::-1],                          # standard steps first
        (muon_oracle.AGGRESSIVE_ABC,) * 10,                         # no standard tail
        ((3.4445, -4.7750, 2.0135),) * 8 + (muon_oracle.STANDARD_ABC,) * 2,  # digit typo
    ]
    for sched in bad:
        monkeypatch.setattr(muon_oracle, "HYBRID_SCHEDULE", sched)
        # the schedule default is bound when the function is defined: wrap it
        monkeypatch.setattr(muon_oracle, "ns_orthogonalize",
                            lambda X, schedule=sched, eps=EPS, _f=muon_oracle.ns_orthogonalize:
                            _f(X, schedule, eps))
        assert _pins(golden_dir), "schedule mistake passed every pin"
        monkeypatch.undo()


# ----------------------------------------------------------------------------
# scale modes
# ----------------------------------------------------------------------------

def test_unit_rms_mode_has_rms_gamma_and_matches_shape_mode():
    """unit_rms_norm: RMS(O) = gamma exactly. The page calls it equivalent in
    theory to the shape rescale, since the RMS of an orthogonalised update is
    close to sqrt(1 / max(n, m)) ("Muon 优化器完全拆解…", section
    "另一条路：开源生态干脆不分片"), so on well-conditioned inputs the two agree
    within the band."""
    rng = np.random.default_rng(31)
    for n, m in [(48, 48), (32, 96), (96, 32)]:
        N = matrix_with_spectrum(rng, n, m, rng.uniform(0.7, 1.2, min(n, m)))
        Z = np.zeros((n, m))
        W_u, _, O_p = oracle.muon_step(Z, N, Z, lr=1.0, mu=0.0, wd=0.0, gamma=0.2, scale_mode="unit_rms")
        assert abs(np.sqrt(np.mean(W_u ** 2)) - 0.2) < 1e-12
        W_s, _, _ = oracle.muon_step(Z, N, Z, lr=1.0, mu=0.0, wd=0.0, gamma=0.2, scale_mode="shape")
        assert rel(W_u, W_s) <= 2.1e-3


def test_none_mode_is_the_plain_direction_and_zero_stays_zero():
    rng = np.random.default_rng(32)
    W = rng.standard_normal((20, 30))
    G = rng.standard_normal((20, 30))
    W_n, _, O_p = oracle.muon_step(W, G, np.zeros_like(W), lr=0.1, mu=0.9, wd=0.01, gamma=1.0,
                                   scale_mode="none")
    assert np.allclose(W_n, W * (1 - 0.1 * 0.01) - 0.1 * O_p, rtol=1e-14, atol=1e-15)
    Z = np.zeros_like(W)
    for mode in ("unit_rms", "none"):
        W_z, _, _ = oracle.muon_step(W, Z, Z, lr=0.1, wd=0.01, scale_mode=mode)
        assert np.array_equal(W_z, W * (1 - 0.1 * 0.01))


@pytest.mark.parametrize("n,m,br,bc", [(24, 96, 6, 24), (96, 24, 24, 6), (30, 30, 10, 10)])
def test_permuted_block_diagonal_inputs_orthogonalise_blockwise(n, m, br, bc):
    """For G and M_prev of the form P blockdiag(B_1 .. B_k) Q the oracle's O'
    is exactly zero off the blocks, and on each block it is the iteration of
    that block divided by the whole matrix's norm ([V4-book] §3: each step
    multiplies by a polynomial in X X^T). The full-size GPU checks of the two
    largest sweep bases rest on this."""
    import workloads
    from tests.parity import blockwise_oracle

    wl, supports = workloads.make_block_permuted(n, m, 2, br, bc, device="cpu", seed=3)
    h = wl.hyper
    for i in range(wl.count):
        W, G, M = (t[i].double().numpy() for t in (wl.W, wl.G, wl.M))
        _, _, O = muon_oracle.muon_step(W, G, M, lr=h["lr"], mu=h["mu"], wd=h["wd"],
                                        gamma=h["gamma"])
        rows, cols = (t.numpy() for t in supports[i])
        idx = (rows[:, :, None], cols[:, None, :])
        off = O.copy()
        off[idx] = 0.0
        assert not off.any()
        ref = blockwise_oracle(G[idx], M[idx], h)
        assert np.max(np.abs(O[idx] - ref)) <= 1e-12 * np.max(np.abs(ref))
        # the blocks share one normalisation: a block orthogonalised alone
        # differs from it by far more than the agreement above
        alone = muon_oracle.ns_orthogonalize(muon_oracle.nesterov(
            muon_oracle.momentum(M[idx][0], G[idx][0], h["mu"]), G[idx][0], h["mu"]))
        assert np.max(np.abs(alone - ref[0])) > 1e-7 * np.max(np.abs(ref))
