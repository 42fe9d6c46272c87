"""Seeded synthetic inputs for the Muon step (W, G, M_prev per matrix).

This module holds no arithmetic of the method: it only draws matrices with the
shapes, scales and spectra of the five workloads below. Both the float64 oracle
(through the tests) and the GPU library consume its fp32 tensors. Inputs are
generated with torch on the requested device from a seeded generator; the same
(workload, seed, device) always gives the same bytes.

Workloads (shapes and distributions):

* ``single_256x512`` - one 256 x 512 matrix. W ~ N(0, 0.02^2); M_prev ~ N(0, 1e-4)
  (variance 1e-4); G = sum_{k=1..16} 10^(-3(k-1)/15) a_k b_k^T / sqrt(512)
  + 1e-4 N(0, 1) with a_k, b_k ~ N(0, 1). Seed 0.
* ``batch64_1024`` - 64 square 1024 x 1024 matrices. G is rank 64 with random
  orthogonal factors and singular values geometric from 1 to 1e-3, plus
  1e-4 N(0, 1) noise.
* ``dense_d4096`` - a 16-layer transformer stack at d = 4096: per layer
  Q, K, V, O 4096 x 4096, FFN gate and up 4096 x 14336, down 14336 x 4096
  (112 matrices). G = N(0, 1e-3^2) + a rank-32 spike with random orthogonal
  factors and singular values geometric over three decades, the smallest at
  1e-3 (sqrt(n) + sqrt(m)) (the noise's spectral edge).
* ``moe_64x3`` - 64 experts x {gate 2048 x 7168, up 2048 x 7168, down
  7168 x 2048} (192 matrices). G_e = s_e U diag(geom 1 -> 1e-4) V^T, full rank,
  random orthogonal U, V, with the expert scale s_e log-uniform in
  [1e-4, 1e-1].
* ``sweep_<b>_<aspect>`` - b in {128, 512, 2048, 8192, 16384}, aspect in
  {1x1, 1x4, 4x1}; batch = floor(16e9 / (12 n m)) matrices (about 16 GB of
  fp32 W, M, G). Singular values geometric from 1 to 1e-4: full rank with
  random orthogonal factors when min(n, m) <= 512, else rank 64 plus noise
  N(0, (1e-4 / sqrt(max(n, m)))^2).

``make_sweep_blocks`` gives a sweep point's shapes and batch with G and M_prev
of the form P blockdiag(B_1, ..., B_k) Q (random row and column permutations P,
Q; full-rank blocks of 512 rows with the sweep's spectrum), for element-wise
checks at sizes where the oracle cannot take a whole matrix.

Except for ``single_256x512``, whose M_prev is specified, M_prev is an
independent draw of the workload's own gradient recipe, so that N keeps the
intended spectrum. W is N(0, 0.02^2) everywhere. Hyper-parameters: lr 0.02,
mu 0.95 (Nesterov), weight decay 0.1, gamma 0.2.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

HYPER = dict(lr=0.02, mu=0.95, wd=0.1, gamma=0.2, nesterov=True)

SWEEP_BASES = (128, 512, 2048, 8192, 16384)
SWEEP_ASPECTS = ("1x1", "1x4", "4x1")


@dataclass
class Workload:
    """Per-matrix fp32 tensors (views into one buffer per shape group)."""

    name: str
    shapes: list
    W: list
    G: list
    M: list
    hyper: dict = field(default_factory=lambda: dict(HYPER))
    groups: dict = field(default_factory=dict)  # (n, m) -> (W, G, M) [k, n, m]

    @property
    def count(self):
        return len(self.shapes)

    def elements(self):
        return sum(n * m for n, m in self.shapes)


# ----------------------------------------------------------------------------
# primitive draws
# ----------------------------------------------------------------------------

def _generator(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _dtype(device):
    # float64 draws on the host (cast to fp32 at the end); fp32 on the GPU
    return torch.float64 if torch.device(device).type == "cpu" else torch.float32


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=_dtype(device))


def random_orthogonal(batch, n, k, g, device):
    """[batch, n, k] with orthonormal columns: QR of a Gaussian, sign-fixed."""
    a = _randn((batch, n, k), g, device)
    q, r = torch.linalg.qr(a)
    d = torch.sign(torch.diagonal(r, dim1=-2, dim2=-1))
    d[d == 0] = 1
    return q * d.unsqueeze(-2)


def spectrum_matrix(batch, n, m, sigma, g, device):
    """[batch, n, m] = U diag(sigma) V^T with random orthogonal U, V.

    ``sigma`` is [k] or [batch, k]."""
    sigma = torch.as_tensor(sigma, device=device, dtype=_dtype(device))
    k = sigma.shape[-1]
    U = random_orthogonal(batch, n, k, g, device)
    V = random_orthogonal(batch, m, k, g, device)
    if sigma.dim() == 1:
        sigma = sigma.expand(batch, k)
    return torch.matmul(U * sigma.unsqueeze(-2), V.transpose(-1, -2))


def _geom(hi, lo, k, device):
    if k == 1:
        return torch.tensor([hi], device=device, dtype=_dtype(device))
    return torch.logspace(math.log10(hi), math.log10(lo), k, device=device,
                          dtype=_dtype(device))


# ----------------------------------------------------------------------------
# gradient recipes (each returns a [batch, n, m] tensor)
# ----------------------------------------------------------------------------

def grad_single(n, m, g, device):
    out = 1e-4 * _randn((1, n, m), g, device)
    for k in range(1, 17):
        a = _randn((n, 1), g, device)
        b = _randn((1, m), g, device)
        out[0] += (10.0 ** (-3.0 * (k - 1) / 15.0)) * (a @ b) / math.sqrt(512.0)
    return out


def grad_lowrank_noise(batch, n, m, rank, hi, lo, noise_std, g, device):
    out = spectrum_matrix(batch, n, m, _geom(hi, lo, min(rank, n, m), device), g, device)
    return out + noise_std * _randn((batch, n, m), g, device)


def grad_dense_spike(batch, n, m, g, device):
    s_min = 1e-3 * (math.sqrt(n) + math.sqrt(m))
    spike = spectrum_matrix(batch, n, m, _geom(1e3 * s_min, s_min, 32, device), g, device)
    return spike + 1e-3 * _randn((batch, n, m), g, device)


def grad_fullrank_scaled(batch, n, m, scales, g, device):
    sig = _geom(1.0, 1e-4, min(n, m), device)
    out = spectrum_matrix(batch, n, m, sig, g, device)
    return out * torch.as_tensor(scales, device=device, dtype=out.dtype).view(batch, 1, 1)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

def _finish(name, order, groups, device):
    """Views per matrix in ``order`` = [(shape, index_in_group)]."""
    W, G, M, shapes = [], [], [], []
    for shape, i in order:
        w, gg, mm = groups[shape]
        W.append(w[i])
        G.append(gg[i])
        M.append(mm[i])
        shapes.append(shape)
    return Workload(name=name, shapes=shapes, W=W, G=G, M=M, groups=groups)


def _to32(t):
    return t.to(torch.float32).contiguous()


def _weights(batch, n, m, g, device):
    return _to32(0.02 * _randn((batch, n, m), g, device))


def make_single_256x512(device="cpu", seed=0):
    n, m = 256, 512
    gw, gm, gg = (_generator(device, 1000 * seed + k) for k in range(3))
    W = _weights(1, n, m, gw, device)
    M = _to32(0.01 * _randn((1, n, m), gm, device))
    G = _to32(grad_single(n, m, gg, device))
    return _finish("single_256x512", [((n, m), 0)], {(n, m): (W, G, M)}, device)


def make_batch64_1024(device="cpu", seed=1, count=64, size=1024):
    n = m = size
    gw, gm, gg = (_generator(device, 1000 * seed + k) for k in range(3))
    W = _weights(count, n, m, gw, device)
    G = torch.empty((count, n, m), device=device, dtype=torch.float32)
    M = torch.empty_like(G)
    chunk = 8
    for s in range(0, count, chunk):
        e = min(count, s + chunk)
        G[s:e] = grad_lowrank_noise(e - s, n, m, 64, 1.0, 1e-3, 1e-4, gg, device)
        M[s:e] = grad_lowrank_noise(e - s, n, m, 64, 1.0, 1e-3, 1e-4, gm, device)
    return _finish("batch64_1024", [((n, m), i) for i in range(count)],
                   {(n, m): (W, G, M)}, device)


DENSE_LAYER = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
               ("gate", 4096, 14336), ("up", 4096, 14336), ("down", 14336, 4096))


def make_dense_d4096(device="cpu", seed=2, layers=16, d=4096, ffn=14336):
    shapes = [(d, d)] * 4 + [(d, ffn), (d, ffn), (ffn, d)]
    return _stack("dense_d4096", shapes, layers, device, seed,
                  lambda b, n, m, g: grad_dense_spike(b, n, m, g, device))


def make_moe_64x3(device="cpu", seed=3, experts=64, d=2048, f=7168):
    shapes = [(d, f), (d, f), (f, d)]
    gs = _generator(device, 1000 * seed + 7)
    # log-uniform expert scales in [1e-4, 1e-1], one per expert for G and for M_prev
    u = torch.rand((2, experts), generator=gs, device=device, dtype=_dtype(device))
    scales = 10.0 ** (-4.0 + 3.0 * u)
    state = {"k": 0}

    def grad(b, n, m, g, which):
        e0 = state["k"]
        return grad_fullrank_scaled(b, n, m, scales[which, e0:e0 + b], g, device)

    return _stack("moe_64x3", shapes, experts, device, seed, grad, expert_state=state)


def _stack(name, per_unit_shapes, units, device, seed, grad_fn, expert_state=None):
    """units x per_unit_shapes matrices, grouped by shape, in unit-major order."""
    gw, gm, gg = (_generator(device, 1000 * seed + k) for k in range(3))
    counts = {}
    order = []
    for u in range(units):
        for shape in per_unit_shapes:
            order.append((shape, counts.get(shape, 0)))
            counts[shape] = counts.get(shape, 0) + 1
    groups = {}
    for shape, k in counts.items():
        n, m = shape
        W = _weights(k, n, m, gw, device)
        G = torch.empty((k, n, m), device=device, dtype=torch.float32)
        M = torch.empty_like(G)
        groups[shape] = (W, G, M)
    # draw gradients matrix by matrix (bounded temporary memory)
    for shape, i in order:
        n, m = shape
        if expert_state is not None:
            per = per_unit_shapes.count(shape)
            expert_state["k"] = i // per
            G1 = grad_fn(1, n, m, gg, 0)
            M1 = grad_fn(1, n, m, gm, 1)
        else:
            G1 = grad_fn(1, n, m, gg)
            M1 = grad_fn(1, n, m, gm)
        groups[shape][1][i] = G1[0].to(torch.float32)
        groups[shape][2][i] = M1[0].to(torch.float32)
    return _finish(name, order, groups, device)


def sweep_shape(base, aspect):
    if aspect == "1x1":
        return base, base
    if aspect == "1x4":
        return base, 4 * base
    if aspect == "4x1":
        return 4 * base, base
    raise ValueError(aspect)


def sweep_batch(n, m, state_bytes=16e9):
    return max(1, int(state_bytes // (12 * n * m)))


def make_sweep(base, aspect, device="cpu", seed=5, count=None):
    n, m = sweep_shape(base, aspect)
    count = sweep_batch(n, m) if count is None else count
    gw, gm, gg = (_generator(device, 1000 * seed + k) for k in range(3))
    W = _weights(count, n, m, gw, device)
    G = torch.empty((count, n, m), device=device, dtype=torch.float32)
    M = torch.empty_like(G)
    r, c = min(n, m), max(n, m)
    chunk = max(1, int(2**27 // (n * m)))
    for s in range(0, count, chunk):
        e = min(count, s + chunk)
        for dst, g in ((G, gg), (M, gm)):
            if r <= 512:
                dst[s:e] = spectrum_matrix(e - s, n, m, _geom(1.0, 1e-4, r, device), g, device)
            else:
                dst[s:e] = grad_lowrank_noise(e - s, n, m, 64, 1.0, 1e-4, 1e-4 / math.sqrt(c),
                                              g, device)
    return _finish(f"sweep_{base}_{aspect}", [((n, m), i) for i in range(count)],
                   {(n, m): (W, G, M)}, device)


def sweep_block_shape(n, m, block=512):
    """Block shape of the permuted block-diagonal sweep inputs: block x block
    for a square matrix, block x 4 block (or 4 block x block) along the
    aspect, so that min(n, m) / block blocks cover every row and column."""
    if n == m:
        return block, block
    return (block, 4 * block) if n < m else (4 * block, block)


def make_block_permuted(n, m, count, block_rows, block_cols, device="cpu", seed=6, name=None):
    """`count` n x m matrices whose G and M_prev have the form
    P blockdiag(B_1, ..., B_k) Q: k = n / block_rows = m / block_cols blocks
    along the diagonal, P and Q random permutations of the rows and columns
    (one pair per matrix, shared by its G and M_prev), every block a full-rank
    block_rows x block_cols matrix with random orthogonal factors and singular
    values geometric from 1 to 1e-4 (the sweep recipe for matrices of up to
    512 rows). W ~ N(0, 0.02^2) as everywhere.

    Returns (workload, supports): supports[i] = (rows, cols), int64 tensors of
    shape [k, block_rows] and [k, block_cols], the row and column indices of
    matrix i's blocks."""
    if n % block_rows or m % block_cols or n // block_rows != m // block_cols:
        raise ValueError("blocks must tile the diagonal")
    k = n // block_rows
    gw, gm, gg, gp = (_generator(device, 1000 * seed + j) for j in range(4))
    W = _weights(count, n, m, gw, device)
    G = torch.zeros((count, n, m), device=device, dtype=torch.float32)
    M = torch.zeros_like(G)
    sig = _geom(1.0, 1e-4, min(block_rows, block_cols), device)
    supports = []
    for i in range(count):
        rows = torch.randperm(n, generator=gp, device=device).view(k, block_rows)
        cols = torch.randperm(m, generator=gp, device=device).view(k, block_cols)
        for dst, g in ((G, gg), (M, gm)):
            blocks = spectrum_matrix(k, block_rows, block_cols, sig, g, device)
            dst[i][rows[:, :, None], cols[:, None, :]] = blocks.to(torch.float32)
        supports.append((rows, cols))
    wl = _finish(name or f"blocks_{n}x{m}", [((n, m), i) for i in range(count)],
                 {(n, m): (W, G, M)}, device)
    return wl, supports


def make_sweep_blocks(base, aspect, device="cpu", seed=6, count=None, block=512):
    """A sweep point's shapes and batch with permuted block-diagonal G and
    M_prev (make_block_permuted, blocks of sweep_block_shape)."""
    n, m = sweep_shape(base, aspect)
    count = sweep_batch(n, m) if count is None else count
    br, bc = sweep_block_shape(n, m, block)
    return make_block_permuted(n, m, count, br, bc, device, seed,
                               name=f"sweep_blocks_{base}_{aspect}")


def make(name, device="cpu", **kw):
    """Build a workload by name (see the module docstring)."""
    if name == "single_256x512":
        return make_single_256x512(device, **kw)
    if name == "batch64_1024":
        return make_batch64_1024(device, **kw)
    if name == "dense_d4096":
        return make_dense_d4096(device, **kw)
    if name == "moe_64x3":
        return make_moe_64x3(device, **kw)
    if name.startswith("sweep_"):
        _, b, a = name.split("_")
        return make_sweep(int(b), a, device, **kw)
    raise KeyError(name)


def make_random(shapes, device="cpu", seed=0, spectrum="geometric"):
    """Small mixed-shape workloads for parity tests: W ~ N(0, 0.02^2),
    G and M_prev = U diag(sigma) V^T (+ 1e-4 N(0,1)) with sigma geometric
    from 1 to 1e-3 ("geometric") or uniform in [0.5, 1.5] ("flat")."""
    gw, gm, gg = (_generator(device, 1000 * seed + k) for k in range(3))
    order, groups, counts = [], {}, {}
    for shape in shapes:
        order.append((tuple(shape), counts.get(tuple(shape), 0)))
        counts[tuple(shape)] = counts.get(tuple(shape), 0) + 1
    for shape, k in counts.items():
        n, m = shape
        r = min(n, m)
        W = _weights(k, n, m, gw, device)
        if spectrum == "geometric":
            sig = _geom(1.0, 1e-3, r, device)
        else:
            sig = 0.5 + torch.rand((r,), generator=gg, device=device, dtype=_dtype(device))
        G = spectrum_matrix(k, n, m, sig, gg, device) + 1e-4 * _randn((k, n, m), gg, device)
        M = spectrum_matrix(k, n, m, sig, gm, device) + 1e-4 * _randn((k, n, m), gm, device)
        groups[shape] = (W, _to32(G), _to32(M))
    return _finish("random", order, groups, device)
