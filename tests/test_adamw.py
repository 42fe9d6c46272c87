"""AdamW companion step and Muon/AdamW routing.

Host-side checks (no GPU): argument validation, workspace size, routing.
GPU checks: the kernel against the float64 AdamW oracle over several steps on
ragged, unaligned and empty tensors, the device-held step counter, the one-shot
call, and the hybrid optimizer end to end.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from muon_step_b200 import _lib
from muon_step_b200._lib import (MUON_ERR_INVALID_ARG, MUON_ERR_WORKSPACE, MUON_OK, AdamwHyper,
                                 AdamwParam)
from muon_step_b200.hybrid import route

FAKE = 0x10000  # plan creation records pointers but never dereferences them
TOL = 1e-6      # relative Frobenius error, fp32 arithmetic against float64


@pytest.fixture(scope="module")
def lib():
    from muon_step_b200 import build
    build.build()
    return _lib.load()


def adamw_params(sizes, offset=0):
    arr = (AdamwParam * len(sizes))()
    for k, n in enumerate(sizes):
        base = FAKE + k * (1 << 30) + offset
        arr[k] = AdamwParam(base, base + (1 << 28), base + (2 << 28), base + (3 << 28), n)
    return arr


def create(lib, arr):
    plan = ctypes.c_void_p()
    st = lib.muon_adamw_plan_create(arr, len(arr), ctypes.byref(plan))
    return st, plan


def test_plan_validation(lib):
    plan = ctypes.c_void_p()
    assert lib.muon_adamw_plan_create(None, 1, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    assert lib.muon_adamw_plan_create(adamw_params([4]), 0, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    assert create(lib, adamw_params([-1]))[0] == MUON_ERR_INVALID_ARG
    assert create(lib, adamw_params([(1 << 40) + 1]))[0] == MUON_ERR_INVALID_ARG
    assert create(lib, adamw_params([8], offset=2))[0] == MUON_ERR_INVALID_ARG  # not 4-byte aligned
    bad = adamw_params([8])
    bad[0].g = None
    assert create(lib, bad)[0] == MUON_ERR_INVALID_ARG
    # empty tensors are skipped, even with NULL pointers
    empty = adamw_params([0, 5])
    empty[0] = AdamwParam(None, None, None, None, 0)
    st, plan = create(lib, empty)
    assert st == MUON_OK
    n = ctypes.c_int64()
    assert lib.muon_adamw_plan_numel(plan, ctypes.byref(n)) == MUON_OK and n.value == 5
    lib.muon_adamw_plan_destroy(plan)


def work_items(sizes, chunk=4096):
    """The work list rule: 4096-element chunks of tensors above 2048 elements;
    runs of smaller tensors in bundles of at most 4096 elements and 64 tensors."""
    items, start, total, count = 0, None, 0, 0
    for n in (s for s in sizes if s > 0):
        if n > chunk // 2:
            items += (start is not None) + -(-n // chunk)
            start, total, count = None, 0, 0
            continue
        if start is not None and (total + n > chunk or count >= 64):
            items += 1
            start, total, count = None, 0, 0
        if start is None:
            start = True
        total += n
        count += 1
    return items + (start is not None)


@pytest.mark.parametrize("sizes", [[1], [4096, 4097, 3], [0, 0, 1, 2, 3, 4, 5, 6],
                                   [128] * 200, [100, 5000, 100, 100, 3000, 2000] * 3])
def test_workspace_holds_the_tensor_table_and_the_work_list(lib, sizes):
    st, plan = create(lib, adamw_params(sizes))
    assert st == MUON_OK
    ws = ctypes.c_size_t()
    assert lib.muon_adamw_plan_workspace_size(plan, ctypes.byref(ws)) == MUON_OK
    nonempty = sum(1 for n in sizes if n > 0)
    al = lambda x: (x + 255) // 256 * 256
    # 48-byte tensor entries, then 16-byte work items
    assert ws.value == al(max(nonempty, 1) * 48) + al(max(work_items(sizes), 1) * 16)
    one = ctypes.c_size_t()
    assert lib.muon_adamw_workspace_size(adamw_params(sizes), len(sizes), ctypes.byref(one)) == MUON_OK
    assert one.value == ws.value
    lib.muon_adamw_plan_destroy(plan)


def test_execute_rejects_bad_hyper_parameters_before_touching_a_device(lib):
    st, plan = create(lib, adamw_params([100]))
    assert st == MUON_OK
    ws = ctypes.c_void_p(1 << 20)
    good = dict(lr=0.02, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1, step=1, step_dev=None)
    for change in [dict(step=0), dict(beta1=1.0), dict(beta2=-0.1), dict(eps=0.0),
                   dict(lr=float("nan")), dict(weight_decay=float("inf")),
                   dict(step=0, step_dev=FAKE + 2)]:
        h = AdamwHyper(**{**good, **change})
        assert lib.muon_adamw_plan_execute(plan, ctypes.byref(h), ws, 1 << 20, None) == \
            MUON_ERR_INVALID_ARG, change
    h = AdamwHyper(**good)
    assert lib.muon_adamw_plan_execute(plan, ctypes.byref(h), ctypes.c_void_p((1 << 20) + 16),
                                       1 << 20, None) == MUON_ERR_WORKSPACE
    assert lib.muon_adamw_plan_execute(plan, ctypes.byref(h), ws, 16, None) == MUON_ERR_WORKSPACE
    lib.muon_adamw_plan_destroy(plan)


def test_route_follows_the_pages_split():
    named = [("tok_embed.weight", (32000, 512)), ("layers.0.attn.q.weight", (512, 512)),
             ("layers.0.attn.q.bias", (512,)), ("layers.0.norm.weight", (512,)),
             ("layers.0.mlp.up.weight", (2048, 512)), ("lm_head.weight", (32000, 512)),
             ("conv.weight", (8, 3, 3, 3)), ("gate.scale", ()), ("Embedding.W", (10, 4))]
    muon, adamw = route(named)
    assert muon == ["layers.0.attn.q.weight", "layers.0.mlp.up.weight"]
    assert adamw == ["tok_embed.weight", "layers.0.attn.q.bias", "layers.0.norm.weight",
                     "lm_head.weight", "conv.weight", "gate.scale", "Embedding.W"]
    muon, adamw = route(named, adamw_names=())
    assert "lm_head.weight" in muon and "tok_embed.weight" in muon


# ----------------------------------------------------------------------------
# GPU
# ----------------------------------------------------------------------------

def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / d) if d > 0 else float(np.linalg.norm(a - b))


def _tensors(sizes, seed, unaligned=()):
    g = torch.Generator(device="cuda").manual_seed(seed)
    out = []
    for k, n in enumerate(sizes):
        pad = 1 if k in unaligned else 0
        def make(scale):
            t = torch.randn(n + pad, generator=g, device="cuda") * scale
            return t[pad:] if pad else t
        p = make(1.0)
        m = make(1e-3)
        v = make(1e-3).abs() ** 2
        out.append([p, m, v])
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("betas,eps,wd", [((0.9, 0.999), 1e-8, 0.1), ((0.8, 0.95), 1e-6, 0.0)])
def test_adamw_matches_the_oracle(betas, eps, wd):
    import muon_step_b200 as ms
    from oracle import companion_oracle as co

    sizes = [1, 3, 4095, 4096, 4097, 12345, 1 << 20, 0, 777]
    state = _tensors(sizes, seed=3, unaligned=(6, 8))
    grads = [torch.empty_like(s[0]) for s in state]
    plan = ms.AdamWPlan([(p, g, m, v) for (p, m, v), g in zip(state, grads)])
    assert plan.numel == sum(sizes)
    ws = plan.alloc_workspace()
    ref = [[s[0].double().cpu().numpy(), s[1].double().cpu().numpy(), s[2].double().cpu().numpy()]
           for s in state]
    gen = torch.Generator(device="cuda").manual_seed(4)
    lr = 0.02
    for t in range(1, 6):
        for g in grads:
            g.copy_(torch.randn(g.shape, generator=gen, device="cuda") * 10.0 ** (-t))
        plan.execute(ws, lr=lr, betas=betas, eps=eps, weight_decay=wd, step=t)
        for k, g in enumerate(grads):
            ref[k] = list(co.adamw_step(ref[k][0], g.double().cpu().numpy(), ref[k][1], ref[k][2],
                                        t, lr=lr, beta1=betas[0], beta2=betas[1], eps=eps, wd=wd))
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    for k, (p, m, v) in enumerate(state):
        for got, want, name in ((p, ref[k][0], "p"), (m, ref[k][1], "m"), (v, ref[k][2], "v")):
            assert _rel(got.double().cpu().numpy(), want) <= TOL, (sizes[k], name)


@pytest.mark.gpu
def test_device_step_counter_and_one_shot_agree():
    import muon_step_b200 as ms

    sizes = [5000, 64]
    a = _tensors(sizes, seed=8)
    b = [[t.clone() for t in s] for s in a]
    grads = [torch.randn(n, device="cuda") for n in sizes]
    plan = ms.AdamWPlan([(p, g, m, v) for (p, m, v), g in zip(a, grads)])
    ws = plan.alloc_workspace()
    counter = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(1, 4):
        counter += 1
        plan.execute(ws, step_tensor=counter)
        ms.adamw_step([(p, g, m, v) for (p, m, v), g in zip(b, grads)], step=t)
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    # the bias corrections come from the device's pow() here and the host's there
    for sa, sb in zip(a, b):
        for x, y in zip(sa, sb):
            assert torch.allclose(x, y, rtol=1e-6, atol=0.0)


@pytest.mark.gpu
def test_hybrid_optimizer_end_to_end():
    """A toy model's parameters: Muon matrices and AdamW tensors updated by the
    library, each group against its float64 oracle."""
    import muon_step_b200 as ms
    from muon_step_b200.hybrid import HybridOptimizer
    from oracle import companion_oracle as co
    from oracle import muon_oracle

    torch.manual_seed(0)
    shapes = {"embed.weight": (1000, 64), "blocks.0.q.weight": (64, 64),
              "blocks.0.up.weight": (256, 64), "blocks.0.norm.weight": (64,),
              "blocks.0.up.bias": (256,), "head.weight": (1000, 64)}
    params = {n: torch.nn.Parameter(torch.randn(s, device="cuda") * 0.02) for n, s in shapes.items()}
    for p in params.values():
        p.grad = torch.zeros_like(p)
    opt = HybridOptimizer(params.items(), lr=0.02, weight_decay=0.1)
    diag = opt.enable_diagnostics()
    assert [n for n, _ in opt.muon_params] == ["blocks.0.q.weight", "blocks.0.up.weight"]
    start = {n: p.detach().double().cpu().numpy() for n, p in params.items()}
    ref = dict(start)
    mom = {n: np.zeros(shapes[n]) for n, _ in opt.muon_params}
    m1 = {n: np.zeros(shapes[n]) for n, _ in opt.adamw_params}
    m2 = {n: np.zeros(shapes[n]) for n, _ in opt.adamw_params}
    for t in range(1, 3):
        for p in params.values():
            p.grad.copy_(torch.randn_like(p) * 1e-2)
        grads = {n: p.grad.double().cpu().numpy() for n, p in params.items()}
        opt.step()
        torch.cuda.synchronize()
        for n, _ in opt.muon_params:
            ref[n], mom[n], _ = muon_oracle.muon_step(ref[n], grads[n], mom[n], lr=0.02,
                                                     mu=0.95, wd=0.1, gamma=0.2)
        for n, _ in opt.adamw_params:
            ref[n], m1[n], m2[n] = co.adamw_step(ref[n], grads[n], m1[n], m2[n], t,
                                                 lr=0.02, wd=0.1)
    assert ms.sync_status() == 0
    muon_names = {n for n, _ in opt.muon_params}
    for n, p in params.items():
        got = p.detach().double().cpu().numpy()
        if n in muon_names:
            # the bf16 orthogonaliser's error, relative to the two steps' total move
            move = np.linalg.norm(ref[n] - start[n])
            assert np.linalg.norm(got - ref[n]) <= 3e-2 * move, n
        else:
            assert _rel(got, ref[n]) <= TOL, n
    assert torch.isfinite(diag).all()
    assert (diag[:, 1] > 0.15).all() and (diag[:, 1] < 0.25).all(), diag


@pytest.mark.gpu
def test_many_small_tensors_in_bundles():
    """Hundreds of bias / norm sized tensors (bundled several per CTA) mixed
    with large ones, against the oracle."""
    import muon_step_b200 as ms
    from oracle import companion_oracle as co

    rng = np.random.default_rng(9)
    sizes = [int(s) for s in rng.integers(1, 3000, 300)] + [70000, 5, 9000]
    state = _tensors(sizes, seed=11, unaligned=(3, 150, 301))
    gen = torch.Generator(device="cuda").manual_seed(12)
    grads = [torch.randn(s[0].shape, generator=gen, device="cuda") * 1e-2 for s in state]
    ref = [[s[0].double().cpu().numpy(), s[1].double().cpu().numpy(), s[2].double().cpu().numpy()]
           for s in state]
    plan = ms.AdamWPlan([(p, g, m, v) for (p, m, v), g in zip(state, grads)])
    ws = plan.alloc_workspace()
    for t in (1, 2):
        plan.execute(ws, step=t)
        for k, g in enumerate(grads):
            ref[k] = list(co.adamw_step(ref[k][0], g.double().cpu().numpy(), ref[k][1], ref[k][2], t,
                                        lr=0.02, wd=0.1))
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    for k, (p, m, v) in enumerate(state):
        for got, want in ((p, ref[k][0]), (m, ref[k][1]), (v, ref[k][2])):
            assert _rel(got.double().cpu().numpy(), want) <= TOL, sizes[k]


def _gpt2_like(tied=True):
    import torch.nn as nn

    class Block(nn.Module):
        def __init__(self):
            super().__init__()
            self.ln = nn.LayerNorm(16)
            self.multi_head_attn = nn.Linear(16, 48)
            self.mlp = nn.Linear(16, 64)

    class Model(nn.Module):
        def __init__(self):
            super().__init__()
            self.wte = nn.Embedding(100, 16)
            self.wpe = nn.Embedding(32, 16)
            self.h = nn.ModuleList([Block()])
            self.out = nn.Linear(16, 100, bias=False)
            if tied:
                self.out.weight = self.wte.weight

    return Model()


def test_route_module_puts_tables_and_heads_on_adamw():
    from muon_step_b200.hybrid import route_module

    muon, adamw = route_module(_gpt2_like(tied=True))
    assert muon == ["h.0.multi_head_attn.weight", "h.0.mlp.weight"]
    assert adamw == ["wte.weight", "wpe.weight", "h.0.ln.weight", "h.0.ln.bias",
                     "h.0.multi_head_attn.bias", "h.0.mlp.bias"]
    muon, adamw = route_module(_gpt2_like(tied=False))
    assert muon == ["h.0.multi_head_attn.weight", "h.0.mlp.weight"]
    assert "out.weight" in adamw                      # untied head: output width = vocabulary
    muon, _ = route_module(_gpt2_like(tied=False), adamw_names=("mlp",))
    assert muon == ["h.0.multi_head_attn.weight"]


def test_hybrid_from_module_and_explicit_split():
    from muon_step_b200.hybrid import HybridOptimizer

    model = _gpt2_like()
    opt = HybridOptimizer.from_module(model)
    assert [n for n, _ in opt.muon_params] == ["h.0.multi_head_attn.weight", "h.0.mlp.weight"]
    assert len(opt.adamw_params) == 6
    with pytest.raises(ValueError):
        HybridOptimizer(model.named_parameters(), muon_names=["nope.weight"])
    with pytest.raises(ValueError):
        HybridOptimizer(model.named_parameters(), muon_names=["h.0.mlp.bias"])


def test_hybrid_rebuilds_when_a_parameter_moves():
    import torch

    from muon_step_b200.hybrid import HybridOptimizer

    w = torch.nn.Parameter(torch.zeros(8, 8))
    b = torch.nn.Parameter(torch.zeros(8))
    w.grad, b.grad = torch.zeros(8, 8), torch.zeros(8)
    opt = HybridOptimizer([("w", w), ("b", b)])
    key = opt._current_ptrs()
    assert opt._current_ptrs() == key
    w.data = torch.ones(8, 8)            # new storage for the parameter
    assert opt._current_ptrs() != key
    key = opt._current_ptrs()
    b.grad = torch.ones(8)               # new storage for a gradient
    assert opt._current_ptrs() != key
