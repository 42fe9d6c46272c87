"""Parity of the CUDA path with the float64 oracle on seeded inputs.

Tolerances (relative Frobenius error per matrix): O' <= 2e-2 in the bf16
precision at every size (matrices of at most 4096 elements take fp32
operands there, and are held to 1e-4 in their own test), <= 1e-4 in the fp32
validation precision; the momentum buffer and the update (given the
library's own O') <= 1e-6.
"""

import math

import numpy as np
import pytest
import torch

import workloads
from tests.parity import TOL_ELEMENTWISE, TOL_O, all_within, check_ns, check_step, rel, tol_o

pytestmark = pytest.mark.gpu

RAGGED = [(1, 1), (1, 7), (7, 1), (3, 5), (5, 3), (64, 64), (80, 96), (128, 128), (129, 257),
          (257, 129), (130, 130), (300, 1000), (1000, 300), (7, 1500), (128, 256), (384, 640)]

# tiny matrices (at most 4096 elements): fp32 operands in the bf16 precision
TINY = [(1, 1), (1, 2), (2, 1), (1, 4096), (4096, 1), (3, 5), (5, 3), (7, 100), (100, 7), (16, 16),
        (64, 64), (33, 47), (47, 33), (17, 240), (240, 17), (2, 2048)]


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available()
    import muon_step_b200 as ms
    ms.library()
    yield


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_single_256x512(precision):
    wl = workloads.make("single_256x512", device="cuda")
    worst = check_step(wl, precision)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE, worst
    assert worst["W_given_O"] <= TOL_ELEMENTWISE, worst


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("spectrum", ["geometric", "flat"])
def test_ragged_mixed_shapes(precision, spectrum):
    wl = workloads.make_random(RAGGED, device="cuda", seed=7, spectrum=spectrum)
    worst = check_step(wl, precision)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE, worst
    assert worst["W_given_O"] <= TOL_ELEMENTWISE, worst


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_ns_orthogonalize(precision):
    wl = workloads.make_random(RAGGED, device="cuda", seed=3)
    errs = check_ns(list(wl.G), precision)
    assert all_within(errs), errs


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_ns_orthogonalize_gaussian_rectangular(precision):
    """Gaussian matrices with aspect >= 2 (well-conditioned: the normalised
    singular values stay away from 0, where the composed map is steepest)."""
    shapes = [(1, 7), (7, 1), (3, 9), (129, 300), (300, 129), (64, 512), (1000, 300)]
    g = torch.Generator(device="cuda").manual_seed(3)
    xs = [torch.randn(n, m, device="cuda", generator=g) for n, m in shapes]
    errs = check_ns(xs, precision)
    assert all_within(errs), errs


def test_zero_matrix_is_pure_decay():
    n, m = 200, 333
    W = torch.randn(n, m, device="cuda")
    W0 = W.double().cpu().numpy()
    G = torch.zeros(n, m, device="cuda")
    M = torch.zeros(n, m, device="cuda")
    O = torch.full((n, m), 7.0, device="cuda")
    import muon_step_b200 as ms
    ms.muon_step([(W, G, M, O)], lr=0.02, weight_decay=0.1)
    torch.cuda.synchronize()
    assert torch.count_nonzero(O).item() == 0
    assert torch.count_nonzero(M).item() == 0
    assert rel(W.double().cpu().numpy(), W0 * (1 - 0.02 * 0.1)) <= TOL_ELEMENTWISE


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_nesterov_off_and_other_hyper(precision):
    wl = workloads.make_random([(96, 160), (160, 96)], device="cuda", seed=9)
    hyper = dict(lr=0.05, mu=0.9, wd=0.01, gamma=0.18, nesterov=False)
    worst = check_step(wl, precision, hyper=hyper)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE and worst["W_given_O"] <= TOL_ELEMENTWISE, worst


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_five_step_quintic_schedule(precision):
    sched = ((3.4445, -4.7750, 2.0315),) * 5
    wl = workloads.make_random([(200, 520), (520, 200)], device="cuda", seed=11)
    worst = check_step(wl, precision, schedule=sched)
    assert worst["O_over_tol"] <= 1.0, worst


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_three_consecutive_steps(precision):
    wl = workloads.make_random([(256, 384), (384, 256)], device="cuda", seed=13)
    worst = check_step(wl, precision, steps=3)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE, worst


def test_batch64_1024_sampled():
    """The benchmark's workload at full size (64 x 1024 x 1024, one grouped
    launch per stage); 6 matrices checked against the oracle."""
    wl = workloads.make("batch64_1024", device="cuda")
    sample = [0, 1, 17, 31, 48, 63]
    worst = check_step(wl, "bf16", sample=sample)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE and worst["W_given_O"] <= TOL_ELEMENTWISE, worst


def test_timeout_is_reported_and_the_context_survives():
    import muon_step_b200 as ms
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    ms.wait_probe(flag, 2_000_000)  # 2 ms, nothing sets the flag
    assert ms.sync_status() == 5    # MUON_ERR_TIMEOUT
    assert ms.sync_status() == 0    # cleared
    flag.fill_(1)
    ms.wait_probe(flag, 2_000_000)
    assert ms.sync_status() == 0
    # the device still runs the library's kernels
    wl = workloads.make_random([(64, 96)], device="cuda", seed=1)
    assert check_step(wl, "bf16")["O_over_tol"] <= 1.0


def test_cuda_graph_replay_matches_eager():
    """A plan executed from a captured CUDA graph gives the same bits as eager
    launches (the kernels are deterministic)."""
    import muon_step_b200 as ms
    shapes = [(256, 640), (640, 256), (300, 300)]
    a = workloads.make_random(shapes, device="cuda", seed=17)
    b = workloads.make_random(shapes, device="cuda", seed=17)
    h = a.hyper
    kw = dict(lr=h["lr"], momentum=h["mu"], weight_decay=h["wd"], gamma=h["gamma"])
    pa = ms.MuonPlan([(a.W[k], a.G[k], a.M[k]) for k in range(a.count)])
    pb = ms.MuonPlan([(b.W[k], b.G[k], b.M[k]) for k in range(b.count)])
    wa, wb = pa.alloc_workspace(), pb.alloc_workspace()
    pa.execute(wa, **kw)
    pa.execute(wa, **kw)
    pb.execute(wb, **kw)  # first execute on this workspace copies the descriptors
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g.capture_begin()
        pb.execute(wb, stream=s, **kw)
        g.capture_end()
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    for k in range(a.count):
        assert torch.equal(a.W[k], b.W[k]) and torch.equal(a.M[k], b.M[k])


def test_distributed_step_world_one_matches_plan():
    """DistributedMuon with its default compute (the library's plan over the
    owned matrices) and an NCCL group of one rank equals a direct plan."""
    import datetime
    import os
    import socket

    import torch.distributed as dist

    import muon_step_b200 as ms
    from muon_step_b200.distributed import DistributedMuon

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shapes = [(300, 500), (500, 300), (64, 64)]
        a = workloads.make_random(shapes, device="cuda", seed=23)
        b = workloads.make_random(shapes, device="cuda", seed=23)
        opt = DistributedMuon([(a.W[k], a.G[k], a.M[k]) for k in range(a.count)])
        opt.step()
        plan = ms.MuonPlan([(b.W[k], b.G[k], b.M[k]) for k in range(b.count)])
        plan.execute()
        torch.cuda.synchronize()
        for k in range(a.count):
            assert torch.equal(a.W[k], b.W[k]) and torch.equal(a.M[k], b.M[k])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("scale_mode", ["unit_rms", "none"])
def test_scale_modes(precision, scale_mode):
    """Unit-RMS and no-rescale updates on small, large, transposed and
    unaligned matrices (small-matrix kernel, grouped kernels, update pass)."""
    shapes = [(64, 64), (100, 37), (100, 120), (300, 520), (520, 300), (257, 129), (1, 7),
              (40, 1024), (130, 2048)]
    wl = workloads.make_random(shapes, device="cuda", seed=29)
    hyper = dict(wl.hyper, gamma=0.2 if scale_mode == "unit_rms" else 1.0)
    worst = check_step(wl, precision, hyper=hyper, scale_mode=scale_mode)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE and worst["W_given_O"] <= TOL_ELEMENTWISE, worst


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("scale_mode", ["shape", "unit_rms", "none"])
def test_diagnostics(precision, scale_mode):
    """||N||_F and RMS(O) per matrix, in the caller's order, against the
    oracle: the norm to fp32 rounding of a double sum; the update RMS against
    the RMS of the GPU's own O' to 1e-5 (the epilogue sums in fp32), and
    against the full oracle within the O' tolerance."""
    import muon_step_b200 as ms
    from oracle import companion_oracle

    shapes = [(300, 520), (64, 64), (520, 300), (1, 7), (257, 129), (100, 37), (96, 80)]
    wl = workloads.make_random(shapes, device="cuda", seed=31)
    h = wl.hyper
    before = [(wl.G[k].double().cpu().numpy(), wl.M[k].double().cpu().numpy())
              for k in range(wl.count)]
    O = [torch.empty_like(wl.W[k]) for k in range(wl.count)]
    plan = ms.MuonPlan([(wl.W[k], wl.G[k], wl.M[k], O[k]) for k in range(wl.count)],
                       precision=precision, scale_mode=scale_mode)
    diag = torch.full((wl.count, 2), -1.0, device="cuda")
    plan.set_diagnostics(diag)
    ws = plan.alloc_workspace()
    plan.execute(ws, lr=h["lr"], momentum=h["mu"], weight_decay=h["wd"], gamma=h["gamma"],
                 nesterov=h["nesterov"])
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    got = diag.double().cpu().numpy()
    for k in range(wl.count):
        G, Mp = before[k]
        n, m = G.shape
        norm, rms_o = companion_oracle.muon_step_diagnostics(
            G, Mp, n, m, mu=h["mu"], gamma=h["gamma"], nesterov_on=h["nesterov"],
            scale_mode=scale_mode)
        assert abs(got[k, 0] - norm) <= 1e-6 * norm, (k, got[k, 0], norm)
        Og = O[k].double().cpu().numpy()
        r = companion_oracle.rms(Og)
        if scale_mode == "shape":
            own = h["gamma"] * math.sqrt(max(n, m)) * r
        elif scale_mode == "unit_rms":
            own = h["gamma"] if r > 0 else 0.0
        else:
            own = h["gamma"] * r
        assert abs(got[k, 1] - own) <= 1e-5 * own, (k, got[k, 1], own)
        assert abs(got[k, 1] - rms_o) <= tol_o(precision, (n, m)) * rms_o, (k, got[k, 1], rms_o)


def test_zero_sharded_step_world_one_matches_plan():
    """ZeroMuon on an NCCL group of one rank (shard kernels, ns_orthogonalize,
    in-place gathers) equals the single-GPU plan bit for bit: both run the
    same fp32 operations on the same values."""
    import datetime
    import socket

    import torch.distributed as dist

    import muon_step_b200 as ms
    from muon_step_b200.distributed import ZeroMuon

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shapes = [(300, 500), (500, 300), (64, 64), (33, 7)]
        a = workloads.make_random(shapes, device="cuda", seed=37)
        b = workloads.make_random(shapes, device="cuda", seed=37)
        opt = ZeroMuon(shapes)
        opt.load_weights([a.W[k] for k in range(a.count)])
        for k in range(a.count):
            opt.momentum_shards[k][: a.M[k].numel()].copy_(a.M[k].reshape(-1))
        plan = ms.MuonPlan([(b.W[k], b.G[k], b.M[k]) for k in range(b.count)])
        for _ in range(2):
            for k in range(a.count):
                opt.grad(k).copy_(a.G[k])
            opt.step()
            plan.execute()
        torch.cuda.synchronize()
        assert ms.sync_status() == 0
        for k, (n, m) in enumerate(shapes):
            assert torch.equal(opt.weight(k), b.W[k]), k
            assert torch.equal(opt.momentum_shards[k][: n * m].view(n, m), b.M[k]), k
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_l2_batching_gives_identical_results(precision):
    """Batch-by-batch stage launches compute every tile as one pass does."""
    import muon_step_b200 as ms

    shapes = [(300, 520), (520, 300), (64, 64), (257, 129), (300, 520), (100, 37), (100, 100)]
    a = workloads.make_random(shapes, device="cuda", seed=41)
    b = workloads.make_random(shapes, device="cuda", seed=41)
    Oa = [torch.empty_like(w) for w in a.W]
    Ob = [torch.empty_like(w) for w in b.W]
    pa = ms.MuonPlan([(a.W[k], a.G[k], a.M[k], Oa[k]) for k in range(a.count)], precision=precision)
    pb = ms.MuonPlan([(b.W[k], b.G[k], b.M[k], Ob[k]) for k in range(b.count)], precision=precision)
    pb.set_l2_batching(1)  # one matrix per batch
    for _ in range(2):
        pa.execute()
        pb.execute()
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    for k in range(a.count):
        assert torch.equal(a.W[k], b.W[k]) and torch.equal(a.M[k], b.M[k]) and torch.equal(Oa[k], Ob[k])


MID = [(128, 512), (512, 128), (100, 300), (300, 100), (9, 500), (128, 129), (64, 512),
       (77, 333), (129, 64)]


@pytest.mark.parametrize("spectrum", ["geometric", "flat"])
def test_mid_size_kernel(spectrum):
    """min(n, m) <= 128 < max(n, m) <= 512: the one-CTA mid-size kernel, both
    orientations, ragged edges, a nine-row matrix, several steps."""
    wl = workloads.make_random(MID, device="cuda", seed=43, spectrum=spectrum)
    worst = check_step(wl, "bf16", steps=2)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE and worst["W_given_O"] <= TOL_ELEMENTWISE, worst


@pytest.mark.parametrize("scale_mode", ["unit_rms", "none"])
def test_mid_size_kernel_scale_modes(scale_mode):
    wl = workloads.make_random(MID[:4], device="cuda", seed=47)
    hyper = dict(wl.hyper, gamma=0.2 if scale_mode == "unit_rms" else 1.0)
    worst = check_step(wl, "bf16", hyper=hyper, scale_mode=scale_mode)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE and worst["W_given_O"] <= TOL_ELEMENTWISE, worst


def test_mid_size_kernel_orthogonalize():
    """ns_orthogonalize through the mid-size kernel (no weight update)."""
    rng = torch.Generator(device="cuda").manual_seed(5)
    xs = [torch.randn(n, m, generator=rng, device="cuda") for n, m in MID]
    errs = check_ns(xs, "bf16")
    assert all_within(errs), errs


def test_megatron_recipe_settings():
    """The DeepSeek-V4-Flash Megatron-Bridge recipe's Muon keys (5-step
    quintic, unit-RMS scale x 0.2, fp32 products) through the config mapper."""
    from muon_step_b200.config import from_megatron

    cfg = from_megatron(muon_momentum=0.95, muon_use_nesterov=True, muon_scale_mode="unit_rms_norm",
                        muon_fp32_matmul_prec="highest", muon_num_ns_steps=5,
                        muon_extra_scale_factor=0.2, muon_coefficient_type="quintic",
                        max_lr=2.7e-4, weight_decay=0.1)
    wl = workloads.make_random([(96, 160), (300, 200), (64, 64)], device="cuda", seed=53)
    hyper = dict(wl.hyper, lr=cfg.lr, mu=cfg.momentum, wd=cfg.weight_decay, gamma=cfg.gamma,
                 nesterov=cfg.nesterov)
    worst = check_step(wl, cfg.precision, hyper=hyper, schedule=cfg.schedule,
                       scale_mode=cfg.scale_mode)
    assert worst["O_over_tol"] <= 1.0, worst
    assert worst["M"] <= TOL_ELEMENTWISE and worst["W_given_O"] <= TOL_ELEMENTWISE, worst


def test_tracing_does_not_change_results():
    """NVTX ranges around the launches change nothing on the device."""
    import muon_step_b200 as ms

    shapes = [(300, 520), (64, 64), (100, 300)]
    a = workloads.make_random(shapes, device="cuda", seed=59)
    b = workloads.make_random(shapes, device="cuda", seed=59)
    pa = ms.MuonPlan([(a.W[k], a.G[k], a.M[k]) for k in range(a.count)])
    pb = ms.MuonPlan([(b.W[k], b.G[k], b.M[k]) for k in range(b.count)])
    ms.set_tracing(True)
    try:
        pa.execute()
    finally:
        ms.set_tracing(False)
    pb.execute()
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    for k in range(a.count):
        assert torch.equal(a.W[k], b.W[k]) and torch.equal(a.M[k], b.M[k])


@pytest.mark.parametrize("spectrum", ["geometric", "flat"])
def test_tiny_matrices_take_fp32_operands(spectrum):
    """Matrices of at most 4096 elements run with fp32 operands even in the
    bf16 precision, so they meet the fp32 bound: O' within 1e-4 of the oracle
    (both orientations, single rows and columns, 4096-element extremes, two
    consecutive steps)."""
    wl = workloads.make_random(TINY, device="cuda", seed=61, spectrum=spectrum)
    worst = check_step(wl, "bf16", steps=2)
    assert worst["O"] <= TOL_O["fp32"], worst
    assert worst["M"] <= TOL_ELEMENTWISE, worst


@pytest.mark.parametrize("scale_mode", ["shape", "unit_rms", "none"])
def test_tiny_matrices_scale_modes_and_nesterov_off(scale_mode):
    wl = workloads.make_random(TINY[:10], device="cuda", seed=67)
    hyper = dict(wl.hyper, nesterov=False, gamma=0.2 if scale_mode != "none" else 1.0)
    worst = check_step(wl, "bf16", hyper=hyper, scale_mode=scale_mode)
    assert worst["O"] <= TOL_O["fp32"], worst
    assert worst["M"] <= TOL_ELEMENTWISE and worst["W_given_O"] <= TOL_ELEMENTWISE, worst


def test_tiny_matrices_orthogonalize():
    """ns_orthogonalize of tiny matrices (no update) in the bf16 precision."""
    rng = torch.Generator(device="cuda").manual_seed(71)
    xs = [torch.randn(n, m, generator=rng, device="cuda") for n, m in TINY]
    errs = check_ns(xs, "bf16")
    assert all(e <= TOL_O["fp32"] for _, e, _ in errs), errs


def test_copy_segments_moves_every_segment():
    """The segment copy of the grouped exchanges: ragged lengths, starts that
    are not 16-byte aligned, an empty segment; bit-exact, nothing else written."""
    import ctypes

    from muon_step_b200 import _lib
    from muon_step_b200._lib import Segment

    lib = _lib.load()
    g = torch.Generator(device="cuda").manual_seed(73)
    src = torch.randn(100_003, generator=g, device="cuda")
    dst = torch.full((100_003,), -1.0, device="cuda")
    # (source offset, destination offset, elements); destinations do not overlap
    cuts = [(0, 0, 4096), (5000, 4100, 17), (9, 20000, 30000), (70001, 50001, 1),
            (1, 60000, 40000), (99999, 100002, 0), (4, 4096, 4)]
    want = dst.clone()
    for so, do, n in cuts:
        want[do:do + n] = src[so:so + n]
    segs = (Segment * len(cuts))(*[Segment(dst.data_ptr() + 4 * do, src.data_ptr() + 4 * so, n)
                                    for so, do, n in cuts])
    nbytes = ctypes.c_size_t()
    assert lib.muon_shard_workspace_size(len(cuts), ctypes.byref(nbytes)) == 0
    ws = torch.empty(nbytes.value, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.muon_copy_segments(segs, len(cuts), ws.data_ptr(), ws.numel(), stream) == 0
    torch.cuda.synchronize()
    assert torch.equal(dst, want)


def test_dependency_wait_timeout_is_reported_and_the_context_survives():
    """The chained launch's dependency wait, on a counter nothing advances,
    gives up after its limit and reports MUON_ERR_TIMEOUT; the same wait on a
    counter that has reached its target passes; the library still runs."""
    import muon_step_b200 as ms
    counter = torch.zeros(1, dtype=torch.int32, device="cuda")
    ms.dep_wait_probe(counter, 16, 2_000_000)  # 2 ms, the signal is withheld
    assert ms.sync_status() == 5                # MUON_ERR_TIMEOUT
    assert ms.sync_status() == 0
    counter.fill_(16)
    ms.dep_wait_probe(counter, 16, 2_000_000)
    assert ms.sync_status() == 0
    wl = workloads.make_random([(300, 520)], device="cuda", seed=2)
    assert check_step(wl, "bf16")["O_over_tol"] <= 1.0


CHAIN_SHAPES = [(300, 520), (520, 300), (257, 129), (1000, 300), (600, 600), (1024, 1024),
                (64, 64), (100, 120), (300, 520)]


@pytest.mark.parametrize("scale_mode", ["shape", "unit_rms", "none"])
@pytest.mark.parametrize("window", [0, 1, 50])
def test_chained_launch_is_bit_identical_to_stagewise(scale_mode, window):
    """Every Newton-Schulz stage in one chained launch (per-matrix dependency
    counters, a window of matrices in flight) gives the same bits as one
    launch per stage: W, M, O' and the diagnostics, over two steps."""
    import muon_step_b200 as ms

    a = workloads.make_random(CHAIN_SHAPES, device="cuda", seed=79)
    b = workloads.make_random(CHAIN_SHAPES, device="cuda", seed=79)
    Oa = [torch.empty_like(w) for w in a.W]
    Ob = [torch.empty_like(w) for w in b.W]
    pa = ms.MuonPlan([(a.W[k], a.G[k], a.M[k], Oa[k]) for k in range(a.count)], scale_mode=scale_mode)
    pb = ms.MuonPlan([(b.W[k], b.G[k], b.M[k], Ob[k]) for k in range(b.count)], scale_mode=scale_mode)
    pa.set_chaining(True, window)
    pb.set_chaining(False)
    da = torch.zeros((a.count, 2), device="cuda")
    db = torch.zeros((b.count, 2), device="cuda")
    pa.set_diagnostics(da)
    pb.set_diagnostics(db)
    assert 10 in pa.launches() and 10 not in pb.launches()
    for _ in range(2):
        pa.execute()
        pb.execute()
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    for k in range(a.count):
        assert torch.equal(a.W[k], b.W[k]), k
        assert torch.equal(a.M[k], b.M[k]), k
        assert torch.equal(Oa[k], Ob[k]), k
    assert torch.equal(da, db)


def test_chained_orthogonalize_matches_stagewise():
    import muon_step_b200 as ms

    rng = torch.Generator(device="cuda").manual_seed(83)
    xs = [torch.randn(n, m, generator=rng, device="cuda") for n, m in CHAIN_SHAPES]
    outs = []
    for chain in (True, False):
        o = [torch.empty_like(x) for x in xs]
        plan = ms.NsPlan(list(zip(xs, o)))
        plan.set_chaining(chain)
        plan.execute()
        outs.append(o)
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    for oa, ob in zip(*outs):
        assert torch.equal(oa, ob)


def test_chained_launch_beside_work_on_another_stream():
    """The chained launch's CTA pairs take tiles from a shared counter as they
    become free, so matrix products running on another stream when it starts
    (holding SMs it would use) only delay it: no timeout, and the same bits
    as the per-stage launches on an otherwise idle GPU."""
    import muon_step_b200 as ms

    shapes = [(1024, 1024)] * 6 + [(512, 2048), (2048, 512), (600, 600)]
    a = workloads.make_random(shapes, device="cuda", seed=89)
    b = workloads.make_random(shapes, device="cuda", seed=89)
    pa = ms.MuonPlan([(a.W[k], a.G[k], a.M[k]) for k in range(a.count)])
    pb = ms.MuonPlan([(b.W[k], b.G[k], b.M[k]) for k in range(b.count)])
    pa.set_chaining(True)
    pb.set_chaining(False)
    wa = pa.alloc_workspace()
    x = torch.randn(8192, 8192, device="cuda", dtype=torch.bfloat16)
    other = torch.cuda.Stream()
    mine = torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(3):
        with torch.cuda.stream(other):
            for _ in range(8):
                y = x @ x
        pa.execute(wa, stream=mine)
        pb.execute()
    torch.cuda.synchronize()
    del y
    assert ms.sync_status() == 0
    for k in range(a.count):
        assert torch.equal(a.W[k], b.W[k]), k
        assert torch.equal(a.M[k], b.M[k]), k
