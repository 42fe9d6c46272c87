"""The Muon step for callers that cannot allocate device memory.

muon_step_static_scratch runs the same step as muon_step, with the library's
own fixed device array as scratch instead of a caller workspace. It is meant
for runtimes that own all of HBM, code that cannot afford the synchronisation
of cudaMalloc / cudaFree, and plugins without an allocator. These tests call
both entry points through the C ABI on identical copies of the inputs, twice
in a row (the second call reuses the array the first one left behind), and
check that W, M and O' agree bit for bit: both run the same deterministic
kernels on the same values, so any difference would be a scratch-reuse bug.
One case needs nearly all of the array, where the descriptor tables and the
per-matrix partial sums sit at their largest offsets. The file runs last
(file name), and also passes on its own in a fresh process.
"""

import ctypes

import pytest
import torch

import workloads
from muon_step_b200 import _lib
from muon_step_b200._lib import MUON_ERR_WORKSPACE, MUON_NS_BF16, MUON_NS_FP32, MUON_OK, MuonParam

pytestmark = pytest.mark.gpu

SHAPES = [(256, 512), (300, 200), (64, 64), (5, 3), (100, 120), (129, 400)]
FAKE = 0x10000  # plan creation records pointers but never dereferences them


def _params(ws_tensors):
    arr = (MuonParam * len(ws_tensors))()
    for k, (W, G, M, O) in enumerate(ws_tensors):
        arr[k] = MuonParam(W.data_ptr(), G.data_ptr(), M.data_ptr(), O.data_ptr(), *W.shape)
    return arr


def _run_both_twice(shapes, prec, seed):
    lib = _lib.load()
    wl = workloads.make_random(shapes, device="cuda", seed=seed)
    h = wl.hyper
    ref = [(wl.W[k].clone(), wl.G[k], wl.M[k].clone(), torch.empty_like(wl.W[k]))
           for k in range(wl.count)]
    new = [(wl.W[k].clone(), wl.G[k], wl.M[k].clone(), torch.zeros_like(wl.W[k]))
           for k in range(wl.count)]
    p_ref, p_new = _params(ref), _params(new)
    n = ctypes.c_size_t()
    assert lib.muon_workspace_size(p_ref, len(ref), prec, ctypes.byref(n)) == MUON_OK
    assert n.value <= _lib.MUON_STATIC_SCRATCH_BYTES
    ws = torch.empty(n.value, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        st = lib.muon_step(p_ref, len(ref), h["lr"], h["mu"], h["wd"], h["gamma"], 1, None,
                           prec, ws.data_ptr(), ws.numel(), stream)
        assert st == MUON_OK
        st = lib.muon_step_static_scratch(p_new, len(new), h["lr"], h["mu"], h["wd"], h["gamma"],
                                          1, None, prec, stream)
        assert st == MUON_OK
        assert lib.muon_sync_status(stream) == MUON_OK
        for k, ((Wr, _, Mr, Or), (Wn, _, Mn, On)) in enumerate(zip(ref, new)):
            assert torch.equal(On, Or), (call, k, "O'")
            assert torch.equal(Mn, Mr), (call, k, "M")
            assert torch.equal(Wn, Wr), (call, k, "W")
    return n.value


@pytest.mark.parametrize("prec", [MUON_NS_BF16, MUON_NS_FP32])
def test_static_scratch_matches_muon_step_twice(prec):
    assert torch.cuda.is_available()
    _run_both_twice(SHAPES, prec, seed=21)


def test_static_scratch_near_its_limit():
    """One 1024 x c matrix with c as large as the array allows."""
    lib = _lib.load()

    def need(c):
        p = (MuonParam * 1)(MuonParam(FAKE, 2 * FAKE, 3 * FAKE, None, 1024, c))
        n = ctypes.c_size_t()
        assert lib.muon_workspace_size(p, 1, MUON_NS_BF16, ctypes.byref(n)) == MUON_OK
        return n.value

    lo, hi = 1024, 65536
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if need(mid) <= _lib.MUON_STATIC_SCRATCH_BYTES else (lo, mid)
    assert need(lo) > 0.95 * _lib.MUON_STATIC_SCRATCH_BYTES
    used = _run_both_twice([(1024, lo)], MUON_NS_BF16, seed=22)
    assert used == need(lo)


def test_static_scratch_rejects_oversized_steps():
    lib = _lib.load()
    # 4096 x 4096 needs about 200 MB of scratch: refused before any device work
    big = (MuonParam * 1)(MuonParam(FAKE, 2 * FAKE, 3 * FAKE, None, 4096, 4096))
    st = lib.muon_step_static_scratch(big, 1, 0.02, 0.95, 0.1, 0.2, 1, None, MUON_NS_BF16, None)
    assert st == MUON_ERR_WORKSPACE
