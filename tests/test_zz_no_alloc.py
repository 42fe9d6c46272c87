"""The Muon step for callers that cannot allocate device memory.

muon_step_static_scratch runs the same step as muon_step, with the library's
own fixed device array as scratch instead of a caller workspace. It is meant
for runtimes that own all of HBM, code that cannot afford the synchronisation
of cudaMalloc / cudaFree, and plugins without an allocator. This test calls
both entry points through the C ABI on identical copies of the inputs, twice
in a row (the second call reuses the array the first one left behind), and
checks that the outputs agree within the parity tolerances. It runs last
(file name), and also passes on its own in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

import workloads
from muon_step_b200 import _lib
from muon_step_b200._lib import MUON_ERR_WORKSPACE, MUON_NS_BF16, MUON_OK, MuonParam
from tests.parity import TOL_ELEMENTWISE, rel, tol_o

pytestmark = pytest.mark.gpu

SHAPES = [(256, 512), (300, 200), (64, 64), (5, 3)]


def _params(ws_tensors):
    arr = (MuonParam * len(ws_tensors))()
    for k, (W, G, M, O) in enumerate(ws_tensors):
        arr[k] = MuonParam(W.data_ptr(), G.data_ptr(), M.data_ptr(), O.data_ptr(), *W.shape)
    return arr


def test_static_scratch_matches_muon_step_twice():
    assert torch.cuda.is_available()
    lib = _lib.load()
    wl = workloads.make_random(SHAPES, device="cuda", seed=21)
    h = wl.hyper
    ref = [(wl.W[k].clone(), wl.G[k], wl.M[k].clone(), torch.empty_like(wl.W[k]))
           for k in range(wl.count)]
    new = [(wl.W[k].clone(), wl.G[k], wl.M[k].clone(), torch.zeros_like(wl.W[k]))
           for k in range(wl.count)]
    p_ref, p_new = _params(ref), _params(new)
    n = ctypes.c_size_t()
    assert lib.muon_workspace_size(p_ref, len(ref), MUON_NS_BF16, ctypes.byref(n)) == MUON_OK
    assert n.value <= _lib.MUON_STATIC_SCRATCH_BYTES
    ws = torch.empty(n.value, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        st = lib.muon_step(p_ref, len(ref), h["lr"], h["mu"], h["wd"], h["gamma"], 1, None,
                           MUON_NS_BF16, ws.data_ptr(), ws.numel(), stream)
        assert st == MUON_OK
        st = lib.muon_step_static_scratch(p_new, len(new), h["lr"], h["mu"], h["wd"], h["gamma"],
                                          1, None, MUON_NS_BF16, stream)
        assert st == MUON_OK
        assert lib.muon_sync_status(stream) == MUON_OK
        for (Wr, _, Mr, Or), (Wn, _, Mn, On) in zip(ref, new):
            shape = tuple(Wr.shape)
            assert rel(On.double().cpu().numpy(), Or.double().cpu().numpy()) <= tol_o("bf16", shape)
            assert rel(Mn.double().cpu().numpy(), Mr.double().cpu().numpy()) <= TOL_ELEMENTWISE
            assert rel(Wn.double().cpu().numpy(), Wr.double().cpu().numpy()) <= TOL_ELEMENTWISE


def test_static_scratch_rejects_oversized_steps():
    lib = _lib.load()
    # 4096 x 4096 needs about 200 MB of scratch: refused before any device work
    big = (MuonParam * 1)(MuonParam(0x10000, 0x20000, 0x30000, None, 4096, 4096))
    st = lib.muon_step_static_scratch(big, 1, 0.02, 0.95, 0.1, 0.2, 1, None, MUON_NS_BF16, None)
    assert st == MUON_ERR_WORKSPACE
