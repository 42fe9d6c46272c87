"""Argument checks of the Python binding: the workspace is passed with its
size in bytes and must sit on the matrices' device, and every tensor of one
call must share a device. (The CUDA-only checks run in the GPU test below.)"""

import pytest
import torch

import muon_step_b200 as ms


def test_workspace_size_is_in_bytes_and_cpu_tensors_are_rejected():
    with pytest.raises(TypeError):
        ms._workspace(torch.empty(16, dtype=torch.uint8), torch.device("cpu"))
    with pytest.raises(TypeError):
        ms._workspace("not a tensor", torch.device("cuda", 0))


def test_one_device():
    a = torch.empty(2)
    b = torch.empty(2, device="meta")
    assert ms._one_device([a, None, a]) == torch.device("cpu")
    with pytest.raises(ValueError):
        ms._one_device([a, b])
    with pytest.raises(ValueError):
        ms._one_device([])


@pytest.mark.gpu
def test_binding_checks_on_gpu():
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(3)
    X = torch.randn(48, 80, device=dev, generator=g)
    # a caller's out must have the input's shape and be float32
    with pytest.raises(ValueError):
        ms.ns_orthogonalize([X], out=[torch.empty(80, 48, device=dev)])
    with pytest.raises(TypeError):
        ms.ns_orthogonalize([X], out=[torch.empty(48, 80, device=dev, dtype=torch.float64)])
    W, G, M = (torch.randn(48, 80, device=dev, generator=g) for _ in range(3))
    with pytest.raises(TypeError):
        ms.muon_step([(W, G, M, torch.empty(48, 80, device=dev, dtype=torch.float16))])
    with pytest.raises(TypeError):
        ms.MuonPlan([(W, G, M)]).execute(torch.empty(4096, dtype=torch.uint8))  # host workspace
    # any workspace dtype: its size counts in bytes, results are the same
    W2, M2 = W.clone(), M.clone()
    plan = ms.MuonPlan([(W, G, M)])
    plan.execute(plan.alloc_workspace())
    plan2 = ms.MuonPlan([(W2, G, M2)])
    ws32 = torch.empty((plan2.workspace_bytes + 3) // 4, dtype=torch.float32, device=dev)
    plan2.execute(ws32)
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    assert torch.equal(W, W2) and torch.equal(M, M2)
