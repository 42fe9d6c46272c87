"""Multi-rank host logic on CPU ranks (gloo, world size 2 and 3): the
benchmark's job-wide aggregation, the ownership partition, and the
distributed step's exchange (with the float64 oracle as each rank's compute,
so no GPU is needed)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from muon_step_b200.distributed import DistributedMuon, ns_cost, partition


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(world, fn, *args):
    port = _free_port()
    mp.spawn(_entry, args=(world, port, fn, args), nprocs=world, join=True)


def _entry(rank, world, port, fn, args):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        fn(rank, world, *args)
    finally:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------ partition

def test_partition_covers_and_balances():
    shapes = [(4096, 4096)] * 4 + [(4096, 14336)] * 3 + [(128, 128)] * 10 + [(14336, 4096)]
    for world in (1, 2, 3, 8):
        owner = partition(shapes, world)
        assert len(owner) == len(shapes) and set(owner) <= set(range(world))
        assert owner == partition(shapes, world)  # deterministic
        load = [sum(ns_cost(s) for s, o in zip(shapes, owner) if o == r) for r in range(world)]
        # greedy largest-first: no rank exceeds the average by more than the largest item
        assert max(load) <= sum(load) / world + max(ns_cost(s) for s in shapes)


def test_partition_single_rank_owns_all():
    assert partition([(3, 5), (7, 2)], 1) == [0, 0]


# ------------------------------------------------------------ bench aggregation

def _agg(rank, world, out_dir):
    ms = [12.5, 30.25, 7.0][rank]
    got = bench.max_over_ranks(ms, "cpu", world)
    with open(os.path.join(out_dir, f"r{rank}"), "w") as f:
        f.write(repr(got))


@pytest.mark.parametrize("world", [2, 3])
def test_bench_max_over_ranks(tmp_path, world):
    _run(world, _agg, str(tmp_path))
    want = max([12.5, 30.25, 7.0][:world])
    for r in range(world):
        assert float(open(tmp_path / f"r{r}").read()) == want
    # FLOPs of all ranks over the slowest rank's time
    assert bench.job_tflops(1e12, world, 10, 2000.0) == pytest.approx(world * 5.0)


# ------------------------------------------------------------ distributed step

SHAPES = [(24, 40), (40, 24), (16, 16), (33, 17), (8, 64), (64, 8), (5, 5)]
HYPER = dict(lr=0.02, momentum=0.95, weight_decay=0.1, gamma=0.2, nesterov=True)


def _inputs(seed=0):
    g = torch.Generator().manual_seed(seed)
    out = []
    for n, m in SHAPES:
        out.append(tuple(torch.randn(n, m, generator=g, dtype=torch.float32) for _ in range(3)))
    return out


def _oracle_compute(params):
    from oracle import muon_oracle

    def compute(owned, hyper):
        for k in owned:
            W, G, M = params[k]
            W_new, M_new, _ = muon_oracle.muon_step(
                W.double().numpy(), G.double().numpy(), M.double().numpy(), lr=hyper["lr"],
                mu=hyper["momentum"], wd=hyper["weight_decay"], gamma=hyper["gamma"],
                nesterov_on=hyper["nesterov"])
            W.copy_(torch.from_numpy(W_new).float())
            M.copy_(torch.from_numpy(M_new).float())
    return compute


def _dist_step(rank, world, out_dir):
    params = [(W.clone(), G.clone(), M.clone()) for W, G, M in _inputs()]
    opt = DistributedMuon(params, compute=_oracle_compute(params))
    opt.step(**HYPER)
    opt.step(**HYPER)
    torch.save({"W": [p[0] for p in params], "M": [p[2] for p in params], "owner": opt.owner},
               os.path.join(out_dir, f"r{rank}.pt"))


@pytest.mark.parametrize("world", [2, 3])
def test_distributed_step_matches_single_process(tmp_path, world):
    _run(world, _dist_step, str(tmp_path))
    # single process: every matrix stepped twice by the same compute
    ref = [(W.clone(), G.clone(), M.clone()) for W, G, M in _inputs()]
    comp = _oracle_compute(ref)
    comp(list(range(len(ref))), HYPER)
    comp(list(range(len(ref))), HYPER)
    outs = [torch.load(tmp_path / f"r{r}.pt") for r in range(world)]
    owner = outs[0]["owner"]
    assert len(set(owner)) == min(world, len(SHAPES))
    for r, out in enumerate(outs):
        for k in range(len(SHAPES)):
            # weights: identical on every rank, equal to the single-process result
            assert torch.equal(out["W"][k], outs[0]["W"][k])
            assert torch.equal(out["W"][k], ref[k][0])
            # momentum: advanced by the owner only
            if owner[k] == r:
                assert torch.equal(out["M"][k], ref[k][2])
            else:
                assert torch.equal(out["M"][k], _inputs()[k][2])
