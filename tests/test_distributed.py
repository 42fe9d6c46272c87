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
    opt = DistributedMuon(params, compute=_oracle_compute(params), copier=TorchCopier())
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


# ------------------------------------------------------------ ZeRO-sharded step

def _zero_kernels():
    """CPU stand-ins of the library calls, written with the float64 oracle."""
    from oracle import muon_oracle

    class K:
        def momentum(self, items, mu, nesterov):
            for M, G, N in items:
                Mn = muon_oracle.momentum(M.double().numpy(), G.double().numpy(), mu)
                Nn = muon_oracle.nesterov(Mn, G.double().numpy(), mu) if nesterov else Mn
                M.copy_(torch.from_numpy(Mn))
                N.copy_(torch.from_numpy(Nn))

        def orthogonalize(self, pairs, precision, schedule, eps):
            for X, O in pairs:
                O.copy_(torch.from_numpy(muon_oracle.ns_orthogonalize(X.double().numpy())))

        def update(self, items, lr, wd, gamma):
            for W, O, (n, m) in items:
                On = muon_oracle.rescale(O.double().numpy(), n, m, gamma)
                W.copy_(torch.from_numpy(muon_oracle.decay_and_update(W.double().numpy(), On, lr, wd)))

        def prepare_copy(self, pairs):
            return TorchCopier().prepare(pairs)

    return K()


class TorchCopier:
    """CPU stand-in of the library's segment copy (host logic of the exchanges)."""

    def prepare(self, pairs):
        pairs = list(pairs)

        def run():
            for d, s in pairs:
                d.copy_(s)
        return run


def _zero_step(rank, world, out_dir):
    from muon_step_b200.distributed import ZeroMuon

    opt = ZeroMuon(SHAPES, device="cpu", kernels=_zero_kernels())
    opt.load_weights([W for W, _, _ in _inputs()])
    for step in range(2):
        grads = _inputs(seed=100 + 10 * step + rank)  # each rank its own local gradient
        for k in range(len(SHAPES)):
            opt.grad(k).copy_(grads[k][1])
        opt.step(**HYPER)
    torch.save({"W": [opt.weight(k).clone() for k in range(len(SHAPES))],
                "M": [s.clone() for s in opt.momentum_shards]},
               os.path.join(out_dir, f"z{rank}.pt"))


@pytest.mark.parametrize("world", [2, 3])
def test_zero_sharded_step_matches_the_oracle(tmp_path, world):
    """Reduce-scatter, shard momentum, gather, Newton-Schulz, shard update and
    all-gather over gloo ranks equal the oracle's step on the summed gradient;
    every rank ends with the same weights; the momentum shards tile the
    oracle's momentum."""
    from muon_step_b200.distributed import shard_size
    from oracle import muon_oracle

    _run(world, _zero_step, str(tmp_path))
    outs = [torch.load(tmp_path / f"z{r}.pt") for r in range(world)]
    W = [w.double().numpy() for w, _, _ in _inputs()]
    M = [np.zeros(s) for s in SHAPES]
    for step in range(2):
        G = [sum(_inputs(seed=100 + 10 * step + r)[k][1].double().numpy() for r in range(world))
             for k in range(len(SHAPES))]
        for k in range(len(SHAPES)):
            W[k], M[k], _ = muon_oracle.muon_step(W[k], G[k], M[k], lr=HYPER["lr"],
                                                  mu=HYPER["momentum"], wd=HYPER["weight_decay"],
                                                  gamma=HYPER["gamma"])
    for k, (n, m) in enumerate(SHAPES):
        for out in outs:
            assert torch.equal(out["W"][k], outs[0]["W"][k])
        # float32 buffers between the float64 pieces
        assert np.abs(outs[0]["W"][k].double().numpy() - W[k]).max() <= 1e-6 * np.abs(W[k]).max()
        s = shard_size(n * m, world)
        flat = torch.cat([outs[r]["M"][k] for r in range(world)])
        assert flat.numel() == s * world
        assert np.abs(flat[: n * m].double().numpy() - M[k].reshape(-1)).max() <= 1e-6 * np.abs(M[k]).max()
        assert not flat[n * m:].any()  # padding stays zero


def test_shard_sizes():
    from muon_step_b200.distributed import shard_size
    for numel in (1, 3, 4, 5, 1000, 4096, 12345):
        for world in (1, 2, 3, 8):
            s = shard_size(numel, world)
            assert s % 4 == 0 and s * world >= numel and (s - 4) * world < numel
