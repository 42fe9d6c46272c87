"""The seeded input generators draw what the input recipe states (shapes,
scales, spectra), and the same seed gives the same bytes. Small instances of
each recipe, on the CPU."""

import math

import numpy as np
import pytest

import workloads
from workloads import synth


def _sv(t):
    return np.linalg.svd(t.double().numpy(), compute_uv=False)


def test_single_256x512():
    wl = workloads.make("single_256x512")
    assert wl.shapes == [(256, 512)]
    assert float(wl.W[0].std()) == pytest.approx(0.02, rel=0.02)
    assert float(wl.M[0].std()) == pytest.approx(0.01, rel=0.02)   # variance 1e-4
    s = _sv(wl.G[0])
    # 16 rank-one terms a b^T / sqrt(512), weights 10^(-3(k-1)/15): about three decades
    assert 200.0 < s[0] / s[15] < 5000.0
    # then the 1e-4 N(0, 1) noise, whose spectral edge is 1e-4 (sqrt(256) + sqrt(512))
    assert s[16] < 1.5e-4 * (16 + math.sqrt(512))


def test_batch_lowrank_plus_noise():
    wl = synth.make_batch64_1024(count=2, size=256)
    assert wl.shapes == [(256, 256)] * 2
    s = _sv(wl.G[1])
    assert s[0] == pytest.approx(1.0, abs=0.01)           # top of the geometric 1 -> 1e-3 spectrum
    sig = np.logspace(0, -3, 64)
    above = int((sig > 0.02).sum())                        # well above the noise edge 3.2e-3
    assert abs(int((s > 0.02).sum()) - above) <= 1
    assert s[64] < 1.5e-4 * 32                             # the 1e-4 noise beyond rank 64


def test_dense_spike_over_noise():
    wl = synth.make_dense_d4096(layers=1, d=64, ffn=224)
    assert wl.shapes == [(64, 64)] * 4 + [(64, 224)] * 2 + [(224, 64)]
    n, m = 64, 224
    s = _sv(wl.G[4])
    s_min = 1e-3 * (math.sqrt(n) + math.sqrt(m))           # the noise's spectral edge
    assert s[0] == pytest.approx(1e3 * s_min, rel=0.02)    # rank-32 spike over three decades
    assert s[31] < 3.0 * s_min and s[40] < 1.5 * s_min


def test_moe_scaled_full_rank():
    wl = synth.make_moe_64x3(experts=2, d=32, f=112)
    assert wl.shapes == [(32, 112), (32, 112), (112, 32)] * 2
    for G in wl.G:
        s = _sv(G)
        assert 1e-4 * 0.999 <= s[0] <= 1e-1 * 1.001        # expert scale, log-uniform in [1e-4, 1e-1]
        assert s[0] / s[-1] == pytest.approx(1e4, rel=0.01)   # geometric over four decades


@pytest.mark.parametrize("aspect,shape", [("1x1", (128, 128)), ("1x4", (128, 512)),
                                          ("4x1", (512, 128))])
def test_sweep_full_rank_bases(aspect, shape):
    wl = synth.make_sweep(128, aspect, count=1)
    assert wl.shapes == [shape]
    s = _sv(wl.G[0])
    assert len(s) == 128
    assert s[0] == pytest.approx(1.0, rel=1e-3) and s[-1] == pytest.approx(1e-4, rel=1e-2)


def test_sweep_large_base_is_rank_64_plus_noise():
    wl = synth.make_sweep(2048, "1x1", count=1)
    s = _sv(wl.G[0])
    assert s[0] == pytest.approx(1.0, rel=1e-3)
    # noise N(0, (1e-4 / sqrt(c))^2): spectral edge 1e-4 (sqrt(r) + sqrt(c)) / sqrt(c) = 2e-4,
    # next to the tail of the rank-64 spectrum
    assert s[64] < 2.2e-4 and s[70] < 2.1e-4
    assert s[40] > 1e-3


def test_batch_sizes_of_the_sweep():
    # about 16 GB of fp32 W, M, G per point
    assert synth.sweep_batch(128, 128) == 81380
    assert synth.sweep_batch(128, 512) == 20345
    assert synth.sweep_batch(16384, 65536) == 1


def test_same_seed_same_bytes():
    a = workloads.make("single_256x512")
    b = workloads.make("single_256x512")
    for x, y in zip(a.W + a.G + a.M, b.W + b.G + b.M):
        assert x.numpy().tobytes() == y.numpy().tobytes()
    c = synth.make_sweep(128, "1x1", seed=6, count=1)
    assert c.G[0].numpy().tobytes() != synth.make_sweep(128, "1x1", count=1).G[0].numpy().tobytes()
