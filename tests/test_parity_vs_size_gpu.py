"""O' error against matrix size, on every workload's shapes.

Each workload is cut to one unit (two matrices of a sweep point or of the
64 x 1024^2 batch, one layer of the d = 4096 stack, one expert of the MoE
bank): the error is a property of each matrix, and the seeded generators
give the same matrices in the cut workload. One step runs through the
library in bf16 and, from the same state, in fp32; both are compared with one
float64 oracle step ("Muon 优化器完全拆解…", Algorithm 1). The test asserts
the tolerances and prints one line per matrix; run it with -s to read the
table:

    python -m pytest tests/test_parity_vs_size_gpu.py -m gpu -s -q
"""

import pytest

import workloads
from oracle import muon_oracle
from tests.parity import rel, run_step, tol_o

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

POINTS = ([("single_256x512", {}, (0,)),
           ("batch64_1024", {"count": 2}, (0,)),
           ("dense_d4096", {"layers": 1}, (0, 6)),   # Q 4096^2; down 14336 x 4096 (transposed)
           ("moe_64x3", {"experts": 1}, (0, 2))]     # gate 2048 x 7168; down 7168 x 2048
          + [(f"sweep_{b}_{a}", {"count": 2}, (0,)) for b in (128, 512, 2048)
             for a in ("1x1", "1x4", "4x1")])


@pytest.mark.parametrize("name,kw,sample", POINTS, ids=[p[0] for p in POINTS])
def test_o_error_vs_size(name, kw, sample):
    wl = workloads.make(name, device="cuda", **kw)
    W0 = [wl.W[k].clone() for k in range(wl.count)]
    M0 = [wl.M[k].clone() for k in range(wl.count)]
    out = {}
    for precision in ("bf16", "fp32"):
        for k in range(wl.count):
            wl.W[k].copy_(W0[k])
            wl.M[k].copy_(M0[k])
        before, _after, history, h = run_step(wl, precision, sample=list(sample))
        out[precision] = history[0]
    for k in sample:
        W, G, M = before[k]
        n, m = W.shape
        _, _, O_ref = muon_oracle.muon_step(W, G, M, lr=h["lr"], mu=h["mu"], wd=h["wd"],
                                            gamma=h["gamma"], nesterov_on=h["nesterov"],
                                            schedule=muon_oracle.HYBRID_SCHEDULE)
        err = {p: rel(out[p][k], O_ref) for p in out}
        print(f"\nO' error {name} #{k} {n}x{m}: bf16 {err['bf16']:.3e}  fp32 {err['fp32']:.3e}")
        for p, e in err.items():
            assert e <= tol_o(p, (n, m)), (p, n, m, e)
