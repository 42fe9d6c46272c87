"""Host-side checks of the C ABI: the library loads and exports every symbol
the header declares; planning (host only) validates arguments, sizes the
workspace and counts tiles and FLOPs; no call here touches a GPU."""

import ctypes
import math
import os
import re

import pytest

from muon_step_b200 import _lib
from muon_step_b200._lib import (MUON_ERR_INVALID_ARG, MUON_ERR_WORKSPACE, MUON_NS_BF16,
                                 MUON_NS_FP32, MUON_OK, MuonHyper, MuonNsMatrix, MuonNsSchedule,
                                 MuonParam)

TINY = 4096  # matrices of at most this many elements take the tiny fp32 kernel (bf16 precision)
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
                 if f.endswith(".h"))


@pytest.fixture(scope="module")
def lib():
    from muon_step_b200 import build
    build.build()
    return _lib.load()


def header_symbols():
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"^MUON_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_exports():
    assert header_symbols() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name


def test_no_other_exported_api_symbols(lib):
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    api = {s for s in exported if s.startswith(("muon_", "ns_"))}
    assert api == set(header_symbols())


def test_version_and_status_strings(lib):
    assert lib.muon_abi_version() == 1
    for s in range(6):
        assert lib.muon_status_string(s)
    assert lib.muon_status_string(99) == b"unknown status"


FAKE = 0x10000  # plan creation records pointers but never dereferences them


def params(shapes, with_o=False):
    arr = (MuonParam * len(shapes))()
    for k, (n, m) in enumerate(shapes):
        base = FAKE * (4 * k + 1)
        arr[k] = MuonParam(base, base + 1 * FAKE, base + 2 * FAKE, base + 3 * FAKE if with_o else None, n, m)
    return arr


def create(lib, shapes, prec=MUON_NS_BF16, sched=None):
    plan = ctypes.c_void_p()
    st = lib.muon_plan_create(params(shapes), len(shapes), prec, sched, ctypes.byref(plan))
    return st, plan


def test_plan_rejects_bad_arguments(lib):
    plan = ctypes.c_void_p()
    assert lib.muon_plan_create(None, 1, 0, None, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    assert lib.muon_plan_create(params([(4, 4)]), 0, 0, None, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    assert lib.muon_plan_create(params([(4, 4)]), 1, 7, None, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    assert lib.muon_plan_create(params([(0, 4)]), 1, 0, None, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    assert lib.muon_plan_create(params([(4, -1)]), 1, 0, None, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    # a side above 2^31 - 8 would overflow the 32-bit leading dimension
    for shape in [(1, 2 ** 31 - 7), (2 ** 31 - 1, 1), (1, 2 ** 40)]:
        assert lib.muon_plan_create(params([shape]), 1, 0, None, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    bad = params([(4, 4)])
    bad[0].G = None
    assert lib.muon_plan_create(bad, 1, 0, None, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG
    assert lib.muon_plan_create(params([(4, 4)]), 1, 0, None, None) == MUON_ERR_INVALID_ARG
    # schedules: zero steps, too many steps, eps <= 0, NaN coefficient
    abc = (ctypes.c_float * 6)(1, 0, 0, 1, 0, 0)
    p = ctypes.cast(abc, ctypes.POINTER(ctypes.c_float))
    for s in (MuonNsSchedule(0, p, 1e-7), MuonNsSchedule(65, p, 1e-7), MuonNsSchedule(2, p, 0.0),
              MuonNsSchedule(2, None, 1e-7)):
        assert create(lib, [(4, 4)], sched=ctypes.byref(s))[0] == MUON_ERR_INVALID_ARG
    abc[4] = float("nan")
    assert create(lib, [(4, 4)], sched=ctypes.byref(MuonNsSchedule(2, p, 1e-7)))[0] == MUON_ERR_INVALID_ARG


def test_execute_rejects_bad_workspace_without_touching_the_device(lib):
    st, plan = create(lib, [(64, 96)])
    assert st == MUON_OK
    try:
        n = ctypes.c_size_t()
        lib.muon_plan_workspace_size(plan, ctypes.byref(n))
        h = MuonHyper(0.02, 0.95, 0.1, 0.2, 1)
        assert lib.muon_plan_execute(plan, ctypes.byref(h), None, n.value, None) == MUON_ERR_WORKSPACE
        assert lib.muon_plan_execute(plan, ctypes.byref(h), FAKE + 128, n.value, None) == MUON_ERR_WORKSPACE
        assert lib.muon_plan_execute(plan, ctypes.byref(h), FAKE, n.value - 1, None) == MUON_ERR_WORKSPACE
        assert lib.muon_plan_execute(plan, None, FAKE, n.value, None) == MUON_ERR_INVALID_ARG
        nan = MuonHyper(float("nan"), 0.95, 0.1, 0.2, 1)
        assert lib.muon_plan_execute(plan, ctypes.byref(nan), FAKE, n.value, None) == MUON_ERR_INVALID_ARG
    finally:
        lib.muon_plan_destroy(plan)


def syrk_tiles(r):
    rb = math.ceil(r / 128)
    return sum(i // 2 + 1 for i in range(rb))


def expected_workspace(shapes, prec):
    """Independent restatement of the documented layout: per shape group an
    fp32 iterate (two in fp32 mode), two bf16 iterates (bf16 mode), A and B;
    rows padded to multiples of 8 elements; regions 1024-byte aligned."""
    groups, order = {}, []
    for n, m in shapes:
        key = (min(n, m), max(n, m))
        if key not in groups:
            order.append(key)
        groups.setdefault(key, []).append((n, m))
    al = lambda x, a: (x + a - 1) // a * a
    ng, nm = len(groups), len(shapes)
    ew = sum(math.ceil(n / 64) * math.ceil(m / 128) for n, m in shapes)
    off = al(ng * 160, 256)          # GroupDesc is 160 bytes
    off = al(off + nm * 88, 256)     # MatDesc is 88 bytes
    off = al(off + (ng * 13 * 128 if prec == MUON_NS_BF16 else 0), 256)
    off = al(off + (nm * 2 * 128 if prec == MUON_NS_BF16 else 0), 256)
    off = al(off + ew * 4, 256)     # matrix of each elementwise tile
    tc = prec == MUON_NS_BF16
    small = [(n, m) for n, m in shapes if tc and n * m > TINY and max(n, m) <= 128]
    off = al(off + len(small) * 4, 256)  # small-matrix list
    mid = [(n, m) for n, m in shapes if tc and n * m > TINY and min(n, m) <= 128 < max(n, m) <= 512]
    off = al(off + len(mid) * 4, 256)  # mid-size list
    tiny = [(n, m) for n, m in shapes if tc and n * m <= TINY]
    off = al(off + len(tiny) * 4, 256)  # tiny-matrix list
    off = al(off + ew * 4, 256)     # partial sums
    off = al(off + nm * 4, 256)
    off = al(off + nm * 4, 256)
    # unit-RMS scale: sums of squares per Apply tile (16 slots on tensor cores), a factor per matrix
    if prec == MUON_NS_BF16:
        apply_tiles = sum(len(mem) * math.ceil(r / 256) * math.ceil(c / 256)
                          for (r, c), mem in groups.items() if r * c > TINY and (r > 128 or c > 512))
        slots = 16
    else:
        apply_tiles = sum(len(mem) * math.ceil(r / 64) * math.ceil(c / 64) for (r, c), mem in groups.items())
        slots = 1
    off = al(off + apply_tiles * slots * 4, 256)
    off = al(off + nm * 4, 256)
    # chained launch (bf16): a 16-byte entry per tile of every stage of every
    # step of every grouped matrix, then a dependency counter per matrix and
    # the tile counter
    if prec == MUON_NS_BF16:
        chain = 0
        for (r, c), mem in groups.items():
            if r * c > TINY and (r > 128 or c > 512):
                pb = math.ceil(r / 256)
                chain += len(mem) * 10 * (2 * (pb * (pb + 1) // 2) + pb * math.ceil(c / 256))
        off = al(off + chain * 16, 256)
        off = al(off + (nm + 1) * 4, 256)
    off = al(off, 1024)
    for (r, c), mem in sorted(groups.items(), key=lambda kv: order.index(kv[0])):
        k = len(mem)
        x = k * r * al(c, 8)
        a = k * r * al(r, 8)
        if prec == MUON_NS_BF16:
            # iterate high part (two, ping-pong) and low part, bf16; A; B
            for nbytes in (2 * x, 2 * x, 2 * x, 2 * a, 2 * a):
                off = al(off + nbytes, 1024)
        else:
            for nbytes in (4 * x, 4 * x, 4 * a, 4 * a):
                off = al(off + nbytes, 1024)
    return off


@pytest.mark.parametrize("prec", [MUON_NS_BF16, MUON_NS_FP32])
def test_workspace_size_matches_layout(lib, prec):
    shapes = [(256, 512), (512, 256), (7, 3), (1000, 130), (130, 1000), (1, 1), (100, 300), (300, 100)]
    shapes += [(k, 2 * k + 1) for k in range(2, 40)]  # many groups: descriptor bytes matter
    st, plan = create(lib, shapes, prec)
    assert st == MUON_OK
    n = ctypes.c_size_t()
    assert lib.muon_plan_workspace_size(plan, ctypes.byref(n)) == MUON_OK
    lib.muon_plan_destroy(plan)
    assert n.value == expected_workspace(shapes, prec)
    m = ctypes.c_size_t()
    assert lib.muon_workspace_size(params(shapes), len(shapes), prec, ctypes.byref(m)) == MUON_OK
    assert m.value == n.value


def launch_list(lib, shapes, prec=MUON_NS_BF16):
    st, plan = create(lib, shapes, prec)
    assert st == MUON_OK
    cnt = ctypes.c_int()
    kinds = (ctypes.c_int * 128)()
    assert lib.muon_plan_launches(plan, ctypes.byref(cnt), kinds, 128) == MUON_OK
    lib.muon_plan_destroy(plan)
    return list(kinds[:cnt.value])


def test_launch_list(lib):
    # bf16: every stage in one chained launch (10), then the last Apply with the update (4)
    grouped = [10, 4]
    stagewise = [1, 2, 3] * 9 + [1, 2, 4]
    # matrices of at most 4096 elements run with fp32 operands in the tiny-matrix kernel (kind 9)
    assert launch_list(lib, [(64, 64)]) == [0, 9]
    assert launch_list(lib, [(1, 1), (7, 100), (1, 4096), (4096, 1), (32, 128)]) == [0, 9]
    # larger matrices up to 128 x 128 run in the one-CTA small-matrix kernel (kind 5)
    assert launch_list(lib, [(65, 64), (128, 128)]) == [0, 5]
    assert launch_list(lib, [(128, 128), (1, 1), (7, 100)]) == [0, 5, 9]
    assert launch_list(lib, [(300, 400)]) == [0] + grouped
    # min(n, m) <= 128 < max(n, m) <= 512: the one-CTA mid-size kernel (kind 8)
    assert launch_list(lib, [(129, 64)]) == [0, 8]
    assert launch_list(lib, [(128, 512), (512, 100), (1, 129)]) == [0, 8, 9]
    assert launch_list(lib, [(128, 513)]) == [0] + grouped
    assert launch_list(lib, [(1, 4097)]) == [0] + grouped
    assert launch_list(lib, [(129, 129)]) == [0] + grouped
    assert launch_list(lib, [(64, 64), (300, 400)]) == [0, 9] + grouped
    assert launch_list(lib, [(65, 65), (100, 300), (300, 400)]) == [0, 5, 8] + grouped
    # the fp32 validation precision runs every matrix on the grouped fp32 kernels, stage by stage
    assert launch_list(lib, [(64, 64)], MUON_NS_FP32) == [0] + stagewise
    assert launch_list(lib, [(2, 3)], MUON_NS_FP32) == [0] + stagewise
    assert launch_list(lib, [(300, 400)], MUON_NS_FP32) == [0] + stagewise


def test_chaining_can_be_turned_off(lib):
    st, plan = create(lib, [(300, 400), (64, 64)])
    cnt = ctypes.c_int()
    kinds = (ctypes.c_int * 128)()

    def kinds_now():
        assert lib.muon_plan_launches(plan, ctypes.byref(cnt), kinds, 128) == MUON_OK
        return list(kinds[:cnt.value])

    assert kinds_now() == [0, 9, 10, 4]
    assert lib.muon_plan_set_chaining(plan, 0, 0) == MUON_OK
    assert kinds_now() == [0, 9] + [1, 2, 3] * 9 + [1, 2, 4]
    assert lib.muon_plan_set_chaining(plan, 1, 7) == MUON_OK
    assert kinds_now() == [0, 9, 10, 4]
    assert lib.muon_plan_set_chaining(plan, 1, -1) == MUON_ERR_INVALID_ARG
    lib.muon_plan_destroy(plan)


def test_scale_modes_change_the_launch_list(lib):
    st, plan = create(lib, [(64, 64), (300, 400)])
    cnt = ctypes.c_int()
    kinds = (ctypes.c_int * 128)()

    def kinds_now():
        assert lib.muon_plan_launches(plan, ctypes.byref(cnt), kinds, 128) == MUON_OK
        return list(kinds[:cnt.value])

    shape = kinds_now()
    assert shape[-2:] == [10, 4]
    # unit-RMS: the chained launch keeps O' from the last Apply, then a
    # per-matrix reduction and an update pass
    assert lib.muon_plan_set_scale_mode(plan, 1) == MUON_OK
    assert kinds_now() == shape[:-1] + [6, 7]
    assert lib.muon_plan_set_scale_mode(plan, 2) == MUON_OK
    assert kinds_now() == shape
    assert lib.muon_plan_set_scale_mode(plan, 3) == MUON_ERR_INVALID_ARG
    lib.muon_plan_destroy(plan)
    # small and tiny matrices only: their one-CTA kernels reduce on chip
    st, plan = create(lib, [(64, 64), (128, 128)])
    assert lib.muon_plan_set_scale_mode(plan, 1) == MUON_OK
    assert kinds_now() == [0, 5, 9]
    lib.muon_plan_destroy(plan)
    # diagnostics add one reduction after the fused last step (shape / none scale)
    st, plan = create(lib, [(64, 64), (300, 400)])
    shape = kinds_now()
    assert lib.muon_plan_set_diagnostics(plan, ctypes.c_void_p(FAKE)) == MUON_OK
    assert kinds_now() == shape + [6]
    assert lib.muon_plan_set_scale_mode(plan, 1) == MUON_OK
    assert kinds_now() == shape[:-1] + [6, 7]
    assert lib.muon_plan_set_diagnostics(plan, None) == MUON_OK
    assert lib.muon_plan_set_scale_mode(plan, 0) == MUON_OK
    assert kinds_now() == shape
    assert lib.muon_plan_set_diagnostics(plan, ctypes.c_void_p(FAKE + 2)) == MUON_ERR_INVALID_ARG
    lib.muon_plan_destroy(plan)
    # orthogonalisation plans have no update to scale
    ns = ctypes.c_void_p()
    mats = (MuonNsMatrix * 1)(MuonNsMatrix(FAKE, 2 * FAKE, 5, 9))
    assert lib.muon_plan_create_ns(mats, 1, MUON_NS_BF16, None, ctypes.byref(ns)) == MUON_OK
    assert lib.muon_plan_set_scale_mode(ns, 1) == MUON_ERR_INVALID_ARG
    assert lib.muon_plan_set_diagnostics(ns, ctypes.c_void_p(FAKE)) == MUON_ERR_INVALID_ARG
    lib.muon_plan_destroy(ns)


def test_flops_count_the_computed_tiles(lib):
    """Tensor-core mode: Gram and polynomial count the 128 x 128 blocks on and
    below the diagonal; apply is dense: 2 r^2 c per step."""
    for r, c in [(256, 512), (1024, 1024), (300, 1000), (4096, 14336)]:
        st, plan = create(lib, [(r, c)])
        g, p, a = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
        lib.muon_plan_flops(plan, ctypes.byref(g), ctypes.byref(p), ctypes.byref(a))
        lib.muon_plan_destroy(plan)
        rb = math.ceil(r / 128)
        lower = sum(min(128, r - 128 * i) * min(128, r - 128 * j) for i in range(rb) for j in range(i + 1))
        assert g.value == pytest.approx(10 * 2 * lower * c)
        assert p.value == pytest.approx(10 * 2 * lower * r)
        assert a.value == pytest.approx(10 * 2 * r * r * c)
        # the lower triangle with its diagonal blocks: r^2/2 <= lower <= r^2/2 + 64 r
        assert r * r / 2 <= lower <= r * r / 2 + 64 * r


def test_ns_plan_arguments(lib):
    plan = ctypes.c_void_p()
    mats = (MuonNsMatrix * 1)(MuonNsMatrix(FAKE, 2 * FAKE, 5, 9))
    assert lib.muon_plan_create_ns(mats, 1, MUON_NS_BF16, None, ctypes.byref(plan)) == MUON_OK
    lib.muon_plan_destroy(plan)
    mats[0].O = None
    assert lib.muon_plan_create_ns(mats, 1, MUON_NS_BF16, None, ctypes.byref(plan)) == MUON_ERR_INVALID_ARG


def test_timing_events_need_two_per_launch(lib):
    st, plan = create(lib, [(300, 300)])
    ev = (ctypes.c_void_p * 62)(*([FAKE] * 62))
    # chained: the elementwise launch, the chain and the fused last Apply
    assert lib.muon_plan_set_events(plan, ev, 5) == MUON_ERR_INVALID_ARG
    assert lib.muon_plan_set_events(plan, ev, 6) == MUON_OK
    assert lib.muon_plan_set_events(plan, None, 0) == MUON_OK
    # stage by stage: 1 + 30 launches
    assert lib.muon_plan_set_chaining(plan, 0, 0) == MUON_OK
    assert lib.muon_plan_set_events(plan, ev, 61) == MUON_ERR_INVALID_ARG
    assert lib.muon_plan_set_events(plan, ev, 62) == MUON_OK
    assert lib.muon_plan_set_events(plan, None, 0) == MUON_OK
    lib.muon_plan_destroy(plan)


def test_shard_calls_validate_before_touching_a_device(lib):
    from muon_step_b200._lib import ShardMomentum, ShardUpdate
    n = ctypes.c_size_t()
    assert lib.muon_shard_workspace_size(0, ctypes.byref(n)) == MUON_ERR_INVALID_ARG
    assert lib.muon_shard_workspace_size(5, ctypes.byref(n)) == MUON_OK and n.value == 256
    assert lib.muon_shard_workspace_size(6, ctypes.byref(n)) == MUON_OK and n.value == 512  # 48 B each
    ws = ctypes.c_void_p(1 << 20)
    mom = (ShardMomentum * 1)(ShardMomentum(FAKE, FAKE + 4096, FAKE + 8192, -1))
    assert lib.muon_shard_momentum(mom, 1, 0.95, 1, ws, 1 << 20, None) == MUON_ERR_INVALID_ARG
    mom[0] = ShardMomentum(FAKE, None, FAKE + 8192, 16)
    assert lib.muon_shard_momentum(mom, 1, 0.95, 1, ws, 1 << 20, None) == MUON_ERR_INVALID_ARG
    mom[0] = ShardMomentum(FAKE + 2, FAKE + 4096, FAKE + 8192, 16)
    assert lib.muon_shard_momentum(mom, 1, 0.95, 1, ws, 1 << 20, None) == MUON_ERR_INVALID_ARG
    assert lib.muon_shard_momentum(mom, 0, 0.95, 1, ws, 1 << 20, None) == MUON_ERR_INVALID_ARG
    mom[0] = ShardMomentum(FAKE, FAKE + 4096, FAKE + 8192, 16)
    assert lib.muon_shard_momentum(mom, 1, float("nan"), 1, ws, 1 << 20, None) == MUON_ERR_INVALID_ARG
    assert lib.muon_shard_momentum(mom, 1, 0.95, 1, ctypes.c_void_p((1 << 20) + 8), 1 << 20,
                                   None) == MUON_ERR_WORKSPACE
    upd = (ShardUpdate * 1)(ShardUpdate(FAKE, FAKE + 4096, 16, 0, 4))
    assert lib.muon_shard_update(upd, 1, 0.02, 0.1, 0.2, ws, 1 << 20, None) == MUON_ERR_INVALID_ARG
    upd[0] = ShardUpdate(FAKE, FAKE + 4096, 16, 4, 4)
    assert lib.muon_shard_update(upd, 1, float("inf"), 0.1, 0.2, ws, 1 << 20, None) == MUON_ERR_INVALID_ARG
    assert lib.muon_shard_update(upd, 1, 0.02, 0.1, 0.2, ws, 16, None) == MUON_ERR_WORKSPACE


def test_l2_batching_repeats_the_stage_launches_per_batch(lib):
    shapes = [(300, 400), (400, 300), (300, 400), (100, 100)]
    st, plan = create(lib, shapes)
    assert st == MUON_OK
    cnt = ctypes.c_int()
    kinds = (ctypes.c_int * 512)()

    def kinds_now():
        assert lib.muon_plan_launches(plan, ctypes.byref(cnt), kinds, 512) == MUON_OK
        return list(kinds[:cnt.value])

    one_pass = [1, 2, 3] * 9 + [1, 2, 4]
    assert kinds_now() == [0, 5, 10, 4]  # chained by default; L2 batching runs stage by stage
    ws0 = ctypes.c_size_t()
    assert lib.muon_plan_workspace_size(plan, ctypes.byref(ws0)) == MUON_OK
    # one 300 x 400 matrix needs 6*300*400 + 4*300*304 = 1,084,800 bytes of buffers
    assert lib.muon_plan_set_l2_batching(plan, 1_200_000) == MUON_OK
    assert kinds_now() == [0, 5] + one_pass * 3
    assert lib.muon_plan_set_l2_batching(plan, 2 * 1_084_800) == MUON_OK
    assert kinds_now() == [0, 5] + one_pass * 2
    assert lib.muon_plan_set_l2_batching(plan, 1) == MUON_OK  # at least one matrix per batch
    assert kinds_now() == [0, 5] + one_pass * 3
    ws1 = ctypes.c_size_t()
    assert lib.muon_plan_workspace_size(plan, ctypes.byref(ws1)) == MUON_OK
    assert ws1.value == ws0.value
    assert lib.muon_plan_set_l2_batching(plan, 0) == MUON_OK
    assert kinds_now() == [0, 5, 10, 4]
    lib.muon_plan_destroy(plan)


try:
    from hypothesis import given, settings
    from hypothesis import strategies as hst
except ImportError:  # pragma: no cover
    given = None


if given is not None:
    @settings(max_examples=60, deadline=None)
    @given(hst.lists(hst.tuples(hst.integers(1, 3000), hst.integers(1, 3000)), min_size=1, max_size=12),
           hst.sampled_from([MUON_NS_BF16, MUON_NS_FP32]))
    def test_planner_layout_and_launches_for_random_shapes(shapes, prec):
        """For any list of shapes the workspace follows the layout rule and the
        launch list holds the elementwise pass, the one-CTA kernels the shapes
        need and one pass of stage launches when a larger matrix is present."""
        lib = _lib.load()
        st, plan = create(lib, shapes, prec)
        assert st == MUON_OK
        n = ctypes.c_size_t()
        assert lib.muon_plan_workspace_size(plan, ctypes.byref(n)) == MUON_OK
        lib.muon_plan_destroy(plan)
        assert n.value == expected_workspace(shapes, prec)
        tc = prec == MUON_NS_BF16
        tiny = tc and any(a * b <= TINY for a, b in shapes)
        small = tc and any(a * b > TINY and max(a, b) <= 128 for a, b in shapes)
        mid = tc and any(a * b > TINY and min(a, b) <= 128 < max(a, b) <= 512 for a, b in shapes)
        large = any(not tc or (a * b > TINY and not (min(a, b) <= 128 and max(a, b) <= 512))
                    for a, b in shapes)
        want = [0] + ([5] if small else []) + ([8] if mid else []) + ([9] if tiny else [])
        if large:
            want += [10, 4] if tc else [1, 2, 3] * 9 + [1, 2, 4]
        assert launch_list(lib, shapes, prec) == want


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-std=c99", "-x", "c"]),
                                            ("g++", ["-std=c++17", "-x", "c++"])])
def test_headers_compile_as_plain_c_and_cpp(tmp_path, compiler, flags):
    """The ABI headers need no CUDA or torch types: a C program that calls
    every entry point (through pointers, never run) compiles warning-free."""
    import shutil
    import subprocess

    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    src = tmp_path / "use_abi.c"
    calls = "\n".join(f"  (void)&{name};" for name in header_symbols())
    src.write_text(
        "#include <string.h>\n"
        "#include \"muon_step.h\"\n#include \"muon_adamw.h\"\n#include \"muon_shard.h\"\n"
        "int main(void) {\n" + calls + "\n"
        "  muon_param_t p;\n  muon_adamw_hyper_t h;\n  muon_shard_update_t u;\n"
        "  memset(&p, 0, sizeof p);\n  memset(&h, 0, sizeof h);\n  memset(&u, 0, sizeof u);\n"
        "  return (int)(sizeof p + sizeof h + sizeof u == 0);\n}\n")
    out = subprocess.run([compiler, *flags, "-Wall", "-Wextra", "-Werror", "-I",
                          os.path.join(ROOT, "include"), "-c", str(src), "-o",
                          str(tmp_path / "use_abi.o")], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
