"""CPU model of the kernels' index arithmetic (compute-sanitizer is closed on
the GPUs these kernels run on, so out-of-bounds accesses are ruled out here).

The functions below restate, line for line in meaning, how each kernel turns
its launch (pairs, CTA rank, warp, lane, chunk) into tile coordinates, TMA
box coordinates and element accesses:

* ``stage_tc_kernel`` (csrc/ns_tc.cu): the planner's tile tables
  (tiles per matrix, prefix bases per group), the tile decode (lower-triangle
  pair tiles for Gram and Poly, row-block-fastest tiles for Apply), the
  producer's operand loads, and the epilogue warps' 32 x 32 chunks with their
  TMA loads and stores (the symmetric stages' outputs in the lower
  triangle of 256-row blocks, their operands read MN-major above it, the
  caller's W and O in its own orientation for the last step);
* ``ns_small_kernel``, ``ns_mid_kernel`` and ``ns_tiny_kernel``: which
  thread touches which element of the iterate, the shared-memory tiles and
  the caller's matrices.

For ragged, transposed and multi-group plans the tests check the TMA rules
(innermost coordinate x a multiple of 16 bytes, stores never start at a
negative coordinate, matrix index inside the group), that every load and
store lies inside its buffer once the tensor map's clipping is applied, and
that every element of every output (A, B, the iterate's high and low parts,
W, O) is written exactly once per launch.
"""

import math

import numpy as np
import pytest

PAIR = 256      # output tile of a CTA pair
HALF = 128      # rows per CTA
BK = 64         # K block (bf16 elements)
SMALL_MAX = 128
MID_MAX_C = 512
TINY_MAX = 4096

GRAM, POLY, APPLY, APPLY_LAST = 0, 1, 2, 3


def cdiv(a, b):
    return -(-a // b)


# ---------------------------------------------------------------- planner tables

def groups_of(shapes):
    """Shape groups in first-seen order, as the planner builds them:
    (r, c, count, [(n, m, transposed) per member])."""
    order, members = [], {}
    for n, m in shapes:
        key = (min(n, m), max(n, m))
        if key not in members:
            order.append(key)
            members[key] = []
        members[key].append((n, m, n > m))
    return [(r, c, len(members[(r, c)]), members[(r, c)]) for r, c in order]


def one_cta(r, c):
    return r * c <= TINY_MAX or (r <= SMALL_MAX and c <= MID_MAX_C)


def tile_tables(groups):
    """Per group: tiles per matrix for (Gram, Poly, Apply) and the prefix
    bases; groups run by a one-CTA kernel have no stage tiles."""
    per, base, tot = [], [], [0, 0, 0]
    for r, c, count, _ in groups:
        if one_cta(r, c):
            t = (0, 0, 0)
        else:
            pb = cdiv(r, PAIR)
            t = (pb * (pb + 1) // 2, pb * (pb + 1) // 2, pb * cdiv(c, PAIR))
        per.append(t)
        base.append(tuple(tot))
        tot = [tot[k] + t[k] * count for k in range(3)]
    return per, base, tot


def lower_tile(u):
    """u = I (I + 1) / 2 + J with J <= I (the kernel's float estimate, then
    the two correcting loops)."""
    i = int((math.sqrt(8.0 * u + 1.0) - 1.0) * 0.5)
    while i * (i + 1) // 2 > u:
        i -= 1
    while (i + 1) * (i + 2) // 2 <= u:
        i += 1
    return i, u - i * (i + 1) // 2


def decode(groups, per, base, kind_table, t):
    """(group, matrix, I, J, kblocks) of tile t of a stage's table."""
    g = 0
    while g + 1 < len(groups) and base[g + 1][kind_table] <= t:
        g += 1
    r, c, _, _ = groups[g]
    local = t - base[g][kind_table]
    p = per[g][kind_table]
    b, u = local // p, local % p
    if kind_table == APPLY:
        rb = cdiv(r, PAIR)
        return g, b, u % rb, u // rb, cdiv(r, BK)
    I, J = lower_tile(u)
    return g, b, I, J, cdiv(c if kind_table == GRAM else r, BK)


# ---------------------------------------------------------------- stage kernel

class Buffers:
    """Write counters for the outputs of one launch, and the TMA checks."""

    def __init__(self, groups):
        self.groups = groups
        self.writes = {}

    def buf(self, name, g, shape):
        key = (name, g)
        if key not in self.writes:
            count = 1 if isinstance(name, tuple) else self.groups[g][2]
            self.writes[key] = np.zeros((count,) + shape, dtype=np.int32)
        return self.writes[key]

    @staticmethod
    def check_box(x, y, z, count, elem_bytes, store):
        assert (x * elem_bytes) % 16 == 0, ("x not 16-byte aligned", x)
        assert 0 <= z < count, ("matrix index", z, count)
        if store:
            assert x >= 0 and y >= 0, ("store at a negative coordinate", x, y)

    def store(self, name, g, b, x, y, box, inner, rows, elem_bytes=2):
        """A clipped TMA tensor store of a box {box[0] cols, box[1] rows}
        (per-matrix maps, named (name, matrix), have one matrix: b = 0)."""
        count = 1 if isinstance(name, tuple) else self.groups[g][2]
        self.check_box(x, y, b, count, elem_bytes, store=True)
        assert x < inner and y < rows, ("store box starts outside the tensor", x, y, inner, rows)
        w = self.buf(name, g, (rows, inner))
        w[b, y:min(y + box[1], rows), x:min(x + box[0], inner)] += 1


def run_stage(shapes, kind, npairs, wide):
    """Walk one launch of stage `kind` (GRAM, POLY, APPLY or APPLY_LAST) and
    return the write counters."""
    groups = groups_of(shapes)
    per, base, tot = tile_tables(groups)
    table = APPLY if kind in (APPLY, APPLY_LAST) else kind
    epi_warps = 8 if (wide or kind == APPLY) else 4
    chunks_per_warp = (PAIR // 32) // (epi_warps // 4)
    out = Buffers(groups)
    seen = set()
    for pair in range(npairs):
        for t in range(pair, tot[table], npairs):
            assert t not in seen
            seen.add(t)
            g, b, I, J, kblocks = decode(groups, per, base, table, t)
            r, c, count, members = groups[g]
            assert I < cdiv(r, PAIR) and J <= (cdiv(c, PAIR) - 1 if table == APPLY else I)
            for rank in range(2):
                # producer: operand loads (zero-filled past the extent); a
                # symmetric operand's K block above the diagonal block is
                # read MN-major from its transposed, stored position
                def sym_half(blk, k0):
                    row = blk * PAIR + rank * HALF
                    if k0 // PAIR > blk:
                        assert k0 // PAIR >= blk  # block (k0 / 256, blk) is in the stored triangle
                        for q in range(HALF // 64):
                            out.check_box(row + q * 64, k0, b, count, 2, store=False)
                        return ("mn", k0 // PAIR, blk)
                    out.check_box(k0, row, b, count, 2, store=False)
                    return ("k", blk, k0 // PAIR)

                for kb in range(kblocks):
                    k0 = kb * BK
                    if table == APPLY:
                        src = sym_half(I, k0)
                        assert src[1] >= src[2]  # only stored (lower-triangle) blocks of B are read
                        for q in range(HALF // 64):
                            out.check_box(J * PAIR + rank * HALF + q * 64, k0, b, count, 2, store=False)
                    elif kind == GRAM:
                        out.check_box(k0, I * PAIR + rank * HALF, b, count, 2, store=False)
                        if I != J:
                            out.check_box(k0, J * PAIR + rank * HALF, b, count, 2, store=False)
                    else:
                        for blk in ((I,) if I == J else (I, J)):
                            src = sym_half(blk, k0)
                            assert src[1] >= src[2]  # only stored (lower-triangle) blocks of A
                # epilogue warps
                for ew in range(epi_warps):
                    quarter = (ew + 2) & 3
                    ch_begin = (ew // 4) * chunks_per_warp
                    row0 = I * PAIR + rank * HALF + quarter * 32
                    limit_c = c if table == APPLY else r
                    for ch in range(ch_begin, ch_begin + chunks_per_warp):
                        col0 = J * PAIR + ch * 32
                        if not (row0 < r and col0 < limit_c):
                            continue
                        if kind in (GRAM, POLY):
                            name = "A" if kind == GRAM else "B"
                            if kind == POLY:
                                out.check_box(col0, row0, b, count, 2, store=False)
                            # the tile's own chunk only: the stored lower triangle
                            out.store(name, g, b, col0, row0, (32, 32), r, r)
                        else:
                            out.check_box(col0, row0, b, count, 2, store=False)  # high part in
                            if kind == APPLY:
                                out.store("X_hi", g, b, col0, row0, (32, 32), c, r)
                                out.store("X_lo", g, b, col0, row0, (32, 32), c, r)
                            else:
                                n, m, tr = members[b]
                                x, y = (row0, col0) if tr else (col0, row0)
                                # caller's W (and O): inner m, n rows, fp32; one map per matrix
                                out.store(("W", b), g, 0, x, y, (32, 32), m, n, elem_bytes=4)
    assert len(seen) == tot[table]
    return groups, out


SHAPE_SETS = [
    [(300, 520), (520, 300), (257, 129), (1000, 300)],
    [(1024, 1024), (256, 256), (255, 257), (513, 1030)],
    [(129, 4097), (4097, 129), (600, 600), (130, 514)],
]


@pytest.mark.parametrize("shapes", SHAPE_SETS)
@pytest.mark.parametrize("npairs", [74, 5])
@pytest.mark.parametrize("wide", [False, True])
def test_symmetric_stages_write_every_element_once(shapes, npairs, wide):
    """Gram and Poly store every element of the lower triangle of 256-row
    blocks of A and B (diagonal blocks in full) exactly once and nothing
    above it; the consumers read the blocks above from their transposed
    positions."""
    for kind, name in ((GRAM, "A"), (POLY, "B")):
        groups, out = run_stage(shapes, kind, npairs, wide)
        for g, (r, c, count, _) in enumerate(groups):
            if one_cta(r, c):
                assert (name, g) not in out.writes
                continue
            w = out.writes[(name, g)]
            assert w.shape == (count, r, r)
            blk = np.arange(r) // PAIR
            lower = blk[:, None] >= blk[None, :]
            assert (w[:, lower] == 1).all(), (name, r, c, np.unique(w[:, lower]))
            assert (w[:, ~lower] == 0).all(), (name, r, c)


@pytest.mark.parametrize("shapes", SHAPE_SETS)
@pytest.mark.parametrize("npairs", [74, 3])
def test_apply_writes_the_iterate_once(shapes, npairs):
    groups, out = run_stage(shapes, APPLY, npairs, True)
    for g, (r, c, count, _) in enumerate(groups):
        if one_cta(r, c):
            continue
        for name in ("X_hi", "X_lo"):
            w = out.writes[(name, g)]
            assert w.shape == (count, r, c) and (w == 1).all(), (name, r, c)


@pytest.mark.parametrize("shapes", SHAPE_SETS)
@pytest.mark.parametrize("wide", [False, True])
def test_last_apply_updates_every_weight_once_in_the_callers_orientation(shapes, wide):
    groups, out = run_stage(shapes, APPLY_LAST, 74, wide)
    for g, (r, c, count, members) in enumerate(groups):
        if one_cta(r, c):
            continue
        for b, (n, m, _) in enumerate(members):
            w = out.writes[(("W", b), g)]
            assert w.shape == (1, n, m) and (w == 1).all(), (n, m)


def test_lower_tile_decode_is_exact_far_out():
    """The float estimate of the triangular root and its correcting loops
    invert u = I (I + 1) / 2 + J for every u up to 2^31 tiles' worth of rows."""
    for I in list(range(0, 300)) + [10 ** 4, 65535, 2 ** 20]:
        for J in {0, I // 2, I}:
            assert lower_tile(I * (I + 1) // 2 + J) == (I, J)


# ---------------------------------------------------------------- one-CTA kernels

def small_kernel_accesses(n, m):
    """ns_small_kernel (256 threads): thread t owns iterate row t % 128 and
    half t / 128 of its columns; its 16-byte loads of the high and low parts
    start at column col_base + 8 q < c; the update walks caller rows, two per
    pass, with lane = column within each 32-column piece."""
    r, c = min(n, m), max(n, m)
    ldc = cdiv(c, 8) * 8
    loads = np.zeros((r, ldc), dtype=np.int32)
    for t in range(256):
        row, half = t & 127, t >> 7
        col_base = half * 64
        for q in range(8):
            if row < r and col_base + 8 * q < c:
                a = col_base + 8 * q
                assert a + 8 <= ldc
                loads[row, a:a + 8] += 1
    assert (loads[:, :c] == 1).all()
    # shared-memory transpose tile: (i & 127) * 128 + ((j & 127) ^ (i & 31)) stays in 128 x 128
    writes = np.zeros((n, m), dtype=np.int32)
    tr = n > m
    rows, cols = (c, r) if tr else (r, c)
    for warp in range(8):
        for crow0 in range(warp, rows, 16):
            for u in range(2):
                crow = crow0 + 8 * u
                if crow >= rows:
                    break
                for q in range(4):
                    for lane in range(32):
                        col = 32 * q + lane
                        if col >= cols:
                            continue
                        i, j = (col, crow) if tr else (crow, col)
                        assert 0 <= (i & 127) * 128 + ((j & 127) ^ (i & 31)) < 128 * 128
                        writes[crow, col] += 1
    return writes


@pytest.mark.parametrize("n,m", [(128, 128), (65, 64), (100, 120), (120, 100), (128, 33), (33, 128)])
def test_small_kernel_touches_every_element_once(n, m):
    w = small_kernel_accesses(n, m)
    assert (w == 1).all()


def mid_kernel_low_index(r, row, col):
    """The mid-size kernel's low part layout: 8-column groups [col/8][row][col%8]."""
    return ((col >> 3) * r + row) * 8 + (col & 7)


@pytest.mark.parametrize("r,c", [(128, 512), (9, 500), (100, 300), (64, 129), (128, 129), (77, 333)])
def test_mid_kernel_low_part_layout_is_a_bijection_into_its_buffer(r, c):
    ldc = cdiv(c, 8) * 8
    seen = np.zeros(r * ldc, dtype=np.int32)
    for row in range(r):
        for col in range(c):
            seen[mid_kernel_low_index(r, row, col)] += 1
    assert seen.max() == 1 and seen.sum() == r * c
    # the 16-byte pieces of 32 consecutive rows form one contiguous 512-byte run
    for g8 in range(cdiv(c, 8)):
        starts = [mid_kernel_low_index(r, row, 8 * g8) for row in range(min(r, 32))]
        assert starts == list(range(starts[0], starts[0] + 8 * len(starts), 8))


MID_TMEM_COLS, MID_LO_COL = 512, 256


def mid_kernel_tmem_columns(c):
    """ns_mid_kernel's TMEM use for a matrix of c columns (128 < c <= 512):
    the Apply product runs one column half h at a time into accumulator
    columns 0 .. 255; in the epilogue of half h, thread quarter cq takes the
    32-column chunks 256 h + 64 cq + 32 j (j = 0, 1) that start inside the
    matrix; the low part of iterate column col sits at column 256 + col / 2,
    loaded by quarter cq for chunks 128 cq + 32 g and read by the update for
    chunks p0 + 32 cq. Returns, per iterate column, the (half, accumulator
    column, low column) the epilogue uses, and the low columns the load and
    the update touch."""
    nh = cdiv(c, 256)
    epi = {}
    for h in range(nh):
        for cq in range(4):
            for j in range(2):
                acc = 64 * cq + 32 * j
                col0 = 256 * h + acc
                if col0 >= c:
                    break
                for e in range(32):
                    epi.setdefault(col0 + e, []).append((h, acc + e, MID_LO_COL + (col0 >> 1) + e // 2))
    loaded = {MID_LO_COL + ((128 * cq + 32 * g) >> 1) + w for cq in range(4) for g in range(4) for w in range(16)}
    updated = {}
    for p0 in range(0, c, 128):
        for cq in range(4):
            col0 = p0 + 32 * cq
            if col0 < c:
                for e in range(32):
                    updated.setdefault(col0 + e, MID_LO_COL + (col0 >> 1) + e // 2)
    return epi, loaded, updated


@pytest.mark.parametrize("c", [129, 200, 256, 257, 300, 383, 384, 500, 512])
def test_mid_kernel_tmem_columns(c):
    epi, loaded, updated = mid_kernel_tmem_columns(c)
    for col in range(c):
        # each column of the matrix goes through the epilogue exactly once, in
        # its own half, from an accumulator column below the low part
        assert len(epi[col]) == 1, col
        h, acc, lo = epi[col][0]
        assert h == col // 256 and acc == col - 256 * h and 0 <= acc < MID_LO_COL
        assert lo == MID_LO_COL + col // 2 < MID_TMEM_COLS
        # the low column was loaded at the start of the matrix; the update
        # reads the same column
        assert lo in loaded and updated[col] == lo
    assert all(MID_LO_COL <= x < MID_TMEM_COLS for x in loaded)


def tiny_kernel_accesses(n, m):
    """ns_tiny_kernel: caller element e = crow * m + ccol maps to iterate
    (i, j) = (ccol, crow) when n > m else (crow, ccol); X lives at i * (c | 1) + j
    inside a buffer of TINY_MAX + 64 floats, A and B at i * (r | 1) + j."""
    r, c = min(n, m), max(n, m)
    ldx, ldr = c | 1, r | 1
    cap = TINY_MAX + 64
    xs = np.zeros(cap, dtype=np.int32)
    tr = n > m
    for e in range(r * c):
        crow, ccol = divmod(e, m)
        i, j = (ccol, crow) if tr else (crow, ccol)
        assert 0 <= i < r and 0 <= j < c
        xs[i * ldx + j] += 1
    assert xs.max() == 1 and xs.sum() == r * c
    assert (r - 1) * ldx + c <= cap and (r - 1) * ldr + r <= cap
    return xs


@pytest.mark.parametrize("n,m", [(1, 1), (1, 4096), (4096, 1), (64, 64), (33, 47), (47, 33),
                                 (17, 240), (2, 2048), (63, 65)])
def test_tiny_kernel_stays_inside_its_buffers(n, m):
    assert n * m <= TINY_MAX
    tiny_kernel_accesses(n, m)


# ---------------------------------------------------------------- chained launch

CHAIN_ARRIVALS = 16  # epilogue warps per tile (8 per CTA, two CTAs)


def build_chain(shapes, npairs, steps=10, window=0):
    """The planner's tile list of the chained launch: a window of matrices in
    flight, in rounds; each round lists the next stage of every matrix in the
    window (all its tiles); finished matrices leave for the next ones."""
    groups = groups_of(shapes)
    per, _, _ = tile_tables(groups)
    mats = []  # (group, index in group)
    for g, (r, c, count, _) in enumerate(groups):
        mats += [(g, b) for b in range(count)]
    grouped = [k for k, (g, b) in enumerate(mats) if sum(per[g]) > 0]
    if not grouped:
        return groups, per, mats, []
    if window <= 0:
        mean = sum(sum(per[mats[k][0]]) / 3.0 for k in grouped) / len(grouped)
        window = max(2, math.ceil(2.5 * max(npairs, 1) / max(mean, 1.0)))
    window = max(1, min(window, len(grouped)))
    out, act, nxt = [], [], 0
    while nxt < len(grouped) or act:
        while len(act) < window and nxt < len(grouped):
            act.append([grouped[nxt], 0])
            nxt += 1
        for x in act:
            g = mats[x[0]][0]
            out += [(x[0], x[1], u) for u in range(per[g][x[1] % 3])]
            x[1] += 1
        act = [x for x in act if x[1] < 3 * steps]
    return groups, per, mats, out


def chain_need(per_g, stage):
    """Counter value at which every tile of the matrix's earlier stages has
    finished (the kernel's chain_pos)."""
    g0, p0, a0 = per_g
    step, kind = divmod(stage, 3)
    return CHAIN_ARRIVALS * (step * (g0 + p0 + a0) + (g0 if kind >= 1 else 0) + (p0 if kind >= 2 else 0))


def simulate_chain(shapes, npairs, steps=10, window=0, chain_stages=None, resident=None):
    """CTA pairs take list indices from one shared counter, in increasing order,
    as they become free (an index of a skipped stage is taken and dropped); a
    pair holding a tile starts it when its matrix's counter has reached the
    target and adds CHAIN_ARRIVALS when it finishes (its time: its K blocks).
    Only `resident` of the launch's pairs ever run (default: all), as when the
    device cannot hold the whole grid at once. Returns the makespan; fails on
    a deadlock."""
    groups, per, mats, tiles = build_chain(shapes, npairs, steps, window)
    nst = 3 * steps if chain_stages is None else chain_stages
    run = npairs if resident is None else resident
    dep = [0] * len(mats)
    nxt = 0                                 # the shared tile counter
    held = [None] * run                     # list index a pair has taken
    busy = [0.0] * run                      # time each pair becomes free
    now, done, running = 0.0, 0, []         # running: (finish time, pair, matrix)
    todo = sum(1 for _, s, _ in tiles if s < nst)
    import heapq
    while done < todo:
        progressed = False
        for p in range(run):
            if busy[p] > now:
                continue
            while held[p] is None and nxt < len(tiles):
                if tiles[nxt][1] < nst:
                    held[p] = nxt
                nxt += 1                    # skipped indices are dropped by every role
            if held[p] is None:
                continue
            mat, stage, u = tiles[held[p]]
            g = mats[mat][0]
            if dep[mat] < chain_need(per[g], stage):
                continue
            r, c, _, _ = groups[g]
            k = c if stage % 3 == 0 else r
            t_end = now + cdiv(k, BK)
            heapq.heappush(running, (t_end, p, mat))
            busy[p] = t_end
            held[p] = None
            progressed = True
        if running:
            t_end, p, mat = heapq.heappop(running)
            now = max(now, t_end)
            dep[mat] += CHAIN_ARRIVALS
            done += 1
        elif not progressed:
            raise AssertionError("deadlock: no pair can start a tile")
    return now, dep, per, mats, tiles


@pytest.mark.parametrize("shapes,npairs", [
    ([(1024, 1024)] * 64, 74),
    ([(512, 512)] * 40 + [(512, 2048)] * 7, 74),
    ([(4096, 4096)] * 4 + [(4096, 14336)] * 2 + [(14336, 4096)], 74),
    ([(300, 520), (520, 300), (257, 129), (1000, 300), (600, 600)], 3),
    ([(1024, 1024)] * 5, 1),
])
def test_chain_list_covers_every_stage_once_and_never_deadlocks(shapes, npairs):
    for window in (0, 1, 3):
        for stages in (None, 29):
            _, dep, per, mats, tiles = simulate_chain(shapes, npairs, window=window, chain_stages=stages)
            # every tile of every stage of every grouped matrix, once
            seen = {}
            for mat, stage, u in tiles:
                seen[(mat, stage, u)] = seen.get((mat, stage, u), 0) + 1
            assert all(v == 1 for v in seen.values())
            for k, (g, _) in enumerate(mats):
                if sum(per[g]) == 0:
                    continue
                for stage in range(30):
                    assert all((k, stage, u) in seen for u in range(per[g][stage % 3]))
                # the counter ends at the arrivals of every tile that ran
                nst = 30 if stages is None else stages
                assert dep[k] == chain_need(per[g], nst), (k, dep[k])
            # a tile's target is reached only by tiles listed before it
            first_pos = {}
            for i, (mat, stage, u) in enumerate(tiles):
                first_pos.setdefault((mat, stage), i)
            for i, (mat, stage, u) in enumerate(tiles):
                if stage > 0:
                    assert first_pos[(mat, stage - 1)] < first_pos[(mat, stage)] <= i


@pytest.mark.parametrize("resident", [1, 2, 37])
def test_chain_finishes_with_any_number_of_resident_pairs(resident):
    """Tiles go to whichever pair asks next, so the list completes even when
    the device runs fewer pairs at once than the launch has (the rest start
    later or, here, never)."""
    shapes = [(1024, 1024)] * 12 + [(512, 2048)] * 3
    full, dep, per, mats, _ = simulate_chain(shapes, 74)
    t, dep_r, _, _, _ = simulate_chain(shapes, 74, resident=resident)
    assert dep_r == dep
    assert t >= full


def test_chain_targets_are_prefix_sums_of_earlier_stages():
    per_g = (10, 10, 16)
    assert chain_need(per_g, 0) == 0
    assert chain_need(per_g, 1) == 16 * 10
    assert chain_need(per_g, 2) == 16 * 20
    assert chain_need(per_g, 3) == 16 * 36
    assert chain_need(per_g, 29) == 16 * (9 * 36 + 20)
