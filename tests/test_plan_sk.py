"""Host-side check of the balanced small-batch kernel's plan (gemv_sk.cuh)
and of its work split, copy boxes and shared-memory offsets (no GPU needed).

The plan comes from the library (an internal export).  The work-split and
stage formulas of the kernel (whole tiles dealt round-robin, the leftover
tiles cut into equal unit ranges) are restated here and replayed for every
CTA of the B200 grid: every (row tile, slice) unit is streamed by exactly
one CTA, no copy box reaches into another CTA's units (codes), metadata
over-reads stay inside the 8-group blocks at a range's two ends, every
shared-memory region fits, and every split row tile has one finisher (the
CTA holding its slice 0) whose publishers are the CTAs whose tail ranges
start inside it."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")
FIELDS = ["M", "N", "K", "ngroups", "tiles", "nk", "waves", "ctas", "split", "depth",
          "red_mode", "stage_bytes", "off_ring", "off_x", "off_sx", "off_red", "x_stride",
          "box_slices", "box_blocks", "smem", "grid", "resident", "max_stages", "max_tiles",
          "tail_tiles"]
B200_SMS = 148
B200_SMEM_OPTIN = 232448
SLICE_BYTES, ROWS, SLICES, BLOCK_GROUPS = 128, 16, 16, 8
WS_CTAS, WS_ROWS = 1024, 128


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.skip("libwq.so not built")
    lib = ctypes.CDLL(LIB)
    lib.wq_internal_plan_sk.restype = ctypes.c_int
    lib.wq_internal_plan_sk.argtypes = [ctypes.c_int] * 9 + [ctypes.POINTER(ctypes.c_int64)]
    return lib


def plan(lib, M, N, K, bits, group, sym=False, split=True, sms=B200_SMS):
    out = (ctypes.c_int64 * 32)()
    ok = lib.wq_internal_plan_sk(M, N, K, bits, group, int(sym), sms, B200_SMEM_OPTIN,
                                 int(split), out)
    return dict(zip(FIELDS, out[:len(FIELDS)])) if ok else None


def tail_begin(c, p):
    base = p["waves"] * p["ctas"] * p["nk"]
    if p["split"]:
        return base + c * (p["tail_tiles"] * p["nk"]) // p["ctas"]
    return base + min(c, p["tail_tiles"]) * p["nk"]


def run_stages(b, e, nk):
    """(tile, s0, s1, last stage of the tile in this run) over units [b, e)."""
    u = b
    while u < e:
        tile, s0 = divmod(u, nk)
        lim = min((s0 // SLICES + 1) * SLICES, nk)
        s1 = lim if lim - s0 <= e - u else s0 + (e - u)
        u += s1 - s0
        yield tile, s0, s1, s1 == nk or u == e


def cta_stages(c, p):
    nk = p["nk"]
    for w in range(p["waves"]):
        t = c + w * p["ctas"]
        yield from run_stages(t * nk, (t + 1) * nk, nk)
    yield from run_stages(tail_begin(c, p), tail_begin(c + 1, p), nk)


def check(p, bits, group, sym):
    M, N, K, nk = p["M"], p["N"], p["K"], p["nk"]
    slice_k = SLICE_BYTES * 8 // bits
    gps = slice_k // group
    meta_blocks = SLICES * gps // BLOCK_GROUPS
    nblk = p["ngroups"] // BLOCK_GROUPS
    assert nk * slice_k == K and p["ngroups"] * group == K and p["ngroups"] % 8 == 0
    units = p["tiles"] * nk
    assert p["tiles"] == -(-N // ROWS)
    assert p["grid"] == p["ctas"] <= B200_SMS and p["ctas"] <= WS_CTAS
    assert p["waves"] == p["tiles"] // p["ctas"] and p["tail_tiles"] == p["tiles"] % p["ctas"]
    assert ROWS * M <= WS_ROWS
    assert p["resident"] == (nk <= SLICES)
    assert p["box_slices"] == min(SLICES, nk) and p["box_blocks"] == min(meta_blocks, nblk)

    # shared memory: barriers, ring of 1024-aligned stages, X, Sx, partials
    assert 1 <= p["depth"] <= 32 and p["depth"] <= p["max_stages"]
    assert p["depth"] >= min(3, p["max_stages"])
    assert p["off_ring"] == 1024 and p["stage_bytes"] % 1024 == 0
    stage_need = SLICES * ROWS * SLICE_BYTES + meta_blocks * 256 * (1 if sym else 2)
    assert p["stage_bytes"] >= stage_need
    assert p["off_x"] == p["off_ring"] + p["depth"] * p["stage_bytes"]
    assert p["x_stride"] >= 2 * K and (p["x_stride"] // 64) % 2 == 1 and p["x_stride"] % 64 == 0
    assert p["off_sx"] >= p["off_x"] + M * p["x_stride"]
    assert p["off_red"] >= p["off_sx"] + M * p["ngroups"] * 8
    slots = p["max_tiles"] if p["red_mode"] == 0 else 2
    assert p["red_mode"] in (0, 2)
    assert p["smem"] >= p["off_red"] + slots * 16 * ROWS * M * 4
    assert p["smem"] <= B200_SMEM_OPTIN

    # the staged activation rows and the fragment offsets the warps read
    for s in range(nk):
        for c in range(8):
            for t in range(4):
                off = (32 * s + 4 * c + t) * 16 + 16 if bits == 4 else 256 * s + 32 * c + 8 * t + 8
                assert off <= 2 * K

    covered = [0] * units
    max_stages = max_tiles = 0
    finisher = {}
    publishers = {}
    loads = []
    for c in range(p["ctas"]):
        sts = list(cta_stages(c, p))
        max_stages = max(max_stages, len(sts))
        max_tiles = max(max_tiles, sum(1 for st in sts if st[3]))
        tb, te = tail_begin(c, p), tail_begin(c + 1, p)
        own = set(range(tb, te))
        for w in range(p["waves"]):
            t = c + w * p["ctas"]
            own.update(range(t * nk, (t + 1) * nk))
        loads.append(len(own))
        for tile, s0, s1, _ in sts:
            assert 0 < s1 - s0 <= SLICES and s1 <= nk
            a16 = s0 // SLICES * SLICES
            assert s1 <= a16 + SLICES             # a stage stays in one 16-slice block
            for s in range(s0, s1):
                covered[tile * nk + s] += 1
                assert 0 <= s - a16 < SLICES      # smem slot s - a16 = the owning warp
            whole = s0 == a16 and s1 == min(a16 + SLICES, nk)
            # codes: the whole box spans [a16, a16 + box_slices) of this tile;
            # everything inside the tensor must be this CTA's
            box = range(a16, a16 + p["box_slices"]) if whole else range(s0, s1)
            for s in box:
                if s < nk:
                    assert tile * nk + s in own
            # metadata blocks: whole box or the blocks the stage touches
            base = a16 * gps // BLOCK_GROUPS
            lo = s0 * gps // BLOCK_GROUPS
            hi = -(-s1 * gps // BLOCK_GROUPS)
            blocks = range(base, base + p["box_blocks"]) if whole else range(lo, hi)
            for blk in blocks:
                assert 0 <= blk - base < meta_blocks   # lands inside the stage's meta area
                if blk < nblk:
                    # a block holds groups of slices [8 blk / gps, 8 (blk + 1) / gps)
                    first = blk * BLOCK_GROUPS // gps
                    last = -(-(blk + 1) * BLOCK_GROUPS // gps)
                    mine = [s for s in range(first, last) if tile * nk + s in own]
                    assert mine, "a metadata block with none of the CTA's slices"
            assert tile * ROWS < N     # rows past N are zero-filled
        # tail tiles: published if slice 0 lies in another CTA's range; finished
        # here if this range holds slice 0 and the tile continues past it
        if te > tb:
            assert p["split"] or (tb % nk == 0 and te - tb == nk)
            t_first, t_last = tb // nk, (te - 1) // nk
            if tb % nk:
                publishers.setdefault(t_first, []).append(c)
            if te % nk and t_last * nk >= tb:
                finisher[t_last] = c
    assert all(v == 1 for v in covered), "every unit exactly once"
    assert max(loads) - min(loads) <= (1 if p["split"] else nk)
    assert max_stages == p["max_stages"] and max_tiles == p["max_tiles"]
    assert set(publishers) == set(finisher)
    for tile, f in finisher.items():
        # the finisher's wait list: CTAs after it whose non-empty tail ranges
        # start inside the tile
        waits = []
        c2 = f + 1
        while c2 < p["ctas"] and tail_begin(c2, p) < (tile + 1) * nk:
            if tail_begin(c2 + 1, p) > tail_begin(c2, p):     # empty ranges publish nothing
                waits.append(c2)
            c2 += 1
        assert waits == publishers[tile]


CASES = [(M, N, K, bits, group, sym)
         for M in (1, 2, 3, 4, 5, 8)
         for (N, K) in ((14336, 4096), (4096, 14336), (4096, 4096), (1024, 4096), (1000, 4096))
         for bits, group in ((4, 128), (4, 64), (4, 32), (8, 128), (8, 32))
         for sym in (False, True)]


@pytest.mark.parametrize("M,N,K,bits,group,sym", CASES)
def test_plan_sk_replay(lib, M, N, K, bits, group, sym):
    for split in (True, False):
        p = plan(lib, M, N, K, bits, group, sym, split)
        if p is None:
            # outside the kernel's scope: activations too large next to the ring
            assert M * K * 2 > 64 * 1024, (M, N, K, bits, group, sym)
            continue
        check(p, bits, group, sym)


def test_headline_shape_is_balanced(lib):
    p = plan(lib, 1, 14336, 4096, 4, 128)
    assert p["resident"] == 1 and p["split"] == 1 and p["ctas"] == B200_SMS
    assert p["waves"] == 6 and p["tail_tiles"] == 8      # 896 tiles = 6 x 148 + 8
    sizes = [tail_begin(c + 1, p) - tail_begin(c, p) for c in range(p["ctas"])]
    assert max(sizes) - min(sizes) <= 1
    # the ring holds all but at most one of a CTA's stages (two of them are
    # the partial stages at the range's ends): nearly every copy issues at once
    assert p["depth"] >= p["max_stages"] - 1


@pytest.mark.parametrize("M,N,K,bits,group", [(1, 256, 512, 4, 128), (9, 4096, 4096, 4, 128),
                                              (1, 4096, 4160, 4, 64), (1, 64, 1024, 4, 32)])
def test_out_of_scope_shapes(lib, M, N, K, bits, group):
    # M > 8, K not a multiple of one slice, or fewer than 8 groups per row
    # (then wq_matmul takes the cluster-split kernel)
    p = plan(lib, M, N, K, bits, group)
    if (M, N, K) == (1, 64, 1024):
        assert p is not None     # 32 groups per row: in scope
        check(p, bits, group, False)
    else:
        assert p is None


def test_small_grids(lib):
    # fewer units than SMs: one unit per CTA, every tile split
    p = plan(lib, 1, 32, 1024, 4, 32, sms=148)
    assert p["ctas"] == p["tiles"] * p["nk"] == 8 and p["waves"] == 0
    check(p, 4, 32, False)
    for sms in (1, 2, 7, 132):
        p = plan(lib, 2, 5000, 4096, 4, 128, sms=sms)
        assert p["ctas"] == sms
        check(p, 4, 128, False)
