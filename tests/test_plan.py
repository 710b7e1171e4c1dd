"""Host-side check of the small-batch matmul's launch plan and of the
kernel's shared-memory index arithmetic (no GPU needed).

The plan comes from the library itself (an internal export); the index
formulas below restate those of gemv.cuh and are replayed for every rank,
stage, warp and lane quarter, so that every shared-memory access stays in
its buffer and the permuted activation layout written by the staging loop
is exactly the one the tensor-core steps read."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")
FIELDS = ["M", "N", "K", "ngroups", "row_tiles", "items", "RT", "SKW", "BPW", "depth", "kc",
          "stage_k", "stages_per_item", "meta_tma", "stage_bytes", "meta_offset", "off_ring",
          "off_x", "off_sx", "off_red", "off_part", "smem", "C", "grid", "x_row_stride",
          "red_bufs", "row_stride", "contig"]
B200_SMS = 148
B200_SMEM_OPTIN = 232448


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from w4a16_decode_matmul_b200 import build
        build.build()
    lib = ctypes.CDLL(LIB)
    lib.wq_internal_plan_gemv.restype = ctypes.c_int
    lib.wq_internal_plan_gemv.argtypes = [ctypes.c_int] * 8 + [ctypes.POINTER(ctypes.c_int64)]
    return lib


def plan(lib, M, N, K, bits, group, cap=0, sms=B200_SMS):
    out = (ctypes.c_int64 * 32)()
    ok = lib.wq_internal_plan_gemv(M, N, K, bits, group, sms, B200_SMEM_OPTIN, cap, out)
    assert ok, (M, N, K, bits, group)
    return dict(zip(FIELDS, out[:len(FIELDS)]))


def geometry(bits, G):
    box_k = 64 * 8 // bits
    gbytes = G * bits // 8
    U = min(gbytes, 64)
    Uk = U * 8 // bits
    return dict(box_k=box_k, U=U, Uk=Uk, QB=U // 4, Qk=Uk // 4, words=U // 16,
                subunits=64 // U, steps=Uk // 16)


def check_plan(p, bits, G):
    geo = geometry(bits, G)
    M, K, C = p["M"], p["K"], p["C"]
    MT = 1 if M <= 8 else (2 if M <= 16 else 4)
    assert p["RT"] * p["SKW"] == 16
    assert 2 <= p["depth"] <= 32
    assert p["smem"] <= B200_SMEM_OPTIN
    assert p["off_ring"] >= 1024 and p["off_ring"] % 1024 == 0
    assert p["stage_bytes"] % 1024 == 0
    sg = p["stage_k"] // G
    assert p["stage_k"] == p["SKW"] * p["BPW"] * geo["box_k"]
    assert p["stage_k"] % G == 0
    rs = p["row_stride"]
    seg_max = p["stage_k"] * bits // 8
    assert rs % 16 == 0 and rs >= seg_max and rs % 64 == 0     # padded to an odd multiple of 64 when it fits
    if p["contig"]:
        # whole rows arrive by single copies: dense rows, all groups' metadata
        assert C == 1 and p["stage_k"] == K and rs == seg_max and p["meta_tma"]
        assert sg == p["ngroups"] and 16 * p["ngroups"] * 2 % 16 == 0
    codes_bytes = p["RT"] * 16 * rs
    meta_rt = 16 * sg * 2
    assert p["meta_offset"] >= codes_bytes and p["meta_offset"] % 128 == 0
    if p["meta_tma"]:
        assert meta_rt % 128 == 0       # TMA destinations stay 128-byte aligned
    assert p["meta_offset"] + 2 * p["RT"] * meta_rt <= p["stage_bytes"]
    assert p["off_ring"] + p["depth"] * p["stage_bytes"] <= p["off_x"]
    xrow = p["x_row_stride"]
    assert xrow % 64 == 0 and xrow >= 2 * p["kc"]
    assert p["off_x"] + xrow * (M + 1) <= p["off_sx"]      # + the zero row
    assert p["off_sx"] + (p["kc"] // G) * 8 * MT * 4 <= p["off_red"]
    clusters = p["grid"] // C
    assert p["grid"] % C == 0 and clusters >= 1 and C <= 16
    per_cluster = -(-p["items"] // clusters)
    assert p["red_bufs"] in (0, 1, 2)
    red_slots = per_cluster if p["red_bufs"] == 0 else p["red_bufs"]
    assert p["off_red"] + red_slots * 16 * 16 * M * 4 <= p["off_part"]
    if C > 1:
        assert p["off_part"] + per_cluster * p["RT"] * 16 * M * 4 <= p["smem"]
    assert p["kc"] % max(geo["box_k"], G) == 0
    assert (C - 1) * p["kc"] < K <= C * p["kc"]
    if p["meta_tma"]:
        assert p["ngroups"] % 8 == 0 and sg % 8 == 0 and (p["kc"] // G) % 8 == 0

    cpq = geo["Qk"] // 8       # 8-k chunks per lane quarter of a sub-unit
    for rank in range(C):
        k_begin = rank * p["kc"]
        k_end = min(K, k_begin + p["kc"])
        nchunks = (k_end - k_begin) // 32
        assert nchunks * 64 <= xrow
        # staging: k -> (chunk, quarter, element of the 16-byte chunk)
        placed = {}
        perm = [0, 4, 1, 5, 2, 6, 3, 7] if bits == 4 else list(range(8))
        for r in range(0, k_end - k_begin, 8):
            su, rr = divmod(r, geo["Uk"])
            tq, rq = divmod(rr, geo["Qk"])
            chunk = su * cpq + rq // 8
            assert chunk < nchunks and tq < 4
            for e8 in range(8):
                key = (chunk, tq, e8)
                assert key not in placed
                placed[key] = k_begin + r + perm[e8]
        assert len(placed) == k_end - k_begin
        # group sums: the G/8 threads of a group are consecutive
        assert (k_end - k_begin) % G == 0 and 32 % (G // 8) == 0
        # consumers: every step pairs x[k] with the code of weight k
        used = 0
        for st in range(p["stages_per_item"]):
            stage_k0 = k_begin + st * p["stage_k"]
            if stage_k0 < k_end:           # producer: one bulk copy per row
                seg = min(p["stage_k"], k_end - stage_k0) * bits // 8
                assert 0 < seg <= seg_max and seg % 16 == 0 and (stage_k0 * bits // 8) % 16 == 0
            g0 = stage_k0 // G
            for sk in range(p["SKW"]):
                for bb in range(p["BPW"]):
                    kb = stage_k0 + (sk * p["BPW"] + bb) * geo["box_k"]
                    if kb >= k_end:
                        break
                    for j in range(geo["subunits"]):
                        ksu = kb + j * geo["Uk"]
                        if ksu >= k_end:
                            break
                        assert j * geo["U"] + 3 * geo["QB"] + geo["QB"] <= 64
                        # this warp's column block, row g+8 of the last row tile
                        col = (sk * p["BPW"] + bb) * 64 + j * geo["U"] + 3 * geo["QB"]
                        last = (p["RT"] - 1) * 16 * rs + 15 * rs + col + geo["QB"]
                        assert col + geo["QB"] <= seg_max and last <= codes_bytes
                        chunk0 = (ksu - k_begin) // geo["Uk"] * cpq
                        for t in range(4):
                            qbase = ksu + t * geo["Qk"]
                            if bits == 4:
                                for wi in range(geo["words"]):
                                    for h in range(2):
                                        nib = [2 * h, 2 * h + 4, 2 * h + 1, 2 * h + 5]
                                        for e in range(4):
                                            k = qbase + 8 * wi + nib[e]
                                            assert placed[(chunk0 + wi, t, 4 * h + e)] == k
                                            used += 1
                            else:
                                assert geo["words"] % 2 == 0
                                for wi in range(0, geo["words"], 2):
                                    for half in range(2):
                                        for e in range(4):
                                            k = qbase + 4 * (wi + half) + e
                                            assert placed[(chunk0 + wi // 2, t, 4 * half + e)] == k
                                            used += 1
                        if (ksu + geo["Uk"]) % G == 0:
                            gi = (ksu + geo["Uk"]) // G - 1
                            assert 0 <= gi - g0 < sg
                            assert 0 <= gi - k_begin // G < p["kc"] // G
        assert used == k_end - k_begin, (used, k_end - k_begin)


CASES = (
    [(1, 256, 512, 4, 128), (1, 4096, 4096, 4, 128), (1, 1024, 4096, 4, 128),
     (1, 14336, 4096, 4, 128), (1, 4096, 14336, 4, 128)]
    + [(m, 14336, 4096, b, g) for m in (1, 2, 4, 8, 16, 32) for b in (4, 8) for g in (32, 64, 128)]
    + [(m, n, k, b, g) for (m, n, k) in [(1, 1, 32), (3, 17, 64), (5, 300, 1024), (1, 1000, 4160),
                                          (32, 33, 4096), (16, 4096, 14336), (32, 4096, 14336)]
       for b in (4, 8) for g in (32, 64, 128) if k % g == 0]
)


@pytest.mark.parametrize("M,N,K,bits,G", CASES)
def test_plan_and_indices(lib, M, N, K, bits, G):
    check_plan(plan(lib, M, N, K, bits, G), bits, G)


@pytest.mark.parametrize("cap", [1, 5, 17])
def test_plan_with_fewer_resident_clusters(lib, cap):
    for bits, G in ((4, 128), (8, 128), (4, 32)):
        p = plan(lib, 4, 1024, 4096, bits, G, cap=cap)
        assert p["grid"] // p["C"] <= cap
        check_plan(p, bits, G)


@pytest.mark.parametrize("C,bpw,depth", [(1, 1, 0), (1, 2, 0), (2, 1, 0), (2, 2, 0), (4, 1, 0),
                                         (4, 2, 0), (1, 2, 3), (2, 1, 4)])
def test_forced_plans(lib, C, bpw, depth):
    """Plans forced through the tuning hook obey the same bounds."""
    lib.wq_internal_force_gemv_plan.argtypes = [ctypes.c_int] * 3
    try:
        lib.wq_internal_force_gemv_plan(C, bpw, depth)
        for shape in [(1, 14336, 4096, 4, 128), (1, 4096, 4096, 4, 128), (4, 1024, 4096, 8, 64)]:
            p = plan(lib, *shape)
            if depth:
                assert p["depth"] == min(depth, p["depth"])
            check_plan(p, shape[3], shape[4])
    finally:
        lib.wq_internal_force_gemv_plan(0, 0, 0)
