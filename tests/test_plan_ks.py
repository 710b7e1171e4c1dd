"""Host-side plan of the k-sliced direct-load small-batch kernel (no GPU):
scope (4-bit, group 128, K = 4096, M <= 4), grid, ring depth, and the
shared-memory layout -- the (scale, 128 + zero) table, the per-warp partial
sums and the per-warp rings -- disjoint, aligned, and at most half an SM."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")
FIELDS = ["M", "N", "tiles", "off_sz", "off_part", "off_ring", "depth", "smem", "grid"]
SMEM_OPTIN, SMS = 232448, 148
WARPS, TILE_ROWS = 16, 8


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.skip("libwq.so not built")
    lib = ctypes.CDLL(LIB)
    lib.wq_internal_plan_ks.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p]
    lib.wq_internal_plan_ks.restype = ctypes.c_int
    return lib


def plan(lib, M, N, K=4096, bits=4, group=128):
    out = (ctypes.c_int64 * 12)()
    ok = lib.wq_internal_plan_ks(M, N, K, bits, group, SMS, SMEM_OPTIN, out)
    return dict(zip(FIELDS, out[:len(FIELDS)])) if ok else None


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N", [14336, 4096, 1024, 28672, 1203, 5, 1])
def test_plan_layout(lib, M, N):
    p = plan(lib, M, N)
    tiles = -(-N // TILE_ROWS)
    mt = -(-tiles // min(tiles, SMS))
    fixed = -(-(mt * TILE_ROWS * 33 * 8) // 16) * 16 + mt * WARPS * TILE_ROWS * M * 4
    if -(-fixed // 128) * 128 + WARPS * 3 * 1024 > SMEM_OPTIN // 2 - 1024:
        assert p is None            # a ring of 3 units per warp would not fit: out of scope
        return
    assert p is not None
    assert p["tiles"] == -(-N // TILE_ROWS) and p["grid"] == min(p["tiles"], SMS)
    max_tiles = -(-p["tiles"] // p["grid"])
    assert p["off_sz"] == 0
    assert p["off_part"] >= max_tiles * TILE_ROWS * 33 * 8 and p["off_part"] % 16 == 0
    assert p["off_ring"] >= p["off_part"] + max_tiles * WARPS * TILE_ROWS * M * 4
    assert p["off_ring"] % 128 == 0
    assert 3 <= p["depth"] <= 5
    assert p["smem"] == p["off_ring"] + WARPS * p["depth"] * 1024
    assert p["smem"] <= SMEM_OPTIN // 2 - 1024


@pytest.mark.parametrize("M,N,K,bits,group", [(5, 100, 4096, 4, 128), (1, 100, 8192, 4, 128),
                                              (1, 100, 4096, 8, 128), (1, 100, 4096, 4, 64),
                                              (1, 100, 14336, 4, 128)])
def test_out_of_scope(lib, M, N, K, bits, group):
    assert plan(lib, M, N, K, bits, group) is None
