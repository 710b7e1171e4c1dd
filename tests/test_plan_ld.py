"""Host-side plan of the direct-load small-batch kernel (no GPU): scope,
grid, and the shared-memory layout every launch relies on -- the activation
rows, group sums, the CTA's (scale, zero) table, the per-warp partial sums and
the per-warp rings of codes, disjoint, aligned, and inside the opt-in limit
(for every CTA's share of 8-row tiles)."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")
FIELDS = ["M", "N", "K", "ngroups", "tiles", "xs_row_bytes", "off_sx", "off_sz", "off_part",
          "off_ring", "smem", "grid"]
SMEM_OPTIN, SMS = 232448, 148
WARPS, DEPTH, TILE_ROWS = 16, 3, 8


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.skip("libwq.so not built")
    lib = ctypes.CDLL(LIB)
    lib.wq_internal_plan_ld.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p]
    lib.wq_internal_plan_ld.restype = ctypes.c_int
    return lib


def plan(lib, M, N, K, bits=4, group=128, sms=SMS):
    out = (ctypes.c_int64 * 16)()
    ok = lib.wq_internal_plan_ld(M, N, K, bits, group, sms, SMEM_OPTIN, out)
    return dict(zip(FIELDS, out[:len(FIELDS)])) if ok else None


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 4096), (1024, 4096), (4096, 14336),
                                 (1000, 4096), (77, 1024), (1, 512), (28672, 4096)])
def test_plan_layout(lib, M, N, K):
    p = plan(lib, M, N, K)
    assert p is not None
    ng = K // 128
    tiles = -(-N // TILE_ROWS)
    assert p["ngroups"] == ng and p["tiles"] == tiles
    assert p["grid"] == min(tiles, SMS)
    max_tiles = -(-tiles // p["grid"])
    # every CTA's share (floor split) is at most max_tiles
    shares = [(b + 1) * tiles // p["grid"] - b * tiles // p["grid"] for b in range(p["grid"])]
    assert max(shares) <= max_tiles and sum(shares) == tiles
    assert p["xs_row_bytes"] == 2 * K + 64 and p["xs_row_bytes"] % 128 == 64
    regions = [(0, M * p["xs_row_bytes"]), (p["off_sx"], M * ng * 4),
               (p["off_sz"], max_tiles * TILE_ROWS * (ng + 1) * 8),
               (p["off_part"], max_tiles * WARPS * TILE_ROWS * M * 4),
               (p["off_ring"], WARPS * DEPTH * 1024)]
    for (a, n), (b, _) in zip(regions, regions[1:]):
        assert a + n <= b and b % 16 == 0
    assert p["off_ring"] % 128 == 0
    assert p["smem"] == p["off_ring"] + WARPS * DEPTH * 1024 <= SMEM_OPTIN


@pytest.mark.parametrize("M,N,K,bits,group", [
    (5, 14336, 4096, 4, 128),    # more tokens than the B columns hold
    (1, 14336, 4096, 8, 128),    # 8-bit codes
    (1, 14336, 4096, 4, 64),     # other group sizes
    (1, 14336, 4096, 4, 32),
    (1, 14336, 384, 4, 128),     # K not a multiple of 512
    (1, 14336, 4224, 4, 128),
    (4, 1 << 20, 16384, 4, 128),  # a CTA's share too large for shared memory
])
def test_plan_out_of_scope(lib, M, N, K, bits, group):
    assert plan(lib, M, N, K, bits, group) is None
