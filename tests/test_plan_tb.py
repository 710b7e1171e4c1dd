"""Host-side plan of the bulk-staged small-batch kernel (no GPU): scope,
grid, ring depth and the shared-memory layout -- partial sums, staged
activations and group sums (when K is more than one chunk), the ring of
17,408-byte stages -- disjoint, aligned for TMA, and no larger than half an
SM, so that the next launch's CTA fits beside it."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")
FIELDS = ["M", "N", "K", "ngroups", "pairs", "nch", "tiles", "depth", "xs_row_bytes", "off_part",
          "off_x", "off_sx", "off_ring", "smem", "grid", "xreg"]
SMEM_OPTIN, SMS = 232448, 148
WARPS, TILE_ROWS, STAGE = 8, 8, 17408


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.skip("libwq.so not built")
    lib = ctypes.CDLL(LIB)
    lib.wq_internal_plan_tb.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p]
    lib.wq_internal_plan_tb.restype = ctypes.c_int
    return lib


def plan(lib, M, N, K, bits=4, group=128):
    out = (ctypes.c_int64 * 20)()
    ok = lib.wq_internal_plan_tb(M, N, K, bits, group, SMS, SMEM_OPTIN, out)
    return dict(zip(FIELDS, out[:len(FIELDS)])) if ok else None


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 4096), (1024, 4096), (4096, 14336),
                                 (1000, 4096), (77, 1024), (1, 1024), (28672, 4096),
                                 (1201, 8192), (300, 2048)])
def test_plan_layout(lib, M, N, K):
    p = plan(lib, M, N, K)
    tiles = -(-N // TILE_ROWS)
    grid = min(tiles, SMS)
    fixed = 1024 + -(-tiles // grid) * WARPS * TILE_ROWS * M * 4
    if K > 4096:       # activations staged in shared memory
        fixed += M * (2 * K + 64) + M * (K // 128) * 4 + 1024
    if fixed + 3 * STAGE > SMEM_OPTIN // 2 - 1024:
        assert p is None            # a ring of 3 stages would not fit: out of scope
        return
    assert p is not None
    assert p["ngroups"] == K // 128 and p["pairs"] == K // 256
    assert p["nch"] == -(-p["pairs"] // 16) and p["xreg"] == (p["nch"] == 1)
    assert p["tiles"] == -(-N // TILE_ROWS) and p["grid"] == min(p["tiles"], SMS)
    max_tiles = -(-p["tiles"] // p["grid"])
    assert p["off_part"] >= 1024
    part_end = p["off_part"] + max_tiles * WARPS * TILE_ROWS * M * 4
    if p["xreg"]:
        x_end = part_end
    else:
        assert p["off_x"] >= part_end and p["off_x"] % 16 == 0
        assert p["xs_row_bytes"] == 2 * K + 64
        assert p["off_sx"] >= p["off_x"] + M * p["xs_row_bytes"]
        x_end = p["off_sx"] + M * p["ngroups"] * 4
    # the ring: TMA destinations 128-byte aligned, whole stages
    assert p["off_ring"] >= x_end and p["off_ring"] % 1024 == 0 and STAGE % 128 == 0
    assert 3 <= p["depth"] <= 8
    assert p["smem"] == p["off_ring"] + p["depth"] * STAGE
    # at most half an SM (1 KB reserved per CTA): two launches' CTAs fit together
    assert p["smem"] <= SMEM_OPTIN // 2 - 1024


@pytest.mark.parametrize("M,N,K,bits,group", [(5, 100, 4096, 4, 128), (1, 100, 4096, 8, 128),
                                              (1, 100, 4096, 4, 64), (1, 100, 1536, 4, 128),
                                              (1, 100, 512, 4, 128)])
def test_out_of_scope(lib, M, N, K, bits, group):
    assert plan(lib, M, N, K, bits, group) is None
