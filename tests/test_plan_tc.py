"""Host-side plan of the tensor-memory small-batch kernel (no GPU): scope
(4- or 8-bit codes, group 128, K = 4096, M <= 2), grid, ring depth (4 stages
of 2 KB per warp for 4-bit codes, 2 of 4 KB for 8-bit), and the
shared-memory layout -- the swizzled activation operand (1,024-aligned,
as the 128-byte swizzle needs), the (scale, 128 + zero) table, the per-warp
partial sums and the per-warp rings -- disjoint, aligned, and at most half
an SM, so that two CTAs (and two 256-column tensor-memory allocations) fit
on one SM."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")
FIELDS = ["M", "N", "tiles", "off_b", "off_sz", "off_part", "off_ring", "depth", "smem", "grid"]
SMEM_OPTIN, SMS = 232448, 148
WARPS, TILE_ROWS, SZ_STRIDE = 8, 8, 36
DEPTH = {4: 4, 8: 2}
SLOT = {4: 2048, 8: 4096}


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.skip("libwq.so not built")
    lib = ctypes.CDLL(LIB)
    lib.wq_internal_plan_tc.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p]
    lib.wq_internal_plan_tc.restype = ctypes.c_int
    return lib


def plan(lib, M, N, K=4096, bits=4, group=128, sms=SMS):
    out = (ctypes.c_int64 * 12)()
    ok = lib.wq_internal_plan_tc(M, N, K, bits, group, sms, SMEM_OPTIN, out)
    return dict(zip(FIELDS, out[:len(FIELDS)])) if ok else None


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("N", [14336, 4096, 1024, 28672, 1203, 5, 1])
def test_plan_layout(lib, M, N, bits):
    p = plan(lib, M, N, bits=bits)
    tiles = -(-N // TILE_ROWS)
    mt = -(-tiles // min(tiles, SMS))
    fixed = 1024 + 4 * 16 * M * 128 + -(-(mt * TILE_ROWS * SZ_STRIDE * 4) // 16) * 16 \
        + mt * 8 * TILE_ROWS * M * 4
    if -(-fixed // 128) * 128 + WARPS * DEPTH[bits] * SLOT[bits] > SMEM_OPTIN // 2 - 1024:
        assert p is None            # the ring would not fit in half an SM: out of scope
        return
    assert p is not None
    assert p["tiles"] == tiles and p["grid"] == min(tiles, SMS)
    max_tiles = -(-tiles // p["grid"])
    # activation operand: 2 halves x 2 boxes x 16 M rows x 128 bytes
    assert p["off_b"] == 1024 and p["off_b"] % 1024 == 0
    assert p["off_sz"] == p["off_b"] + 4 * 16 * M * 128
    assert p["off_part"] >= p["off_sz"] + max_tiles * TILE_ROWS * SZ_STRIDE * 4
    assert p["off_part"] % 16 == 0
    assert p["off_ring"] >= p["off_part"] + max_tiles * 8 * TILE_ROWS * M * 4
    assert p["off_ring"] % 128 == 0
    assert p["depth"] == DEPTH[bits]
    assert p["smem"] == p["off_ring"] + WARPS * p["depth"] * SLOT[bits]
    assert p["smem"] <= SMEM_OPTIN // 2 - 1024


def test_headline_shapes_in_scope(lib):
    """Both code widths at M = 1 and 2 on the Llama-8B layer shapes with
    K = 4096 fit in half an SM."""
    for bits in (4, 8):
        for M in (1, 2):
            for N in (4096, 1024, 14336):
                assert plan(lib, M, N, bits=bits) is not None


@pytest.mark.parametrize("M,N,K,bits,group", [(3, 100, 4096, 4, 128), (1, 100, 8192, 4, 128),
                                              (1, 100, 4096, 2, 128), (1, 100, 4096, 4, 64),
                                              (1, 100, 14336, 4, 128), (0, 100, 4096, 4, 128),
                                              (1, 0, 4096, 4, 128)])
def test_out_of_scope(lib, M, N, K, bits, group):
    assert plan(lib, M, N, K, bits, group) is None
