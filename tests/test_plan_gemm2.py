"""Host-side check of the plan of the prefill kernel that keeps the
dequantized weights in tensor memory (gemm2.cuh): shared-memory rings in
bounds and 1024-byte aligned (the 128-byte swizzle of the activation boxes
and the 64/128-byte swizzle of the code boxes), copy boxes inside the TMA
limits with 16-byte aligned inner extents, the epilogue's output staging
(8 warps x two 2 KB buffers, 1024-byte aligned, after the rings, where it
fits), the tile count and persistent grid, and the kernel's scope (groups 32/64/128, K a multiple of 128: a load
stage is 128 k, eight MMAs of K = 16)."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")
FIELDS = ["M", "N", "K", "ngroups", "tiles_t", "tiles_w", "num_tiles", "codes_stage_bytes",
          "smem", "grid", "off_out"]
SMEM_OPTIN, SMS = 232448, 148
BW = 128
BK, HEAD = 128, 1024


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.skip("libwq.so not built")
    lib = ctypes.CDLL(LIB)
    lib.wq_internal_plan_gemm2.restype = ctypes.c_int
    lib.wq_internal_plan_gemm2.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_int64)]
    return lib


def plan(lib, M, N, K, bits, group):
    out = (ctypes.c_int64 * 12)()
    ok = lib.wq_internal_plan_gemm2(M, N, K, bits, group, SMS, SMEM_OPTIN, out)
    return dict(zip(FIELDS, out[:len(FIELDS)])) if ok else None


CASES = [(M, N, K, bits, group)
         for M in (33, 64, 65, 129, 512, 2048, 8192)
         for (N, K) in ((14336, 4096), (4096, 14336), (300, 1024), (257, 384))
         for bits in (4, 8) for group in (32, 64, 128) if K % group == 0]


@pytest.mark.parametrize("M,N,K,bits,group", CASES)
def test_plan_gemm2(lib, M, N, K, bits, group):
    p = plan(lib, M, N, K, bits, group)
    assert p is not None
    # 64-token tiles (6 load stages) up to M = 64, 128-token tiles above
    BT, STAGES = (64, 6) if M <= 64 else (128, 4)
    assert p["ngroups"] == K // group
    assert p["tiles_t"] == -(-M // BT) and p["tiles_w"] == -(-N // BW)
    assert p["num_tiles"] == p["tiles_t"] * p["tiles_w"]
    assert p["grid"] == min(p["num_tiles"], SMS)
    # code boxes: 128 rows x (128 k of codes) = 64 or 128 bytes per row, a
    # multiple of 16 bytes, swizzled 64B / 128B (the swizzle span covers the
    # row); stage size a multiple of 1 KB
    row = BK * bits // 8
    assert row % 16 == 0 and row in (64, 128)
    assert p["codes_stage_bytes"] == BW * row and p["codes_stage_bytes"] % 1024 == 0
    # activation stage: two boxes of 64 k x BT tokens of bfloat16 (128-byte
    # rows, the 128-byte swizzle's span), each 1024-byte aligned
    x_box = BT * 64 * 2
    x_stage = 2 * x_box
    assert x_box % 1024 == 0 and x_stage == BT * BK * 2
    off_codes = HEAD + STAGES * x_stage
    assert off_codes % 1024 == 0
    # the ring of scale / zero blocks (8 slots of 128 rows x 8 groups x 2
    # tensors) when K / group is a multiple of 8 (the tensor maps' row pitch)
    meta = 8 * 2 * 128 * 8 * 2 if (K // group) % 8 == 0 else 0
    assert (off_codes + STAGES * p["codes_stage_bytes"]) % 128 == 0
    rings = off_codes + STAGES * p["codes_stage_bytes"] + meta
    staging = 8 * 2 * 16 * 32 * 4
    off_out = -(-rings // 1024) * 1024
    if off_out + staging <= SMEM_OPTIN:
        assert p["off_out"] == off_out and p["smem"] == off_out + staging
    else:
        assert p["off_out"] == 0 and p["smem"] == rings
    assert p["smem"] <= SMEM_OPTIN
    # 4-bit codes always leave room for the staging
    assert bits == 8 or p["off_out"] != 0
    # every TMA x coordinate (k * 2 bytes for X: stage start and start + 64;
    # bytes for the codes) stays a multiple of 16 bytes
    assert (BK * 2) % 16 == 0 and (64 * 2) % 16 == 0 and row % 16 == 0
    # the code tensor's row pitch is a multiple of 16 bytes (TMA stride rule)
    assert (K * bits // 8) % 16 == 0


@pytest.mark.parametrize("M,N,K,bits,group", [(64, 256, 4128, 4, 32), (64, 256, 96, 4, 32),
                                              (64, 256, 4160, 4, 32), (129, 256, 192, 8, 64),
                                              (64, 256, 4096, 2, 128)])
def test_out_of_scope(lib, M, N, K, bits, group):
    # K not a multiple of 128; unsupported code width
    assert plan(lib, M, N, K, bits, group) is None
