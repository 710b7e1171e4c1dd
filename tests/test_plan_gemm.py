"""Host-side check of the prefill kernel's plan (gemm.cuh): shared-memory
regions in bounds and aligned as the 128-byte swizzle and the tensor-core
descriptors need, copy boxes inside the TMA limits, and the scope the
kernel declares (group 64/128, whole 64-k stages, at most 256 groups)."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")
FIELDS = ["M", "N", "K", "ngroups", "tiles_m", "codes_stage_bytes", "meta_bytes", "off_a",
          "off_b", "off_codes", "off_meta_s", "off_meta_z", "off_stab", "smem", "grid"]
SMEM_OPTIN = 232448
BM, BN, BK, STAGES = 128, 128, 64, 4


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.skip("libwq.so not built")
    lib = ctypes.CDLL(LIB)
    lib.wq_internal_plan_gemm.restype = ctypes.c_int
    lib.wq_internal_plan_gemm.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_int64)]
    return lib


def plan(lib, M, N, K, bits, group, sym):
    out = (ctypes.c_int64 * 16)()
    ok = lib.wq_internal_plan_gemm(M, N, K, bits, group, int(sym), SMEM_OPTIN, out)
    return dict(zip(FIELDS, out[:len(FIELDS)])) if ok else None


CASES = [(M, N, K, bits, group, sym)
         for M in (33, 512, 2048, 8192)
         for (N, K) in ((14336, 4096), (4096, 4096), (300, 1024))
         for bits in (4, 8) for group in (64, 128) for sym in (False, True)]


@pytest.mark.parametrize("M,N,K,bits,group,sym", CASES)
def test_plan_gemm(lib, M, N, K, bits, group, sym):
    p = plan(lib, M, N, K, bits, group, sym)
    assert p is not None
    ng = K // group
    assert p["ngroups"] == ng and ng % 8 == 0 and ng <= 256
    assert p["tiles_m"] == -(-M // BM) and p["grid"] == p["tiles_m"] * -(-N // BN)
    tile = BM * BK * 2
    # swizzled tiles: 1024-byte aligned atoms, rings back to back
    assert p["off_a"] == 1024 and p["off_a"] % 1024 == 0
    assert p["off_b"] == p["off_a"] + STAGES * tile and p["off_b"] % 1024 == 0
    assert p["off_codes"] == p["off_b"] + STAGES * tile
    assert p["codes_stage_bytes"] == BN * BK * bits // 8
    # TMA destinations 128-byte aligned; boxes: codes rows of 32/64 bytes,
    # metadata rows of ngroups halves (a multiple of 16 bytes, <= 256 elements)
    for k in ("off_codes", "off_meta_s", "off_meta_z"):
        assert p[k] % 128 == 0
    assert (BK * bits // 8) % 16 == 0 and (ng * 2) % 16 == 0
    assert p["meta_bytes"] == BN * ng * 2
    assert p["off_meta_s"] >= p["off_codes"] + STAGES * p["codes_stage_bytes"]
    assert p["off_meta_z"] >= p["off_meta_s"] + p["meta_bytes"]
    assert p["off_stab"] >= p["off_meta_z"] + (0 if sym else p["meta_bytes"])
    assert p["off_stab"] % 16 == 0
    assert p["smem"] == p["off_stab"] + ng * BN * 4 <= SMEM_OPTIN
    # more than half the SM's shared memory: one CTA (and one TMEM
    # allocation of 256 columns) per SM
    assert p["smem"] > SMEM_OPTIN // 2


@pytest.mark.parametrize("M,N,K,bits,group", [(64, 256, 4096, 4, 32), (64, 256, 4160, 4, 64),
                                              (64, 256, 512, 4, 128), (64, 256, 65536, 4, 128)])
def test_out_of_scope(lib, M, N, K, bits, group):
    # group 32, K not a multiple of 64, fewer than 8 groups, more than 256
    assert plan(lib, M, N, K, bits, group, False) is None
