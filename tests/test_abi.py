"""The C-ABI library on the host (no GPU needed): it loads, exports every
entry point declared in include/*.h, computes the payload sizes of page 1
section 2, and rejects bad arguments before touching the device."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "w4a16_decode_matmul_b200", "libwq.so")


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from w4a16_decode_matmul_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("wq_quantize", "wq_matmul", "wq_dequantize", "wq_codes_bytes",
                     "wq_meta_elems", "wq_get_device_error", "wq_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_payload_sizes_match_page_1(lib):
    lib.wq_codes_bytes.restype = ctypes.c_size_t
    lib.wq_codes_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
    lib.wq_meta_elems.restype = ctypes.c_size_t
    lib.wq_meta_elems.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
    # page 1 section 2: 1024 INT4 @ group 128 -> 512 + 8*(2+2) = 544 B;
    # 4096 INT4 @ group 64 -> 2048 + 64*4 = 2304 B
    assert lib.wq_codes_bytes(1, 1024, 4) + 4 * lib.wq_meta_elems(1, 1024, 128) == 544
    assert lib.wq_codes_bytes(1, 4096, 4) + 4 * lib.wq_meta_elems(1, 4096, 64) == 2304
    assert lib.wq_codes_bytes(14336, 4096, 4) == 29360128
    assert lib.wq_meta_elems(14336, 4096, 128) == 14336 * 32
    assert lib.wq_codes_bytes(2, 64, 8) == 128
    assert lib.wq_codes_bytes(0, 64, 4) == 0 and lib.wq_codes_bytes(4, 64, 3) == 0
    assert lib.wq_meta_elems(4, 100, 32) == 0


def test_superblock_sizes(lib):
    """Page 2's superblock budget: 4.5 bits per weight, 144 bytes per 256."""
    lib.wq_q4k_bytes.restype = ctypes.c_size_t
    lib.wq_q4k_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
    assert lib.wq_q4k_bytes(1, 256) == 144
    assert lib.wq_q4k_bytes(14336, 4096) == 14336 * 4096 * 9 // 16  # 4.5 / 8 bytes per weight
    assert lib.wq_q4k_bytes(1, 384) == 0 and lib.wq_q4k_bytes(0, 256) == 0
    assert lib.wq_q4k_bytes(3, 128) == 0


def test_superblock_rejections_without_gpu(lib):
    """Host checks come before any device work: invalid sizes, M and
    alignment are refused with nothing launched."""
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.wq_q4k_quantize.argtypes = [vp, i64, i64, vp, vp]
    lib.wq_q4k_quantize.restype = ctypes.c_int
    lib.wq_q4k_matmul.argtypes = [vp, i64, vp, i64, i64, vp, ctypes.c_int, vp]
    lib.wq_q4k_matmul.restype = ctypes.c_int
    buf = ctypes.create_string_buffer(4096 + 32)
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    assert lib.wq_q4k_quantize(base, 4, 384, base, None) == 1      # K % 256
    assert lib.wq_q4k_quantize(None, 4, 256, base, None) == 1      # null W
    assert lib.wq_q4k_quantize(base + 2, 1, 256, base, None) == 3  # misaligned
    assert lib.wq_q4k_matmul(base, 9, base, 4, 256, base, 0, None) == 1   # M > 8
    assert lib.wq_q4k_matmul(base, 1, base, 4, 256, base, 7, None) == 1   # out dtype
    assert lib.wq_q4k_matmul(base, 1, base + 8, 4, 256, base, 0, None) == 3
    lib.wq_q4k_matmul_ex.argtypes = [vp, i64, vp, i64, i64, vp, ctypes.c_int, ctypes.c_uint, vp]
    lib.wq_q4k_matmul_ex.restype = ctypes.c_int
    assert lib.wq_q4k_matmul_ex(base, 1, base, 4, 256, base, 0, 2, None) == 1   # unknown flag
    assert lib.wq_q4k_matmul_ex(base, 9, base, 4, 256, base, 0, 1, None) == 1   # M > 8
    assert lib.wq_q4k_matmul_ex(base, 1, base + 8, 4, 256, base, 0, 1, None) == 3


def test_status_strings(lib):
    lib.wq_status_string.restype = ctypes.c_char_p
    lib.wq_status_string.argtypes = [ctypes.c_int]
    assert lib.wq_status_string(0) == b"ok"
    assert lib.wq_status_string(5) == b"device wait timed out"
    lib.wq_version.restype = ctypes.c_char_p
    assert b"sm_100a" in lib.wq_version()


def _quantize_args(lib):
    f = lib.wq_quantize
    f.restype = ctypes.c_int
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    f.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp, vp, vp]
    return f


def test_quantize_rejects_bad_arguments_before_launch(lib):
    q = _quantize_args(lib)
    p = ctypes.c_void_p(1 << 20)            # never dereferenced: checks fail first
    bad = ctypes.c_void_p((1 << 20) + 2)
    assert q(p, 16, 100, 4, 32, 0, p, p, p, None) == 1       # K not a multiple of 32
    assert q(p, 16, 128, 3, 32, 0, p, p, p, None) == 1       # bits
    assert q(p, 16, 128, 4, 48, 0, p, p, p, None) == 1       # group
    assert q(p, 0, 128, 4, 32, 0, p, p, p, None) == 1        # N
    assert q(p, 16, 128, 4, 32, 0, p, p, None, None) == 1    # asymmetric needs zeros
    assert q(p, 16, 128, 4, 32, 1, p, p, p, None) == 1       # symmetric takes no zeros
    assert q(p, 16, 128, 4, 32, 2, p, p, None, None) == 1    # symmetric flag
    assert q(bad, 16, 128, 4, 32, 0, p, p, p, None) == 3     # alignment
    assert q(p, 16, 128, 4, 32, 0, p, bad, p, None) == 3


def test_matmul_rejects_bad_arguments_before_launch(lib):
    f = lib.wq_matmul
    f.restype = ctypes.c_int
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    sz, u32 = ctypes.c_size_t, ctypes.c_uint
    f.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, i32, i32, vp, i32, vp, sz, u32, vp]
    p = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    assert f(p, 0, p, p, p, 64, 128, 4, 32, 0, p, 0, None, 0, 0, None) == 1      # M
    assert f(p, 1, p, p, p, 64, 128, 4, 32, 0, p, 7, None, 0, 0, None) == 1      # out dtype
    assert f(p, 1, p, p, None, 64, 128, 4, 32, 0, p, 0, None, 0, 0, None) == 1   # zeros missing
    assert f(p, 1, p, p, p, 64, 120, 4, 32, 0, p, 0, None, 0, 0, None) == 1      # K
    assert f(p, 1, p, p, p, 64, 128, 4, 32, 0, p, 0, None, 0, 2, None) == 1      # flags
    assert f(p, 1, p, p, p, 64, 128, 4, 32, 0, p, 0, None, 64, 0, None) == 1     # bytes, no buffer
    assert f(bad, 1, p, p, p, 64, 128, 4, 32, 0, p, 0, None, 0, 0, None) == 3    # X alignment
    assert f(p, 1, p, p, p, 64, 128, 4, 32, 0, bad, 0, None, 0, 0, None) == 3    # Y alignment
    assert f(p, 1, p, p, p, 64, 128, 4, 32, 0, p, 0, bad, 1 << 20, 0, None) == 3  # workspace


def test_workspace_size(lib):
    f = lib.wq_matmul_workspace_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = []
    # flags for 1024 CTAs + 1024 x 16 rows x 8 activation rows of binary32 partials
    assert f() == 1024 * 4 + 1024 * 128 * 4


def test_dequantize_rejects_bad_arguments_before_launch(lib):
    f = lib.wq_dequantize
    f.restype = ctypes.c_int
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    f.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, vp, vp]
    p = ctypes.c_void_p(1 << 20)
    assert f(p, p, p, 4, 96, 4, 64, 0, p, None) == 1     # K % group
    assert f(p, p, None, 4, 128, 8, 64, 0, p, None) == 1
    assert f(p, p, p, 4, 128, 4, 64, 0, ctypes.c_void_p((1 << 20) + 4), None) == 3
