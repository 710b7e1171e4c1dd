"""CPU oracle for groupwise affine weight quantization and the W4A16 matmul.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the library under
``w4a16_decode_matmul_b200`` never does, and shares no code with it.

Two parts:

* ``oracle.c`` (loaded here through ctypes): the storage-mode reference the
  CUDA path must match -- binary16 weights in, packed codes, binary16 scales
  and binary16 integer zeros out; dequantization and the matmul in double.
* ``oracle.paper``: the pages' own Python-float semantics ("paper mode"),
  used for the worked examples.
* the nested-superblock quantizer (page 2's Q4_K figure; 4.5 bits per
  weight) in ``oracle.c``, pinned by ``tests/test_oracle_q4k.py``.
* ``oracle.snr_table``: information-only error and traffic tables.

Every function states the passage it follows in its docstring or in the C
source.  Parity of the storage-mode quantizer is pinned by exact-rational
recomputation, the error bound, exact zero and brute-force nearest-code
tests; the matmul by one-hot/zero inputs, exact-rational sums and page 2's
K-major per-group formulation (see ``tests/test_oracle_pins.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-std=c11", "-shared", "-fPIC"]

_lock = threading.Lock()


def build(source: str = SOURCE, output: str = LIBRARY, force: bool = False) -> str:
    """Compile the C oracle with gcc (no FMA contraction, no fast math)."""
    with _lock:
        if (not force and os.path.exists(output)
                and os.path.getmtime(output) >= os.path.getmtime(source)):
            return output
        tmp = output + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, source, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, output)
        return output


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes handle on one compiled copy of ``oracle.c``."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.oracle_quantize.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp, vp, vp]
        lib.oracle_quantize.restype = None
        lib.oracle_dequantize.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, vp]
        lib.oracle_dequantize.restype = None
        lib.oracle_matmul.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, i32, i32, vp, vp]
        lib.oracle_matmul.restype = None
        lib.oracle_matmul_at.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, i32, i32,
                                         vp, vp, i64, vp, vp]
        lib.oracle_matmul_at.restype = None
        lib.oracle_matmul_dense_bf16.argtypes = [vp, i64, vp, i64, i64, vp]
        lib.oracle_matmul_dense_bf16.restype = None
        lib.oracle_q4k_quantize.argtypes = [vp, i64, i64, vp]
        lib.oracle_q4k_quantize.restype = None
        lib.oracle_q4k_dequantize.argtypes = [vp, i64, i64, vp]
        lib.oracle_q4k_dequantize.restype = None
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_half_round_up.argtypes = [ctypes.c_double]
        lib.oracle_half_round_up.restype = ctypes.c_uint16
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = None
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def set_threads(self, n: int) -> None:
        """Threads of the OpenMP loops (timing only; no effect on results)."""
        self.lib.oracle_set_threads(int(n))

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    # -- quantize ----------------------------------------------------------
    def quantize(self, W_half_bits: np.ndarray, bits: int, group: int,
                 symmetric: bool, pack: bool = True):
        """Storage-mode quantizer (page 1 section 1; page 2 "解法" when
        symmetric).  ``W_half_bits`` is uint16 [N, K] (binary16 patterns).

        Returns ``(q, codes, scales, zeros)``: int32 codes [N, K] (signed for
        symmetric), packed bytes [N, K*bits/8], binary16 scale patterns and
        binary16 zero patterns [N, K/group] (``zeros`` is None if symmetric).
        With ``pack=False`` no bytes are produced (``codes`` is None), which
        allows an odd K.
        """
        W = np.ascontiguousarray(W_half_bits, dtype=np.uint16)
        N, K = W.shape
        assert bits in (4, 8) and K % group == 0
        assert not pack or (K * bits) % 8 == 0
        q = np.empty((N, K), dtype=np.int32)
        codes = np.zeros((N, K * bits // 8), dtype=np.uint8) if pack else None
        scales = np.empty((N, K // group), dtype=np.uint16)
        zeros = np.empty((N, K // group), dtype=np.uint16)
        self.lib.oracle_quantize(_p(W), N, K, bits, group, int(bool(symmetric)),
                                 _p(q), _p(codes) if pack else None, _p(scales),
                                 _p(zeros))
        return q, codes, scales, (None if symmetric else zeros)

    # -- dequantize --------------------------------------------------------
    def dequantize(self, codes, scales, zeros, N: int, K: int, bits: int,
                   group: int, symmetric: bool) -> np.ndarray:
        """What = s * (q - z) in double, [N, K] (page 1 section 1)."""
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        zp = (np.zeros_like(scales) if zeros is None
              else np.ascontiguousarray(zeros, dtype=np.uint16))
        out = np.empty((N, K), dtype=np.float64)
        self.lib.oracle_dequantize(_p(codes), _p(scales), _p(zp), N, K, bits, group,
                                   int(bool(symmetric)), _p(out))
        return out

    # -- nested superblocks -----------------------------------------------
    Q4K_BLOCK_BYTES = 144  # per 256 weights: 4.5 bits per weight

    def q4k_quantize(self, W_half_bits: np.ndarray) -> np.ndarray:
        """Superblock quantizer (page 2 "量化", the Q4_K figure; the reading is
        stated in oracle.c).  ``W_half_bits`` is uint16 [N, K], K a multiple of
        256.  Returns the blocks, uint8 [N, K/256 * 144]."""
        W = np.ascontiguousarray(W_half_bits, dtype=np.uint16)
        N, K = W.shape
        assert K % 256 == 0
        blocks = np.zeros((N, K // 256 * self.Q4K_BLOCK_BYTES), dtype=np.uint8)
        self.lib.oracle_q4k_quantize(_p(W), N, K, _p(blocks))
        return blocks

    def q4k_dequantize(self, blocks: np.ndarray, N: int, K: int) -> np.ndarray:
        """What = S_j q - M_j in double, [N, K], from the blocks' bytes."""
        blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
        assert blocks.shape == (N, K // 256 * self.Q4K_BLOCK_BYTES)
        out = np.empty((N, K), dtype=np.float64)
        self.lib.oracle_q4k_dequantize(_p(blocks), N, K, _p(out))
        return out

    def q4k_matmul(self, X_bf16_bits, blocks: np.ndarray, N: int, K: int):
        """``(Y, Yabs)`` for superblock weights: Y = X What^T and sum |x w|
        per output, in double."""
        X = np.asarray([self.lib.oracle_bf16_to_double(int(v)) for v in
                        np.asarray(X_bf16_bits, dtype=np.uint16).ravel()],
                       dtype=np.float64).reshape(-1, K)
        Wh = self.q4k_dequantize(blocks, N, K)
        return X @ Wh.T, np.abs(X) @ np.abs(Wh).T

    # -- matmul ------------------------------------------------------------
    def matmul(self, X_bf16_bits, codes, scales, zeros, N: int, K: int, bits: int,
               group: int, symmetric: bool):
        """``(Y, Yabs)``: Y = X What^T and the sum of |x*w| per output, in
        double ([M, N] each)."""
        X = np.ascontiguousarray(X_bf16_bits, dtype=np.uint16)
        M = X.shape[0]
        assert X.shape[1] == K
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        zp = (np.zeros_like(scales) if zeros is None
              else np.ascontiguousarray(zeros, dtype=np.uint16))
        Y = np.empty((M, N), dtype=np.float64)
        Yabs = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_matmul(_p(X), M, _p(codes), _p(scales), _p(zp), N, K, bits,
                               group, int(bool(symmetric)), _p(Y), _p(Yabs))
        return Y, Yabs

    def matmul_at(self, X_bf16_bits, codes, scales, zeros, N: int, K: int, bits: int,
                  group: int, symmetric: bool, ms, ns):
        """The same sums for chosen output coordinates (ms[i], ns[i])."""
        X = np.ascontiguousarray(X_bf16_bits, dtype=np.uint16)
        M = X.shape[0]
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        ns = np.ascontiguousarray(ns, dtype=np.int64)
        assert ms.shape == ns.shape
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        zp = (np.zeros_like(scales) if zeros is None
              else np.ascontiguousarray(zeros, dtype=np.uint16))
        y = np.empty(ms.shape, dtype=np.float64)
        yabs = np.empty(ms.shape, dtype=np.float64)
        self.lib.oracle_matmul_at(_p(X), M, _p(codes), _p(scales), _p(zp), N, K, bits,
                                  group, int(bool(symmetric)), _p(ms), _p(ns),
                                  ms.size, _p(y), _p(yabs))
        return y, yabs

    def matmul_dense_bf16(self, X_bf16_bits, B_bf16_bits):
        """Y = X B^T in double for bfloat16 X [M, K] and B [N, K]."""
        X = np.ascontiguousarray(X_bf16_bits, dtype=np.uint16)
        B = np.ascontiguousarray(B_bf16_bits, dtype=np.uint16)
        M, K = X.shape
        N = B.shape[0]
        assert B.shape[1] == K
        Y = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_matmul_dense_bf16(_p(X), M, _p(B), N, K, _p(Y))
        return Y

    # -- scalar helpers (for the decoder pins) ------------------------------
    def half_to_double(self, h: int) -> float:
        return self.lib.oracle_half_to_double(h)

    def half_round_up(self, x: float) -> int:
        return self.lib.oracle_half_round_up(x)

    def bf16_to_double(self, b: int) -> float:
        return self.lib.oracle_bf16_to_double(b)


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle compiled from this directory's ``oracle.c`` (built on first
    use when missing or stale)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default
