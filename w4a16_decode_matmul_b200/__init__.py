"""Python binding of ``libwq.so`` (the C ABI in ``include/wq.h``).

Argument marshalling only: every step of quantize, dequantize and matmul
runs in the library's CUDA kernels.  PyTorch provides device memory and the
current stream.  The library must have been built (``python
w4a16_decode_matmul_b200/build.py``); importing this package without it raises.

Functions keep the C names without the ``wq_`` prefix:

    codes, scales, zeros = quantize(W, bits=4, group=128, symmetric=False)
    Y = matmul(X, codes, scales, zeros, N, K, bits=4, group=128)
    W_hat = dequantize(codes, scales, zeros, N, K, bits=4, group=128)

``QuantizedWeight`` bundles the three tensors with their format.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libwq.so")

WQ_OK = 0
WQ_OUT_F32 = 0
WQ_OUT_BF16 = 1
WQ_MATMUL_STATIC_WEIGHTS = 1

STATUS_NAMES = {0: "WQ_OK", 1: "WQ_ERR_INVALID_ARG", 2: "WQ_ERR_UNSUPPORTED",
                3: "WQ_ERR_ALIGNMENT", 4: "WQ_ERR_CUDA", 5: "WQ_ERR_TIMEOUT"}


class WQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        detail = status_string(status)
        if status == 4:
            detail += ": " + lib.wq_internal_last_cuda_error().decode()
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({detail})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIBRARY_PATH):
        raise ImportError(
            f"{LIBRARY_PATH} is missing: build it with `python w4a16_decode_matmul_b200/build.py`")
    lib = ctypes.CDLL(LIBRARY_PATH)
    i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    lib.wq_codes_bytes.argtypes = [i64, i64, i32]
    lib.wq_codes_bytes.restype = sz
    lib.wq_meta_elems.argtypes = [i64, i64, i32]
    lib.wq_meta_elems.restype = sz
    lib.wq_quantize.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp, vp, vp]
    lib.wq_quantize.restype = i32
    lib.wq_dequantize.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, vp, vp]
    lib.wq_dequantize.restype = i32
    lib.wq_matmul_workspace_bytes.argtypes = []
    lib.wq_matmul_workspace_bytes.restype = sz
    lib.wq_matmul.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, i32, i32, vp, i32, vp, sz,
                              ctypes.c_uint, vp]
    lib.wq_matmul.restype = i32
    lib.wq_matmul_noalloc.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, i32, i32, vp, i32,
                                      ctypes.c_uint, vp]
    lib.wq_matmul_noalloc.restype = i32
    lib.wq_matmul_noalloc_scratch_bytes.argtypes = []
    lib.wq_matmul_noalloc_scratch_bytes.restype = sz
    lib.wq_q4k_bytes.argtypes = [i64, i64]
    lib.wq_q4k_bytes.restype = sz
    lib.wq_q4k_quantize.argtypes = [vp, i64, i64, vp, vp]
    lib.wq_q4k_quantize.restype = i32
    lib.wq_q4k_matmul.argtypes = [vp, i64, vp, i64, i64, vp, i32, vp]
    lib.wq_q4k_matmul.restype = i32
    lib.wq_q4k_matmul_ex.argtypes = [vp, i64, vp, i64, i64, vp, i32, ctypes.c_uint, vp]
    lib.wq_q4k_matmul_ex.restype = i32
    lib.wq_get_device_error.argtypes = [vp]
    lib.wq_get_device_error.restype = i32
    lib.wq_status_string.argtypes = [i32]
    lib.wq_status_string.restype = ctypes.c_char_p
    lib.wq_version.argtypes = []
    lib.wq_version.restype = ctypes.c_char_p
    lib.wq_internal_last_cuda_error.argtypes = []
    lib.wq_internal_last_cuda_error.restype = ctypes.c_char_p
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.wq_status_string(status).decode()


def version() -> str:
    return lib.wq_version().decode()


def _check(status: int, what: str):
    if status != WQ_OK:
        raise WQError(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require_cuda(*tensors):
    """Every tensor given is a contiguous CUDA tensor, all on one device; the
    library runs on the current device, so calls are made with that device
    current (``torch.cuda.device``)."""
    device = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensor must be on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensor must be contiguous")
        if device is None:
            device = t.device
        elif t.device != device:
            raise ValueError(f"tensors on different devices: {device} and {t.device}")
    return device


def codes_bytes(N: int, K: int, bits: int) -> int:
    return lib.wq_codes_bytes(N, K, bits)


def meta_elems(N: int, K: int, group: int) -> int:
    return lib.wq_meta_elems(N, K, group)


@dataclasses.dataclass
class QuantizedWeight:
    """Packed codes [N, K*bits/8] u8, scales [N, K/group] f16, zeros [N, K/group]
    f16 (None when symmetric), and the format."""
    codes: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor | None
    N: int
    K: int
    bits: int = 4
    group: int = 128
    symmetric: bool = False

    @property
    def nbytes(self) -> int:
        return (self.codes.nbytes + self.scales.nbytes
                + (0 if self.zeros is None else self.zeros.nbytes))


def quantize(W: torch.Tensor, bits: int = 4, group: int = 128, symmetric: bool = False,
             out: QuantizedWeight | None = None) -> QuantizedWeight:
    """``wq_quantize``: W [N, K] float16 on the GPU -> QuantizedWeight."""
    if W.dtype != torch.float16 or W.dim() != 2:
        raise ValueError("W must be a 2-D float16 tensor")
    _require_cuda(W)
    N, K = W.shape
    if out is None:
        dev = W.device
        nb = codes_bytes(N, K, bits)
        ne = meta_elems(N, K, group)
        if nb == 0 or ne == 0:
            raise WQError(1, "wq_quantize")
        out = QuantizedWeight(
            codes=torch.empty((N, nb // N), dtype=torch.uint8, device=dev),
            scales=torch.empty((N, ne // N), dtype=torch.float16, device=dev),
            zeros=None if symmetric else torch.empty((N, ne // N), dtype=torch.float16, device=dev),
            N=N, K=K, bits=bits, group=group, symmetric=symmetric)
    dev = _require_cuda(W, out.codes, out.scales, out.zeros)
    with torch.cuda.device(dev):
        _check(lib.wq_quantize(_ptr(W), N, K, bits, group, int(symmetric), _ptr(out.codes),
                               _ptr(out.scales), _ptr(out.zeros), _stream(dev)), "wq_quantize")
    return out


def dequantize(qw: QuantizedWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    """``wq_dequantize``: materialise What [N, K] bfloat16 (unfused baseline)."""
    _require_cuda(qw.codes, qw.scales, qw.zeros)
    if out is None:
        out = torch.empty((qw.N, qw.K), dtype=torch.bfloat16, device=qw.codes.device)
    dev = _require_cuda(qw.codes, qw.scales, qw.zeros, out)
    with torch.cuda.device(dev):
        _check(lib.wq_dequantize(_ptr(qw.codes), _ptr(qw.scales), _ptr(qw.zeros), qw.N, qw.K,
                                 qw.bits, qw.group, int(qw.symmetric), _ptr(out),
                                 _stream(dev)), "wq_dequantize")
    return out


_workspaces: dict = {}


def workspace(device: torch.device, stream: int) -> torch.Tensor:
    """The zero-filled ``wq_matmul`` workspace used for calls on ``stream``
    (one per device and stream, so that calls on different streams never
    share one)."""
    key = (device.index, stream)
    ws = _workspaces.get(key)
    if ws is None:
        ws = torch.zeros(lib.wq_matmul_workspace_bytes(), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def matmul(X: torch.Tensor, qw: QuantizedWeight, out_dtype: torch.dtype = torch.float32,
           out: torch.Tensor | None = None, static_weights: bool = False,
           use_workspace: bool = True) -> torch.Tensor:
    """``wq_matmul``: Y [M, N] = X [M, K] (bfloat16) times What^T.

    X may live on the host: it is then copied to the weights' device, the
    product is computed there and Y is copied back to the host (the
    end-to-end path; pinned host memory makes the copies asynchronous).
    ``static_weights`` passes WQ_MATMUL_STATIC_WEIGHTS: the weights are not
    written by the kernel that precedes the call on the stream.
    ``use_workspace=False`` passes no workspace (whole row tiles per SM)."""
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != qw.K:
        raise ValueError("X must be a 2-D bfloat16 tensor [M, K]")
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out_dtype must be float32 or bfloat16")
    dev = qw.codes.device
    host = not X.is_cuda
    Xd = X.to(dev, non_blocking=True) if host else X
    _require_cuda(Xd, qw.codes, qw.scales, qw.zeros)
    M = Xd.shape[0]
    Yd = out if (out is not None and out.is_cuda) else torch.empty(
        (M, qw.N), dtype=out_dtype, device=dev)
    _require_cuda(Xd, qw.codes, qw.scales, qw.zeros, Yd)
    stream = torch.cuda.current_stream(dev).cuda_stream
    ws = workspace(dev, stream) if use_workspace else None
    with torch.cuda.device(dev):
        _check(lib.wq_matmul(_ptr(Xd), M, _ptr(qw.codes), _ptr(qw.scales), _ptr(qw.zeros), qw.N,
                             qw.K, qw.bits, qw.group, int(qw.symmetric), _ptr(Yd),
                             WQ_OUT_BF16 if Yd.dtype == torch.bfloat16 else WQ_OUT_F32,
                             _ptr(ws), 0 if ws is None else ws.numel(),
                             WQ_MATMUL_STATIC_WEIGHTS if static_weights else 0,
                             ctypes.c_void_p(stream)), "wq_matmul")
    if not host:
        return Yd
    if out is not None and not out.is_cuda:
        out.copy_(Yd, non_blocking=True)
        return out
    return Yd.cpu()


def q4k_bytes(N: int, K: int) -> int:
    """``wq_q4k_bytes``: bytes of the superblocks of an [N, K] matrix."""
    return int(lib.wq_q4k_bytes(N, K))


def q4k_quantize(W: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """``wq_q4k_quantize``: W [N, K] float16 on the GPU -> uint8 blocks
    [N, K/256 * 144] (nested superblocks, 4.5 bits per weight)."""
    if W.dtype != torch.float16 or W.dim() != 2:
        raise ValueError("W must be a 2-D float16 tensor")
    N, K = W.shape
    nb = q4k_bytes(N, K)
    if nb == 0:
        raise WQError(1, "wq_q4k_quantize")
    if out is None:
        out = torch.empty((N, nb // N), dtype=torch.uint8, device=W.device)
    dev = _require_cuda(W, out)
    with torch.cuda.device(dev):
        _check(lib.wq_q4k_quantize(_ptr(W), N, K, _ptr(out), _stream(dev)), "wq_q4k_quantize")
    return out


def q4k_matmul(X: torch.Tensor, blocks: torch.Tensor, N: int, K: int,
               out_dtype: torch.dtype = torch.float32,
               out: torch.Tensor | None = None, static_weights: bool = False) -> torch.Tensor:
    """``wq_q4k_matmul_ex``: Y [M, N] = X [M, K] (bfloat16, M <= 8) times What^T
    for superblock weights; X, blocks and Y on the GPU.  ``static_weights``
    passes WQ_MATMUL_STATIC_WEIGHTS (nothing enqueued before writes the
    blocks)."""
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != K:
        raise ValueError("X must be a 2-D bfloat16 tensor [M, K]")
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out_dtype must be float32 or bfloat16")
    M = X.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=X.device)
    dev = _require_cuda(X, blocks, Y)
    with torch.cuda.device(dev):
        _check(lib.wq_q4k_matmul_ex(_ptr(X), M, _ptr(blocks), N, K, _ptr(Y),
                                    WQ_OUT_BF16 if Y.dtype == torch.bfloat16 else WQ_OUT_F32,
                                    WQ_MATMUL_STATIC_WEIGHTS if static_weights else 0,
                                    _stream(dev)), "wq_q4k_matmul_ex")
    return Y


def matmul_noalloc(X: torch.Tensor, qw: QuantizedWeight, out_dtype: torch.dtype = torch.float32,
                   out: torch.Tensor | None = None, static_weights: bool = False) -> torch.Tensor:
    """``wq_matmul_noalloc``: as ``matmul`` with device tensors, the workspace
    being the library's own fixed block (see ``include/wq.h``)."""
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != qw.K:
        raise ValueError("X must be a 2-D bfloat16 tensor [M, K]")
    _require_cuda(X, qw.codes, qw.scales, qw.zeros)
    dev = qw.codes.device
    M = X.shape[0]
    Y = out if out is not None else torch.empty((M, qw.N), dtype=out_dtype, device=dev)
    _require_cuda(X, qw.codes, qw.scales, qw.zeros, Y)
    # the library's scratch block is looked up on the current device
    with torch.cuda.device(dev):
        _check(lib.wq_matmul_noalloc(_ptr(X), M, _ptr(qw.codes), _ptr(qw.scales),
                                     _ptr(qw.zeros), qw.N, qw.K, qw.bits, qw.group,
                                     int(qw.symmetric), _ptr(Y),
                                     WQ_OUT_BF16 if Y.dtype == torch.bfloat16 else WQ_OUT_F32,
                                     WQ_MATMUL_STATIC_WEIGHTS if static_weights else 0,
                                     _stream(dev)), "wq_matmul_noalloc")
    return Y


def get_device_error(device: torch.device | None = None) -> int:
    """``wq_get_device_error``: read and clear the device status word."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(device):
        return lib.wq_get_device_error(_stream(device))
