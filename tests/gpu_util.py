"""Helpers shared by the GPU parity tests: run the CUDA path through the
binding (which calls the C ABI) and the oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth


def wq():
    import w4a16_decode_matmul_b200 as mod    # raises if libwq.so is missing
    return mod


_cache: dict = {}


def cached(key, fn):
    """Memoise expensive CPU work (weight generation, oracle quantization)
    across tests in one process."""
    if key not in _cache:
        if len(_cache) > 64:
            _cache.clear()
        _cache[key] = fn()
    return _cache[key]


def weight(N: int, K: int, seed: int = 0, **kw) -> torch.Tensor:
    return cached(("w", N, K, seed, tuple(sorted(kw.items()))),
                  lambda: synth.weight(N, K, seed=seed, **kw))


def oracle_quantize(W: torch.Tensor, key, bits: int, group: int, sym: bool):
    """(None, codes, scales, zeros) from the oracle, memoised under `key`
    (the unpacked int32 codes are dropped to keep the cache small)."""
    def run():
        _, codes, scales, zeros = oracle.get().quantize(synth.half_bits(W), bits, group, sym)
        return None, codes, scales, zeros
    return cached(("q", key, bits, group, sym), run)


def gpu_quantize(W: torch.Tensor, bits: int, group: int, sym: bool):
    """Quantize on the GPU; returns the QuantizedWeight (on the GPU)."""
    return wq().quantize(W.cuda(), bits=bits, group=group, symmetric=sym)


def host_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def assert_quantize_parity(W: torch.Tensor, bits: int, group: int, sym: bool):
    """Codes, packed bytes, scales and zeros bit-exact against the oracle."""
    qw = gpu_quantize(W, bits, group, sym)
    _, codes, scales, zeros = oracle.get().quantize(synth.half_bits(W), bits, group, sym)
    got_codes = host_bits(qw.codes)
    mism = np.flatnonzero(got_codes != codes)
    assert mism.size == 0, f"{mism.size} code bytes differ, first at flat index {mism[0]}"
    assert np.array_equal(host_bits(qw.scales), scales), "scales differ"
    if sym:
        assert qw.zeros is None
    else:
        assert np.array_equal(host_bits(qw.zeros), zeros), "zeros differ"
    return qw, codes, scales, zeros


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """One bfloat16 ulp at |v| (0 where v == 0)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 7), 0.0)


def check_tolerance(y: np.ndarray, y_ref: np.ndarray, y_abs: np.ndarray, bf16_out: bool,
                    rel: float = 1e-4):
    """|y - y_ref| <= rel * sum|x w| (+ one bfloat16 ulp of y_ref for bf16)."""
    y = y.astype(np.float64)
    bound = rel * y_abs + (bf16_ulp(y_ref) if bf16_out else 0.0)
    err = np.abs(y - y_ref)
    bad = err > bound
    assert np.all(np.isfinite(y)), "non-finite outputs"
    assert not bad.any(), (f"{int(bad.sum())} of {y.size} outputs out of tolerance; worst "
                           f"err/bound = {float(np.max(err / np.maximum(bound, 1e-300)))}")
    return float(np.max(err / np.maximum(y_abs, 1e-300)))
