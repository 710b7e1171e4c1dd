"""Paper mode: the pages' own Python-float semantics, for their worked examples.

TEST INFRASTRUCTURE ONLY (see the package docstring).

These functions restate what each page's code computes, in code written for
this oracle; they keep the pages' precision (Python float = binary64, scales
not rounded to binary16) and their exact steps:

* ``affine_quantize`` -- page 1 ("vLLM 量化与推测解码"), section 1, the
  per-tensor / per-group executable example: range widened to contain 0,
  scale = (hi - lo)/(qmax - qmin) or 1.0 for a degenerate range, zero =
  clamp(round(qmin - lo/scale)), code = clamp(round(v/scale) + zero),
  reconstruction scale*(code - zero).
* ``quantize_dequantize_p3`` -- page 3 ("量化：为何加速推理与精度权衡"), section
  "代码": the same map with the raw min/max (no widening to 0) and no clamp on
  the zero point; returns the reconstruction and the step.
* ``quantize_group_symmetric`` / ``dequantize_group_symmetric`` -- page 2
  ("量化", llminference s08), section "解法": zero point 0, scale = max|w| /
  (2^(b-1) - 1), codes clipped to [-2^(b-1), 2^(b-1) - 1].
* ``fused_matmul_kmajor`` -- page 2, section "实现": codes laid out
  [n_groups, group, out_features] and scales [n_groups, out_features]; the
  output accumulates one group's dequantized block at a time.

``round`` is Python's round(), i.e. round-half-to-even.
"""
from __future__ import annotations

import numpy as np


def affine_quantize(x, bits: int = 8, group_size: int | None = None):
    """Page 1, section 1.  Returns (codes, reconstruction, [(scale, zero), ...])."""
    values = [float(v) for v in x]
    size = len(values) if group_size is None else group_size
    qmin, qmax = 0, (1 << bits) - 1
    codes, recon, meta = [], [], []
    for start in range(0, len(values), size):
        chunk = values[start:start + size]
        lo = min(0.0, min(chunk))        # the range always contains real 0
        hi = max(0.0, max(chunk))
        scale = 1.0 if hi == lo else (hi - lo) / (qmax - qmin)
        zero = min(qmax, max(qmin, round(qmin - lo / scale)))
        for v in chunk:
            c = min(qmax, max(qmin, round(v / scale) + zero))
            codes.append(c)
            recon.append(scale * (c - zero))
        meta.append((scale, zero))
    return codes, recon, meta


def quantize_dequantize_p3(xs, bits: int):
    """Page 3, "代码".  Returns (reconstruction, scale)."""
    qmax = (1 << bits) - 1
    lo, hi = min(xs), max(xs)
    scale = (hi - lo) / qmax
    zero = round(-lo / scale)
    recon = []
    for v in xs:
        c = min(qmax, max(0, round(v / scale) + zero))
        recon.append(scale * (c - zero))
    return recon, scale


def quantize_group_symmetric(w, bits: int = 4):
    """Page 2, "解法" (symmetric, one scale per group).  ``w`` is a 1-D array
    of one group.  Returns (int codes, scale as binary16)."""
    w = np.asarray(w, dtype=np.float64)
    qmax = (1 << (bits - 1)) - 1
    scale = float(np.abs(w).max()) / qmax
    q = np.clip(np.round(w / scale), -qmax - 1, qmax).astype(np.int64)
    return q, np.float16(scale)


def dequantize_group_symmetric(q, scale) -> np.ndarray:
    """Page 2, "解法": q * scale."""
    return np.asarray(q, dtype=np.float64) * float(scale)


def fused_matmul_kmajor(x, q_kmajor, scales_kmajor, group: int) -> np.ndarray:
    """Page 2, "实现": out += x[:, group g] @ (q[g] * scales[g]) for each g.

    ``x`` is [M, K] float64, ``q_kmajor`` is [n_groups, group, out_features]
    integer-valued (here already q - z), ``scales_kmajor`` is [n_groups,
    out_features].  Everything in float64, one group block at a time.
    """
    n_groups, gsize, out_f = q_kmajor.shape
    assert gsize == group
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros((x.shape[0], out_f), dtype=np.float64)
    for g in range(n_groups):
        block = q_kmajor[g].astype(np.float64) * scales_kmajor[g].astype(np.float64)
        out += x[:, g * group:(g + 1) * group] @ block
    return out
