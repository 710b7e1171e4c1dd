"""Paper mode: the pages' affine quantizer in Python floats (binary64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Written from the pages' equations, in the pages' precision (binary64,
scales not rounded to binary16), for their worked examples and the
information-only error table:

* ``affine_quantize`` -- page 1 ("vLLM 量化与推测解码"), section 1: the affine
  map q = clamp(round(x/s) + z, qmin, qmax), x^ = s (q - z) with the
  min-max calibration s = (x_max - x_min)/(q_max - q_min),
  z = round(q_min - x_min/s), unsigned b-bit codes (q_min = 0,
  q_max = 2^b - 1), one (s, z) per group (per tensor when no group size is
  given).  Where the section's prose leaves a step open, its executable
  per-tensor / per-group example fixes it: the calibration range is widened
  to contain real 0, a degenerate range gets s = 1, and z is clamped into
  [q_min, q_max].
* ``quantize_dequantize_p3`` -- page 3 ("量化：为何加速推理与精度权衡"),
  section "直接答案": scale = (h - l)/q_max over the raw range [l, h],
  z = round(-l/scale) (not clamped), x^ = scale (clamp(round(x/scale) + z,
  0, q_max) - z); returns x^ and the step (the scale).
* ``fused_matmul_kmajor`` -- page 2 ("量化", llminference s08), section
  "实现": the output is the sum over groups of x[:, group g] times group g's
  dequantized block, with the weights laid out [n_groups, group, out].

``round`` is half-to-even (``_round``, numpy's rint, the rounding of the
Python ``round`` that the pages' examples call).
"""
from __future__ import annotations

import numpy as np

# Round half to even.  A module-level name so that the planted-mistake tests
# can swap it for a wrong rounding and check that the pins catch it.
_round = np.rint


def _group_starts(n: int, size: int) -> np.ndarray:
    return np.arange(0, n, size)


def affine_quantize(x, bits: int = 8, group_size: int | None = None):
    """Page 1, section 1: groupwise affine quantization of a 1-D sequence.

    Returns (codes, reconstruction, [(scale, zero) per group]) as Python
    lists; the last group may be shorter than ``group_size``."""
    v = np.asarray([float(e) for e in x], dtype=np.float64)
    n = v.size
    size = n if group_size is None else int(group_size)
    q_min, q_max = 0.0, float((1 << bits) - 1)
    starts = _group_starts(n, size)
    # calibration range of each group, widened to contain real 0
    x_min = np.minimum(np.minimum.reduceat(v, starts), 0.0)
    x_max = np.maximum(np.maximum.reduceat(v, starts), 0.0)
    degenerate = x_max == x_min
    s = np.where(degenerate, 1.0, (x_max - x_min) / np.where(degenerate, 1.0, q_max - q_min))
    z = np.clip(_round(q_min - x_min / s), q_min, q_max)
    g = np.arange(n) // size                      # group of each element
    q = np.clip(_round(v / s[g]) + z[g], q_min, q_max)
    x_hat = s[g] * (q - z[g])
    codes = [int(c) for c in q]
    meta = [(float(a), int(b)) for a, b in zip(s, z)]
    return codes, [float(e) for e in x_hat], meta


def quantize_dequantize_p3(xs, bits: int):
    """Page 3, "直接答案": one scale over the raw range; returns
    (reconstruction as a list, scale)."""
    v = np.asarray([float(e) for e in xs], dtype=np.float64)
    q_max = float((1 << bits) - 1)
    l, h = float(v.min()), float(v.max())
    scale = (h - l) / q_max
    z = _round(-l / scale)
    q = np.clip(_round(v / scale) + z, 0.0, q_max)
    return [float(e) for e in scale * (q - z)], scale


def fused_matmul_kmajor(x, q_kmajor, scales_kmajor, group: int) -> np.ndarray:
    """Page 2, "实现": Y = sum over groups g of x[:, g-th group of K] times
    (q[g] * scales[g]).

    ``x`` is [M, K], ``q_kmajor`` is [n_groups, group, out_features]
    integer-valued (here already q - z), ``scales_kmajor`` is [n_groups,
    out_features]; everything in binary64."""
    n_groups, gsize, out_f = q_kmajor.shape
    assert gsize == group
    x = np.asarray(x, dtype=np.float64)
    blocks = q_kmajor.astype(np.float64) * scales_kmajor.astype(np.float64)[:, None, :]
    x_groups = x.reshape(x.shape[0], n_groups, group)
    # one group's partial product per g, then their sum
    partial = np.einsum("mgk,gko->gmo", x_groups, blocks)
    return partial.sum(axis=0)
