"""Quantization error and traffic tables, from the oracle (information only).

TEST INFRASTRUCTURE / INFORMATION ONLY: the values are not pinned to any page;
"量化" (llminference s08) reports this kind of readout (an SNR and a maximum
error for one 4-bit setting) on inputs it does not give.

Error table: page 1 ("vLLM 量化与推测解码") section 1's affine quantizer
(paper mode: binary64, range widened to contain 0, round-half-to-even), over
groups of G consecutive weights along K, per channel (G = K) and per tensor,
for b in {2, 3, 4, 8}, on the synthetic decode weights (N(0, 0.02) with
outlier input channels scaled x20).  SNR = 10 log10(sum w^2 / sum (w - w^)^2).
Effective bits per weight count a binary16 scale and a binary16 zero per
group ("量化" section 所谓「4-bit」; page 1 section 2's payload count).

Traffic table: bytes per weight that a decode matmul moves, fused (codes and
metadata read once) against the unfused path of "量化" section 实现
(dequantize to a 16-bit copy, write it, read it back in the matmul) and a
16-bit dense layer.

    python -m oracle.snr_table [N K] > table.md
"""
from __future__ import annotations

import math
import sys

import numpy as np

from oracle.paper import affine_quantize

BITS = (2, 3, 4, 8)


def error_row(w: np.ndarray, bits: int, group: int | None):
    """(snr_db, max_abs_err, max_err_over_half_scale) of page 1's quantizer
    over consecutive groups of `group` weights (None: the whole tensor)."""
    flat = [float(v) for v in w.ravel()]
    _, recon, meta = affine_quantize(flat, bits, group)
    err = np.asarray(flat) - np.asarray(recon)
    size = len(flat) if group is None else group
    half = np.repeat([m[0] / 2 for m in meta], size)[:len(flat)]
    snr = 10.0 * math.log10(float(np.sum(np.square(flat))) / float(np.sum(np.square(err))))
    return snr, float(np.max(np.abs(err))), float(np.max(np.abs(err) / half))


def effective_bits(bits: int, group: int | None, n_weights: int) -> float:
    g = n_weights if group is None else group
    return bits + 32.0 / g


def tables(N: int = 256, K: int = 1024, seed: int = 0) -> str:
    import synth
    w = synth.weight(N, K, seed=seed).float().numpy().astype(np.float64)
    groups = [(32, "32"), (64, "64"), (128, "128"), (K, f"per channel ({K})"),
              (None, "per tensor")]
    lines = [f"Quantization error, page 1's affine quantizer (paper mode), W[{N}, {K}] "
             f"N(0, 0.02) with {len(synth.outlier_columns(K, seed))} outlier input "
             f"channels x20 (seed {seed})",
             "",
             "| bits | group | bits/weight | SNR dB | max abs error | max error / (scale/2) |",
             "|---|---|---|---|---|---|"]
    for b in BITS:
        for g, name in groups:
            snr, emax, ratio = error_row(w, b, g)
            lines.append(f"| {b} | {name} | {effective_bits(b, g, N * K):.3f} | {snr:.2f} | "
                         f"{emax:.4g} | {ratio:.4f} |")
    lines += ["", "Bytes per weight moved by a decode matmul (asymmetric, binary16 scale and zero)",
              "", "| bits | group | fused | unfused (dequantize, write, re-read 16-bit) | "
              "16-bit dense | fused vs dense |", "|---|---|---|---|---|---|"]
    for b in (4, 8):
        for g in (32, 64, 128):
            fused = b / 8 + 4.0 / g
            unfused = fused + 2.0 + 2.0
            lines.append(f"| {b} | {g} | {fused:.4f} | {unfused:.4f} | 2 | {2 / fused:.2f}x |")
    return "\n".join(lines) + "\n"


if __name__ == "__main__":
    args = [int(a) for a in sys.argv[1:3]]
    sys.stdout.write(tables(*args))
