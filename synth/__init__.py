"""Seeded synthetic inputs shared by the oracle checks, the GPU tests and the
benchmark.  Random numbers only: nothing here quantizes, dequantizes or
multiplies -- the method's arithmetic lives in the CUDA library and, as an
independent restatement, in the oracle.

Recipe (Llama-8B-shaped decode layers; no trained weights or datasets exist
here, so these stand in for real layers):

* weights  W[N, K] = randn * 0.02 in float32, then a set of input channels
  (columns k) scaled by an outlier factor, rounded to binary16;
  default outliers: round(0.005*K) columns chosen by ``randperm(K)`` with the
  seed + 1, scaled x20;  the tiny case uses columns 7 and 300 scaled x50.
* activations X[M, K] = randn in float32, rounded to bfloat16.
* seeds: the tiny case uses seed 0 for W and X; the other cases use seed 0
  for W and seed 1 for X unless a test says otherwise.

CPU generators are used unless ``device`` is given, so that every process
(and the oracle) sees the same values.
"""
from __future__ import annotations

import torch

LAYER_SHAPES = {          # (K, N) of the Llama-8B projections
    "qo": (4096, 4096),
    "kv": (4096, 1024),
    "gate_up": (4096, 14336),
    "down": (14336, 4096),
}


# The seven projections of one Llama-8B decoder layer, as (name, N, K): the
# weight of a projection is [N out features, K in features].
LLAMA8B_PROJECTIONS = (
    ("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
    ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336),
)
LLAMA8B_LAYERS = 32


def llama8b_matrices(layers: int = LLAMA8B_LAYERS):
    """(layer, projection index, name, N, K, seed) of every quantized matrix
    of the whole model: 32 layers x 7 projections = 224 matrices,
    6,979,321,856 weights.  Matrix (layer, j) is drawn with seed
    1000 * layer + j (outlier columns from seed + 1, as everywhere)."""
    return [(layer, j, name, n, k, 1000 * layer + j)
            for layer in range(layers)
            for j, (name, n, k) in enumerate(LLAMA8B_PROJECTIONS)]


def outlier_columns(K: int, seed: int, fraction: float = 0.005) -> torch.Tensor:
    count = int(round(fraction * K))
    g = torch.Generator().manual_seed(seed + 1)
    return torch.randperm(K, generator=g)[:count]


def weight(N: int, K: int, seed: int = 0, outlier_cols=None, outlier_scale: float = 20.0,
           std: float = 0.02, device: str | torch.device = "cpu") -> torch.Tensor:
    """binary16 weights [N, K]: N(0, std) with scaled outlier input channels."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(seed)
    W = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * std
    cols = outlier_columns(K, seed) if outlier_cols is None else torch.as_tensor(outlier_cols)
    if len(cols):
        W[:, cols.to(device)] *= outlier_scale
    return W.to(torch.float16)


def activation(M: int, K: int, seed: int = 1, device: str | torch.device = "cpu",
               std: float = 1.0) -> torch.Tensor:
    """bfloat16 activations [M, K]: N(0, std)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(seed)
    return (torch.randn(M, K, generator=g, device=device, dtype=torch.float32) * std).to(
        torch.bfloat16)


def tiny():
    """The tiny case: W[256, 512] with channels 7 and 300 scaled x50, X[1, 512],
    seed 0 for both."""
    W = weight(256, 512, seed=0, outlier_cols=[7, 300], outlier_scale=50.0)
    X = activation(1, 512, seed=0)
    return W, X


# The page 1 and page 3 worked inputs (page 1 section 1 example; page 3 "代码").
P1_EXAMPLE = [-8.0, -0.2, 0.1, 0.3, 7.0, 7.1, 7.2, 7.3]
P3_EXAMPLE = [-0.9, -0.2, 0.1, 0.5, 3.0]


def half_bits(t: torch.Tensor):
    """uint16 numpy view of a binary16 tensor's bit patterns (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bfloat16 tensor's bit patterns (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
