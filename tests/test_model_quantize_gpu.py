"""Whole-model quantize on the B200 against the oracle: every one of the 224
matrices of a Llama-8B-shaped model (32 layers x q, k, v, o, gate, up, down,
drawn on the GPU with seed 1000 * layer + projection), INT4 asymmetric group
128.  Codes, scales and zeros are bit-exact against the oracle on sampled
rows of every matrix (rows are independent: a group never crosses a row),
and on every row of the first and the last layer."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import host_bits
from tests.gpu_util import wq as gpu_wq

pytestmark = pytest.mark.gpu

BITS, GROUP, SYM = 4, 128, False
MATRICES = synth.llama8b_matrices()


def check_rows(W: torch.Tensor, qw, rows: np.ndarray):
    Wh = W[torch.as_tensor(rows, device=W.device)].cpu()
    _, codes, scales, zeros = oracle.get().quantize(synth.half_bits(Wh), BITS, GROUP, SYM)
    idx = torch.as_tensor(rows, device=W.device)
    got_c = host_bits(qw.codes[idx])
    got_s = host_bits(qw.scales[idx])
    got_z = host_bits(qw.zeros[idx])
    bad = np.flatnonzero(got_c != codes.reshape(got_c.shape))
    assert bad.size == 0, f"{bad.size} code bytes differ (rows {rows.tolist()})"
    assert np.array_equal(got_s, scales.reshape(got_s.shape)), "scales differ"
    assert np.array_equal(got_z, zeros.reshape(got_z.shape)), "zeros differ"


def test_model_matrix_list():
    """32 x 7 matrices, 6,979,321,856 weights, distinct seeds."""
    assert len(MATRICES) == 224
    assert sum(n * k for (_, _, _, n, k, _) in MATRICES) == 6_979_321_856
    assert len({m[5] for m in MATRICES}) == 224


@pytest.mark.parametrize("layer", range(synth.LLAMA8B_LAYERS))
def test_every_matrix_sampled_rows(layer):
    wq = gpu_wq()
    rng = np.random.default_rng(layer)
    for (_, _, name, n, k, seed) in MATRICES[7 * layer: 7 * layer + 7]:
        W = synth.weight(n, k, seed=seed, device="cuda")
        qw = wq.quantize(W, bits=BITS, group=GROUP, symmetric=SYM)
        rows = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 6)]))
        check_rows(W, qw, rows)


@pytest.mark.parametrize("layer", [0, synth.LLAMA8B_LAYERS - 1])
def test_first_and_last_layer_every_row(layer):
    wq = gpu_wq()
    for (_, _, name, n, k, seed) in MATRICES[7 * layer: 7 * layer + 7]:
        W = synth.weight(n, k, seed=seed, device="cuda")
        qw = wq.quantize(W, bits=BITS, group=GROUP, symmetric=SYM)
        check_rows(W, qw, np.arange(n))
