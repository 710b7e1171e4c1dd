"""Quantize on the B200 against the oracle: codes, bytes, scales and zeros
bit-exact, at the tiny case, the four Llama-8B layer shapes at full size,
every format of the small-batch sweep at full size, and edge cases."""
import numpy as np
import pytest
import torch

import synth
from tests.gpu_util import assert_quantize_parity, gpu_quantize, host_bits
from tests.gpu_util import wq as gpu_wq
from tests.gpu_util import weight as gpu_weight

pytestmark = pytest.mark.gpu

FORMATS = [(b, g, s) for b in (4, 8) for g in (32, 64, 128) for s in (False, True)]


def test_tiny_case():
    W, _ = synth.tiny()
    assert_quantize_parity(W, 4, 128, False)


@pytest.mark.parametrize("name", list(synth.LAYER_SHAPES))
def test_layer_shapes_full_size(name):
    K, N = synth.LAYER_SHAPES[name]
    W = synth.weight(N, K, seed=0)
    assert_quantize_parity(W, 4, 128, False)


@pytest.mark.parametrize("bits,group,sym", FORMATS)
def test_sweep_formats_full_size(bits, group, sym):
    W = gpu_weight(14336, 4096, seed=0)
    assert_quantize_parity(W, bits, group, sym)


@pytest.mark.parametrize("bits,group,sym", FORMATS)
def test_edge_values(bits, group, sym):
    N, K = 24, 512
    W = synth.weight(N, K, seed=5).view(torch.int16).clone()
    W[0] = 0                                                   # all-zero row
    W[1] = torch.tensor(np.float16(0.25)).view(torch.int16)    # constant positive
    W[2] = torch.tensor(np.float16(-3.0)).view(torch.int16)    # constant negative
    W[3, ::2] = 0x7BFF                                         # +65504
    W[3, 1::2] = -1025                                         # 0xFBFF = -65504
    W[4] = torch.arange(1, K + 1, dtype=torch.int16)           # subnormals
    W[5] = W[5] & 0x7FFF                                       # all positive
    W[6] = W[6] | -32768                                       # all negative (sign bit)
    W[7, ::3] = -32768                                         # -0.0
    W[8, 5] = 0x7BFF                                           # one outlier
    W[9, :group] = 0x0001                                      # tiniest subnormal group
    assert_quantize_parity(W.view(torch.float16), bits, group, sym)


@pytest.mark.parametrize("N,K", [(1, 32), (1, 128), (3, 96), (17, 1024), (33, 4160), (257, 64)])
def test_ragged_shapes(N, K):
    for bits in (4, 8):
        for group in (32, 64, 128):
            if K % group:
                continue
            for sym in (False, True):
                W = synth.weight(N, K, seed=N * 7 + K)
                assert_quantize_parity(W, bits, group, sym)


def test_page_examples_on_gpu():
    # page 1 section 1 example (group 4 is below the library's smallest group,
    # so the 8 values are tiled into a group of 32) and page 3's five values
    x = np.array([-8.0, -0.2, 0.1, 0.3, 7.0, 7.1, 7.2, 7.3] * 4, dtype=np.float16)
    W = torch.from_numpy(x).view(1, 32)
    qw, codes, _, _ = assert_quantize_parity(W, 4, 32, False)
    assert np.array_equal(host_bits(qw.codes)[0, :4], [0 | 8 << 4, 8 | 8 << 4,
                                                       15 | 15 << 4, 15 | 15 << 4])
    assert host_bits(qw.scales).view(np.float16)[0, 0] == np.float16(1.0205078125)
    y = np.array([-0.9, -0.2, 0.1, 0.5, 3.0] + [0.0] * 27, dtype=np.float16)
    qw, _, _, _ = assert_quantize_parity(torch.from_numpy(y).view(1, 32), 4, 32, False)
    assert host_bits(qw.scales).view(np.float16)[0, 0] == np.float16(0.260009765625)
    assert host_bits(qw.zeros).view(np.float16)[0, 0] == 3


def test_quantize_is_deterministic_and_status_clean():
    wq = gpu_wq()
    W = synth.weight(4096, 4096, seed=3)
    a = gpu_quantize(W, 4, 128, False)
    b = gpu_quantize(W, 4, 128, False)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
    assert wq.get_device_error() == 0
