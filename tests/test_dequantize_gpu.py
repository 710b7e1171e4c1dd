"""The unfused baseline's dequantize on the B200: What rounded to bfloat16,
bit-exact against the oracle's exact What rounded to nearest-even."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import host_bits, wq

pytestmark = pytest.mark.gpu

FORMATS = [(b, g, s) for b in (4, 8) for g in (32, 64, 128) for s in (False, True)]


@pytest.mark.parametrize("bits,group,sym", FORMATS)
@pytest.mark.parametrize("N,K", [(256, 512), (14336, 4096), (33, 4160)])
def test_dequantize_bit_exact(N, K, bits, group, sym):
    if K % group:
        pytest.skip("K not a multiple of the group")
    W = synth.weight(N, K, seed=1)
    qw = wq().quantize(W.cuda(), bits=bits, group=group, symmetric=sym)
    got = host_bits(wq().dequantize(qw))
    _, codes, scales, zeros = oracle.get().quantize(synth.half_bits(W), bits, group, sym)
    what = oracle.get().dequantize(codes, scales, zeros, N, K, bits, group, sym)
    want = torch.from_numpy(what).float().to(torch.bfloat16)       # exact in fp32, then RNE
    assert np.array_equal(got, host_bits(want))


def test_unfused_path_matches_dense_reference():
    """dequantize -> torch bf16 matmul equals the oracle's dense product of the
    same bfloat16 weights (to bf16 GEMM rounding)."""
    N, K = 512, 1024
    W = synth.weight(N, K, seed=2)
    X = synth.activation(3, K, seed=3)
    qw = wq().quantize(W.cuda())
    What = wq().dequantize(qw)
    Y = (X.cuda().float() @ What.float().T).cpu().numpy()
    ref = oracle.get().matmul_dense_bf16(synth.bf16_bits(X), host_bits(What))
    assert np.allclose(Y, ref, rtol=1e-5, atol=1e-4)
