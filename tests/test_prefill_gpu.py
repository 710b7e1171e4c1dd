"""Prefill-sized matmul (M > 32) on the tensor cores against the oracle's
binary64 product of X and the oracle-dequantized weights:
|y - y_ref| <= 1e-4 * sum_k |x_k w^_k| (binary32 out), plus one bfloat16
ulp for bfloat16 out.  Full outputs at reduced sizes that span several
tiles and ragged M/N tails; sampled outputs (computed one by one by the
oracle) at the full prefill sizes M in {512, 2048, 8192}, K=4096, N=14336;
one-hot activations bit-exact (each output is one exact product s (q - z)).
Every test runs on both prefill kernels: the one with both operands in
shared memory ("shared", groups of 64 or 128 with a multiple of 8 groups per
row) and the one with the dequantized weights in tensor memory ("tmem",
every group size, K a multiple of 128)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import check_tolerance, host_bits, oracle_quantize, weight, wq

pytestmark = pytest.mark.gpu

KERNELS = {"shared": 1, "tmem": 2}


@pytest.fixture(params=sorted(KERNELS), autouse=True)
def kernel(request):
    lib = wq().lib
    lib.wq_internal_set_prefill.argtypes = [ctypes.c_int]
    lib.wq_internal_set_prefill(KERNELS[request.param])
    yield request.param
    lib.wq_internal_set_prefill(0)


def in_scope(kernel, K, group):
    if kernel == "shared":
        return group in (64, 128) and (K // group) % 8 == 0 and K // group <= 256
    return K % 128 == 0


def quantize_both(W, bits, group, sym, key=None):
    qw = wq().quantize(W.cuda(), bits=bits, group=group, symmetric=sym)
    if key is None:
        _, codes, scales, zeros = oracle.get().quantize(synth.half_bits(W), bits, group, sym)
    else:
        _, codes, scales, zeros = oracle_quantize(W, key, bits, group, sym)
    assert np.array_equal(host_bits(qw.codes), codes)
    return qw, codes, scales, zeros


@pytest.mark.parametrize("bits,group,sym", [(4, 128, False), (4, 64, True), (8, 128, False),
                                            (8, 64, True), (4, 64, False), (8, 128, True),
                                            (4, 32, False), (8, 32, True), (4, 32, True)])
@pytest.mark.parametrize("M,N,K", [(33, 130, 1024), (64, 200, 1024), (128, 256, 1024), (200, 300, 2048),
                                   (300, 1000, 512), (256, 128, 4096), (129, 257, 384)])
def test_reduced_sizes_full_outputs(kernel, M, N, K, bits, group, sym):
    if K % group:
        pytest.skip("K is not a multiple of the group")
    if not in_scope(kernel, K, group):
        pytest.skip(f"outside the {kernel} prefill kernel's scope")
    W = synth.weight(N, K, seed=N + K + 1)
    X = synth.activation(M, K, seed=M + 7)
    qw, codes, scales, zeros = quantize_both(W, bits, group, sym)
    y_ref, y_abs = oracle.get().matmul(synth.bf16_bits(X), codes, scales, zeros, N, K, bits, group,
                                       sym)
    Y = wq().matmul(X.cuda(), qw)
    Yb = wq().matmul(X.cuda(), qw, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert wq().get_device_error() == 0
    check_tolerance(Y.cpu().numpy(), y_ref, y_abs, False)
    check_tolerance(Yb.float().cpu().numpy(), y_ref, y_abs, True)


@pytest.mark.parametrize("M", [512, 2048, 8192])
def test_prefill_sizes_sampled(M):
    """The prefill workload at its full size; 1,024 outputs checked one by
    one against the oracle, including the corners of the first and last
    tiles."""
    N, K = 14336, 4096
    W = weight(N, K, seed=0)
    qw, codes, scales, zeros = quantize_both(W, 4, 128, False, key=("sweep", N, K))
    X = synth.activation(M, K, seed=1)
    Y = wq().matmul(X.cuda(), qw)
    torch.cuda.synchronize()
    assert wq().get_device_error() == 0
    rng = np.random.default_rng(M)
    ms = np.r_[rng.integers(0, M, 1000), [0, 0, M - 1, M - 1, 127, 128, M - 128, M - 129] * 3]
    ns = np.r_[rng.integers(0, N, 1000), [0, N - 1] * 12]
    ms, ns = ms[:1024], ns[:1024]
    y_ref, y_abs = oracle.get().matmul_at(synth.bf16_bits(X), codes, scales, zeros, N, K, 4, 128,
                                          False, ms, ns)
    check_tolerance(Y.cpu().numpy()[ms, ns], y_ref, y_abs, False)


@pytest.mark.parametrize("bits,group,sym", [(4, 128, False), (8, 64, True), (4, 32, False)])
def test_one_hot_and_zero_activations_exact(kernel, bits, group, sym):
    if not in_scope(kernel, 2048, group):
        pytest.skip(f"outside the {kernel} prefill kernel's scope")
    N, K = 384, 2048
    W = synth.weight(N, K, seed=5)
    qw, codes, scales, zeros = quantize_both(W, bits, group, sym)
    what = oracle.get().dequantize(codes, scales, zeros, N, K, bits, group, sym)
    ks = np.r_[np.arange(0, K, 37), K - 1][:40]
    X = torch.zeros(len(ks), K, dtype=torch.bfloat16)
    X[np.arange(len(ks)), ks] = 1.0
    Y = wq().matmul(X.cuda(), qw).cpu().numpy()
    assert np.array_equal(Y.astype(np.float64), what[:, ks].T)
    Z = wq().matmul(torch.zeros(64, K, dtype=torch.bfloat16).cuda(), qw).cpu().numpy()
    assert np.all(Z == 0)


def test_deterministic_and_out_of_scope(kernel):
    N, K = 512, 4096
    qw = wq().quantize(synth.weight(N, K, seed=9).cuda())
    X = synth.activation(300, K, seed=10).cuda()
    assert torch.equal(wq().matmul(X, qw), wq().matmul(X, qw))
    if kernel == "shared":
        q32 = wq().quantize(synth.weight(N, K, seed=9).cuda(), group=32)
        with pytest.raises(wq().WQError) as e:
            wq().matmul(X, q32)
        assert e.value.status == 2     # group 32 is outside this kernel's scope
