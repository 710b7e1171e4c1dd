"""Fused small-batch matmul on the B200 against the oracle's float64 product
of X and the oracle-dequantized weights:
|y - y_ref| <= 1e-4 * sum_k |x_k w^_k| (float32 out), plus one bfloat16 ulp
for bfloat16 out.  Full outputs at the tiny case, the four layer shapes and
reduced sizes that span several tiles and a ragged tail; sampled outputs
(computed one by one by the oracle) at the full sweep size; closed forms
(one-hot and zero activations) bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import check_tolerance, host_bits, oracle_quantize, weight, wq

pytestmark = pytest.mark.gpu

FORMATS = [(b, g, s) for b in (4, 8) for g in (32, 64, 128) for s in (False, True)]


def quantize_both(W, bits, group, sym, key=None):
    qw = wq().quantize(W.cuda(), bits=bits, group=group, symmetric=sym)
    if key is None:
        _, codes, scales, zeros = oracle.get().quantize(synth.half_bits(W), bits, group, sym)
    else:
        _, codes, scales, zeros = oracle_quantize(W, key, bits, group, sym)
    assert np.array_equal(host_bits(qw.codes), codes)
    return qw, codes, scales, zeros


def run_full(W, X, bits, group, sym, out_dtype=torch.float32):
    qw, codes, scales, zeros = quantize_both(W, bits, group, sym)
    Y = wq().matmul(X.cuda(), qw, out_dtype=out_dtype)
    torch.cuda.synchronize()
    N, K = W.shape
    y_ref, y_abs = oracle.get().matmul(synth.bf16_bits(X), codes, scales, zeros, N, K, bits,
                                       group, sym)
    check_tolerance(Y.float().cpu().numpy(), y_ref, y_abs, out_dtype == torch.bfloat16)
    return Y, y_ref


def test_tiny_case():
    W, X = synth.tiny()
    run_full(W, X, 4, 128, False)
    run_full(W, X, 4, 128, False, torch.bfloat16)


@pytest.mark.parametrize("name", list(synth.LAYER_SHAPES))
def test_layer_shapes_full_size(name):
    K, N = synth.LAYER_SHAPES[name]
    W = synth.weight(N, K, seed=0)
    X = synth.activation(1, K, seed=1)
    run_full(W, X, 4, 128, False)


@pytest.mark.parametrize("bits,group,sym", FORMATS)
@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 32])
def test_sweep_full_size_sampled(M, bits, group, sym):
    """The small-batch sweep at its full size (K=4096, N=14336); 768 outputs
    checked one by one against the oracle, plus every output of rows 0-15
    and the last row tile."""
    N, K = 14336, 4096
    W = weight(N, K, seed=0)
    X = synth.activation(M, K, seed=1)
    qw, codes, scales, zeros = quantize_both(W, bits, group, sym, key=("sweep", N, K))
    Y = wq().matmul(X.cuda(), qw).cpu().numpy()
    rng = np.random.default_rng(M * 100 + bits * 10 + group + sym)
    ms = rng.integers(0, M, 768)
    ns = rng.integers(0, N, 768)
    edge_n = np.r_[np.arange(16), np.arange(N - 16, N)]
    ms = np.r_[ms, np.repeat(np.arange(M), edge_n.size)]
    ns = np.r_[ns, np.tile(edge_n, M)]
    y_ref, y_abs = oracle.get().matmul_at(synth.bf16_bits(X), codes, scales, zeros, N, K, bits,
                                          group, sym, ms, ns)
    check_tolerance(Y[ms, ns], y_ref, y_abs, False)


@pytest.mark.parametrize("bits,group,sym", FORMATS)
@pytest.mark.parametrize("M,N,K", [(1, 300, 1024), (3, 333, 2048), (8, 1000, 4160),
                                   (17, 250, 1024), (32, 129, 4096), (5, 4096, 14336)])
def test_reduced_sizes_full_outputs(M, N, K, bits, group, sym):
    if K % group:
        pytest.skip("K not a multiple of the group")
    W = synth.weight(N, K, seed=N + K)
    X = synth.activation(M, K, seed=M)
    run_full(W, X, bits, group, sym)
    run_full(W, X, bits, group, sym, torch.bfloat16)


@pytest.mark.parametrize("N,K", [(1, 32), (1, 128), (15, 64), (17, 96), (31, 4096), (2, 8192)])
def test_degenerate_shapes(N, K):
    for bits, group, sym in FORMATS:
        if K % group:
            continue
        W = synth.weight(N, K, seed=11)
        X = synth.activation(2, K, seed=12)
        run_full(W, X, bits, group, sym)


@pytest.mark.parametrize("bits,group,sym", FORMATS)
def test_one_hot_and_zero_activations_exact(bits, group, sym):
    """X = e_k gives Y[:, n] = w^[n, k] bit-exactly; X = 0 gives Y = 0."""
    N, K = 1000, 4096
    W = synth.weight(N, K, seed=2)
    qw, codes, scales, zeros = quantize_both(W, bits, group, sym)
    what = oracle.get().dequantize(codes, scales, zeros, N, K, bits, group, sym)
    ks = [0, 1, 127, 128, 2049, K - 1]
    X = torch.zeros(len(ks), K, dtype=torch.bfloat16)
    for i, k in enumerate(ks):
        X[i, k] = 1.0
    Y = wq().matmul(X.cuda(), qw).cpu().numpy()
    assert np.array_equal(Y.astype(np.float64), what[:, ks].T)
    Z = wq().matmul(torch.zeros(3, K, dtype=torch.bfloat16).cuda(), qw).cpu().numpy()
    assert np.all(Z == 0)


def test_outlier_heavy_inputs():
    """Large activations and outlier channels: tolerance is relative to
    sum |x w|, so it must hold however skewed the terms are."""
    N, K = 2048, 4096
    W = synth.weight(N, K, seed=21, outlier_scale=200.0)
    X = synth.activation(4, K, seed=22, std=100.0)
    for bits, group, sym in [(4, 128, False), (8, 32, True), (4, 32, True)]:
        run_full(W, X, bits, group, sym)


def test_deterministic():
    K, N = 4096, 4096
    W = synth.weight(N, K, seed=4)
    X = synth.activation(4, K, seed=5).cuda()
    qw = wq().quantize(W.cuda())
    a = wq().matmul(X, qw)
    b = wq().matmul(X, qw)
    assert torch.equal(a, b)


def test_host_buffers_end_to_end():
    """X on the host in pinned memory: the binding copies in, runs, copies out."""
    K, N = 4096, 1024
    W = synth.weight(N, K, seed=6)
    X = synth.activation(1, K, seed=7).pin_memory()
    qw, codes, scales, zeros = quantize_both(W, 4, 128, False)
    Y = wq().matmul(X, qw)
    assert not Y.is_cuda
    y_ref, y_abs = oracle.get().matmul(synth.bf16_bits(X), codes, scales, zeros, N, K, 4, 128,
                                       False)
    check_tolerance(Y.numpy(), y_ref, y_abs, False)


def test_rejections_and_status():
    mod = wq()
    K, N = 4096, 256
    qw = mod.quantize(synth.weight(N, K).cuda())
    X = synth.activation(1, K).cuda()
    bad = torch.empty(2 * K + 8, dtype=torch.bfloat16, device="cuda")[1:K + 1].view(1, K)
    with pytest.raises(mod.WQError) as e:
        mod.matmul(bad, qw)
    assert e.value.status == 3
    assert mod.get_device_error() == 0
