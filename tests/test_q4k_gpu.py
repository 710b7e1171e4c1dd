"""Nested superblocks (4.5 bits per weight) on the B200 against the oracle:
the quantizer's blocks bit-exact (tiny, ragged-row, edge-value and full
Llama-8B layer shapes), and the fused small-batch matmul within
|y - y_ref| <= 1e-4 sum|x w| (+ one bfloat16 ulp for bfloat16 out), with
y_ref the binary64 product of X and the oracle's reconstruction."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import check_tolerance, host_bits, wq

pytestmark = pytest.mark.gpu


def quantize_both(W):
    blocks = wq().q4k_quantize(W.cuda())
    ref = oracle.get().q4k_quantize(synth.half_bits(W))
    got = host_bits(blocks)
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, f"{bad.size} block bytes differ, first at flat index {bad[0]}"
    return blocks, ref


@pytest.mark.parametrize("N,K", [(1, 256), (3, 512), (17, 4096), (4096, 4096),
                                 (1024, 14336), (14336, 4096)])
def test_quantize_bit_exact(N, K):
    quantize_both(synth.weight(N, K, seed=N + K))


def test_quantize_edge_values():
    N, K = 12, 512
    W = synth.weight(N, K, seed=9).view(torch.int16).clone()
    W[0] = 0                                                   # all-zero row
    W[1] = torch.tensor(np.float16(0.25)).view(torch.int16)    # constant positive
    W[2] = torch.tensor(np.float16(-3.0)).view(torch.int16)    # constant negative
    W[3, ::2] = 0x7BFF                                         # +65504
    W[3, 1::2] = -1025                                         # -65504
    W[4] = torch.arange(1, K + 1, dtype=torch.int16)           # subnormals
    W[5] = W[5] & 0x7FFF                                       # non-negative
    W[6] = W[6] | -32768                                       # non-positive
    W[7, ::3] = -32768                                         # -0.0
    W[8, 5] = 0x7BFF                                           # one outlier
    W[9, :32] = 0x0001                                         # tiniest sub-block
    W[10, :256] = 0                                            # one zero superblock
    quantize_both(W.view(torch.float16))


def sampled_reference(X, ref_blocks, N, K, rows):
    o = oracle.get()
    Wh = o.q4k_dequantize(np.ascontiguousarray(ref_blocks[rows]), len(rows), K)
    x = np.asarray([o.lib.oracle_bf16_to_double(int(v)) for v in synth.bf16_bits(X).ravel()],
                   dtype=np.float64).reshape(-1, K)
    return x @ Wh.T, np.abs(x) @ np.abs(Wh).T


@pytest.mark.parametrize("M", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("N,K", [(1000, 4096), (77, 1024), (14336, 4096), (520, 14336)])
def test_matmul_tolerance(M, N, K):
    W = synth.weight(N, K, seed=2 * N + K)
    X = synth.activation(M, K, seed=M + 5)
    blocks, ref = quantize_both(W)
    rng = np.random.default_rng(N + M)
    rows = np.unique(np.r_[np.arange(min(N, 24)), np.arange(max(0, N - 24), N),
                           rng.integers(0, N, 200)])
    y_ref, y_abs = sampled_reference(X, ref, N, K, rows)
    Y = wq().q4k_matmul(X.cuda(), blocks, N, K)
    Yb = wq().q4k_matmul(X.cuda(), blocks, N, K, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    check_tolerance(Y.cpu().numpy()[:, rows], y_ref, y_abs, False)
    check_tolerance(Yb.float().cpu().numpy()[:, rows], y_ref, y_abs, True)


@pytest.mark.parametrize("N", [1, 15, 16, 17, 1000, 2323, 14336])
@pytest.mark.parametrize("kernel", [0, 1])
def test_kernels_at_k4096(N, kernel):
    """M = 1, K = 4096 runs the tensor-core kernel (16-row tiles, one warp per
    superblock; ragged N exercises the zero-filled rows of the last tile);
    the tuning hook forces the scalar kernel.  Both against the oracle, and
    bit-identical between a plain call and one with static weights
    (programmatic dependent launch)."""
    K = 4096
    lib = wq().lib
    lib.wq_internal_set_q4k_kernel.argtypes = [ctypes.c_int]
    lib.wq_internal_set_q4k_kernel(kernel)
    try:
        W = synth.weight(N, K, seed=3 * N + 7)
        X = synth.activation(1, K, seed=N + 11)
        blocks, ref = quantize_both(W)
        rng = np.random.default_rng(N)
        rows = np.unique(np.r_[np.arange(min(N, 40)), np.arange(max(0, N - 40), N),
                               rng.integers(0, N, 200)])
        y_ref, y_abs = sampled_reference(X, ref, N, K, rows)
        Y = wq().q4k_matmul(X.cuda(), blocks, N, K)
        Y2 = wq().q4k_matmul(X.cuda(), blocks, N, K, static_weights=True)
        Yb = wq().q4k_matmul(X.cuda(), blocks, N, K, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y2)
        check_tolerance(Y.cpu().numpy()[:, rows], y_ref, y_abs, False)
        check_tolerance(Yb.float().cpu().numpy()[:, rows], y_ref, y_abs, True)
    finally:
        lib.wq_internal_set_q4k_kernel(0)


def test_matmul_deterministic_and_one_hot():
    N, K = 640, 1024
    W = synth.weight(N, K, seed=21)
    blocks, ref = quantize_both(W)
    X = torch.zeros(2, K, dtype=torch.bfloat16)
    X[0, 300] = 1.0
    X[1, 1023] = -2.0
    y1 = wq().q4k_matmul(X.cuda(), blocks, N, K)
    y2 = wq().q4k_matmul(X.cuda(), blocks, N, K)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    y_ref, y_abs = sampled_reference(X, ref, N, K, np.arange(N))
    check_tolerance(y1.cpu().numpy(), y_ref, y_abs, False)


def test_rejections():
    W = torch.zeros(4, 384, dtype=torch.float16, device="cuda")
    with pytest.raises(wq().WQError):
        wq().q4k_quantize(W)                               # K not a multiple of 256
    blocks = wq().q4k_quantize(torch.zeros(4, 256, dtype=torch.float16, device="cuda"))
    X = torch.zeros(9, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wq().WQError):
        wq().q4k_matmul(X, blocks, 4, 256)                 # M > 8
