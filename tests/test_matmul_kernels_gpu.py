"""The small-batch kernels behind wq_matmul, each forced in turn, on the
same seeded inputs against the oracle: the balanced kernel with and without
its workspace (row tiles summed across CTAs, or whole tiles per SM), under
programmatic dependent launch, the cluster-split kernel it replaces for
M <= 8, the direct-load kernel (4-bit codes, groups of 128, M <= 4), the
bulk-staged kernel (the same formats, K a multiple of 1,024), the
k-sliced direct-load kernel (the same formats, K = 4096) and the
tensor-memory kernel (4- and 8-bit codes, groups of 128, K = 4096, M <= 2).  Tolerance as in test_matmul_gpu: |y - y_ref| <= 1e-4 sum|x w|
(+ one bfloat16 ulp for bfloat16 out)."""
import contextlib
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import check_tolerance, host_bits, oracle_quantize, weight, wq

pytestmark = pytest.mark.gpu

AUTO, CLUSTER, BALANCED, BALANCED_SPLIT, DIRECT, BULK, KSLICE, TMEM = 0, 1, 2, 3, 4, 5, 6, 7


@contextlib.contextmanager
def kernel(choice):
    lib = wq().lib
    lib.wq_internal_set_kernel.argtypes = [ctypes.c_int]
    lib.wq_internal_set_kernel(choice)
    try:
        yield
    finally:
        lib.wq_internal_set_kernel(AUTO)


def quantized(W, bits, group, sym, key):
    qw = wq().quantize(W.cuda(), bits=bits, group=group, symmetric=sym)
    _, codes, scales, zeros = oracle_quantize(W, key, bits, group, sym)
    assert np.array_equal(host_bits(qw.codes), codes)
    return qw, codes, scales, zeros


def workspace_clear():
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = wq().workspace(dev, torch.cuda.current_stream(dev).cuda_stream)
    torch.cuda.synchronize()
    flags = ws[:4096].view(torch.int32)
    return int(flags.abs().sum().item()) == 0


SHAPES = [(1, 14336, 4096), (2, 1000, 4096), (3, 4096, 4096), (5, 1024, 4096), (8, 700, 4096),
          (1, 4096, 14336), (2, 520, 14336), (1, 77, 1024), (4, 300, 2048), (1, 1201, 8192),
          (4, 1203, 4096), (1, 5, 4096), (2, 1203, 4096)]
FORMATS = [(4, 128, False), (4, 128, True), (4, 64, True), (4, 32, False), (8, 128, False),
           (8, 128, True), (8, 64, True),
           (8, 32, False)]


@pytest.mark.parametrize("bits,group,sym", FORMATS)
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_balanced_kernel_modes(M, N, K, bits, group, sym):
    W = weight(N, K, seed=N + K)
    X = synth.activation(M, K, seed=M + 3)
    qw, codes, scales, zeros = quantized(W, bits, group, sym, ("modes", N, K))
    if N * M <= 16384:
        y_ref, y_abs = oracle.get().matmul(synth.bf16_bits(X), codes, scales, zeros, N, K, bits,
                                           group, sym)
        ms, ns = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        ms, ns = ms.ravel(), ns.ravel()
        y_ref, y_abs = y_ref.ravel(), y_abs.ravel()
    else:
        rng = np.random.default_rng(N + M)
        # every row of the first and last tiles and of the tiles around each
        # of a few CTA boundaries, plus random rows
        ns = np.unique(np.r_[np.arange(48), np.arange(N - 48, N), rng.integers(0, N, 600)])
        ms = np.repeat(np.arange(M), ns.size)
        ns = np.tile(ns, M)
        y_ref, y_abs = oracle.get().matmul_at(synth.bf16_bits(X), codes, scales, zeros, N, K,
                                              bits, group, sym, ms, ns)
    Xd = X.cuda()
    outs = {}
    with kernel(BALANCED_SPLIT):
        outs["split"] = wq().matmul(Xd, qw)
        outs["pdl"] = wq().matmul(Xd, qw, static_weights=True)
    with kernel(BALANCED):
        outs["whole"] = wq().matmul(Xd, qw, use_workspace=False)
        outs["bf16"] = wq().matmul(Xd, qw, out_dtype=torch.bfloat16)
    with kernel(CLUSTER):
        outs["cluster"] = wq().matmul(Xd, qw)
        outs["cluster_pdl"] = wq().matmul(Xd, qw, static_weights=True)
    direct = bits == 4 and group == 128 and M <= 4 and K % 512 == 0
    if direct:
        with kernel(DIRECT):
            outs["direct"] = wq().matmul(Xd, qw)
            outs["direct_pdl"] = wq().matmul(Xd, qw, static_weights=True)
            outs["direct_bf16"] = wq().matmul(Xd, qw, out_dtype=torch.bfloat16)
    bulk = bits == 4 and group == 128 and M <= 4 and K % 1024 == 0
    if bulk:
        with kernel(BULK):
            outs["bulk"] = wq().matmul(Xd, qw)
            outs["bulk_pdl"] = wq().matmul(Xd, qw, static_weights=True)
            outs["bulk_bf16"] = wq().matmul(Xd, qw, out_dtype=torch.bfloat16)
    kslice = bits == 4 and group == 128 and M <= 4 and K == 4096
    if kslice:
        with kernel(KSLICE):
            outs["kslice"] = wq().matmul(Xd, qw)
            outs["kslice_pdl"] = wq().matmul(Xd, qw, static_weights=True)
            outs["kslice_bf16"] = wq().matmul(Xd, qw, out_dtype=torch.bfloat16)
    tmem = group == 128 and M <= 2 and K == 4096
    if tmem:
        with kernel(TMEM):
            outs["tmem"] = wq().matmul(Xd, qw)
            outs["tmem_pdl"] = wq().matmul(Xd, qw, static_weights=True)
            outs["tmem_bf16"] = wq().matmul(Xd, qw, out_dtype=torch.bfloat16)
    outs["auto"] = wq().matmul(Xd, qw, static_weights=True)
    torch.cuda.synchronize()
    assert wq().get_device_error() == 0
    assert workspace_clear()
    for name, Y in outs.items():
        y = Y.float().cpu().numpy()[ms, ns]
        check_tolerance(y, y_ref, y_abs, name.endswith("bf16"))
    # the same kernel and plan give the same bits with and without PDL
    assert torch.equal(outs["split"], outs["pdl"])
    assert torch.equal(outs["cluster"], outs["cluster_pdl"])
    if direct:
        assert torch.equal(outs["direct"], outs["direct_pdl"])
    if bulk:
        assert torch.equal(outs["bulk"], outs["bulk_pdl"])
    if kslice:
        assert torch.equal(outs["kslice"], outs["kslice_pdl"])
    if tmem:
        assert torch.equal(outs["tmem"], outs["tmem_pdl"])


@pytest.mark.parametrize("choice", [AUTO, BULK, KSLICE, TMEM])
def test_back_to_back_static_weights(choice):
    """A chain of launches with programmatic dependent launch, each over a
    different copy of the weights and reading the previous call's output as
    its activations (so every launch depends on the one before)."""
    N = K = 4096
    W = weight(N, K, seed=31)
    X = synth.activation(1, K, seed=32)
    qws = [wq().quantize(W.cuda() * (1.0 + 0.25 * i)) for i in range(3)]
    x = X.cuda()
    chain = [x]
    with kernel(choice):
        for i in range(9):
            y = wq().matmul(chain[-1], qws[i % 3], static_weights=True)
            chain.append((y / y.abs().amax()).to(torch.bfloat16))  # keep the scale sane
        torch.cuda.synchronize()
        ref = [x]
        for i in range(9):
            y = wq().matmul(ref[-1], qws[i % 3])
            torch.cuda.synchronize()
            ref.append((y / y.abs().amax()).to(torch.bfloat16))
    for a, b in zip(chain, ref):
        assert torch.equal(a, b)
    assert wq().get_device_error() == 0
    assert workspace_clear()


@pytest.mark.parametrize("choice", [AUTO, BULK, KSLICE, TMEM])
def test_graph_replay_with_static_weights(choice):
    """Captured in a CUDA graph (the bench's launch mode), replayed twice."""
    N, K = 14336, 4096
    W = weight(N, K, seed=0)
    qws = [wq().quantize(W.cuda()) for _ in range(2)]
    X = synth.activation(1, K, seed=1).cuda()
    with kernel(choice):
        ref = [wq().matmul(X, q) for q in qws]
    s = torch.cuda.Stream()
    Y = torch.empty(1, N, device="cuda")
    with kernel(choice), torch.cuda.stream(s):
        wq().matmul(X, qws[0], out=Y, static_weights=True)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(6):
                wq().matmul(X, qws[i % 2], out=Y, static_weights=True)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, ref[1])
    assert wq().get_device_error() == 0


@pytest.mark.parametrize("bits,group,sym", [(4, 128, False), (8, 32, True), (8, 128, False)])
def test_activation_rows_of_wide_dynamic_range(bits, group, sym):
    """The balanced kernel rounds each activation row to binary16 after a
    power-of-two scaling that puts the row's largest magnitude near 2^15:
    exact within 2^32 of that magnitude.  Rows here span 2^-36 .. 2^12 and
    one row is all zeros but one element; the tolerance bound still holds."""
    N, K = 640, 4096
    W = weight(N, K, seed=41)
    g = torch.Generator().manual_seed(42)
    mags = torch.pow(2.0, torch.randint(-36, 13, (4, K), generator=g).float())
    sign = torch.where(torch.rand(4, K, generator=g) < 0.5, -1.0, 1.0)
    X = (mags * sign).to(torch.bfloat16)
    X[3] = 0
    X[3, 17] = 3.0e-5
    qw, codes, scales, zeros = quantized(W, bits, group, sym, ("dyn", N, K))
    y_ref, y_abs = oracle.get().matmul(synth.bf16_bits(X), codes, scales, zeros, N, K, bits,
                                       group, sym)
    with kernel(BALANCED):
        Y = wq().matmul(X.cuda(), qw)
    torch.cuda.synchronize()
    check_tolerance(Y.cpu().numpy(), y_ref, y_abs, False)
    if bits == 4 and group == 128:
        for choice in (DIRECT, BULK, KSLICE):
            with kernel(choice):
                Y = wq().matmul(X.cuda(), qw)
            torch.cuda.synchronize()
            check_tolerance(Y.cpu().numpy(), y_ref, y_abs, False)
    if group == 128:
        with kernel(TMEM):  # two rows at a time: the kernel's scope is M <= 2
            for m0 in (0, 2):
                Y = wq().matmul(X[m0:m0 + 2].cuda(), qw)
                torch.cuda.synchronize()
                check_tolerance(Y.cpu().numpy(), y_ref[m0:m0 + 2], y_abs[m0:m0 + 2], False)
