"""wq_matmul_noalloc: the matmul for callers that cannot call cudaMalloc
(code running where the allocator must not be entered, or that must not
grow its memory after start-up), with the library's own fixed scratch block
instead of a caller workspace.  Two calls in a row must give the same bits
as wq_matmul with a workspace (same kernel and plan, deterministic), with
the default kernel choice and with row tiles split across CTAs (the path
that uses the scratch), and leave no error and every flag of the block
clear (read back through a test hook)."""
import contextlib
import ctypes

import pytest
import torch

import synth
from tests.gpu_util import weight, wq

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def kernel(choice):
    lib = wq().lib
    lib.wq_internal_set_kernel.argtypes = [ctypes.c_int]
    lib.wq_internal_set_kernel(choice)
    try:
        yield
    finally:
        lib.wq_internal_set_kernel(0)


@pytest.mark.parametrize("choice", [0, 3])
@pytest.mark.parametrize("M,N,K,bits,group,sym", [(1, 14336, 4096, 4, 128, False),
                                                  (3, 1000, 4096, 8, 32, False),
                                                  (1, 4096, 14336, 4, 64, True)])
def test_two_calls_match_the_workspace_entry_point(M, N, K, bits, group, sym, choice):
    mod = wq()
    W = weight(N, K, seed=N + K)
    qw = mod.quantize(W.cuda(), bits=bits, group=group, symmetric=sym)
    X = synth.activation(M, K, seed=M).cuda()
    with kernel(choice):
        ref = mod.matmul(X, qw)
        first = mod.matmul_noalloc(X, qw)
        second = mod.matmul_noalloc(X, qw, static_weights=True)
    torch.cuda.synchronize()
    assert mod.get_device_error() == 0
    assert torch.equal(first, ref)
    assert torch.equal(second, ref)
    lib = mod.lib
    lib.wq_internal_noalloc_flags_set.argtypes = []
    lib.wq_internal_noalloc_flags_set.restype = ctypes.c_int
    assert lib.wq_internal_noalloc_flags_set() == 0


def test_scratch_size_and_rejections():
    mod = wq()
    assert mod.lib.wq_matmul_noalloc_scratch_bytes() >= mod.lib.wq_matmul_workspace_bytes()
    qw = mod.quantize(synth.weight(256, 512).cuda())
    bad = torch.empty(2 * 512 + 8, dtype=torch.bfloat16, device="cuda")[1:513].view(1, 512)
    with pytest.raises(mod.WQError) as e:
        mod.matmul_noalloc(bad, qw)
    assert e.value.status == 3


def test_block_is_cleared_after_a_timed_out_call():
    """A split-tile wait that times out can leave flags of the library's block
    set (a late publisher's, or ones the waiter had not reset); after
    wq_get_device_error has reported the timeout, the next call must clear
    the block first and give the clean result again."""
    from tests.test_timeout_gpu import BITS, GROUP, K, M, N, SYM, _lib, publishing_cta
    mod = wq()
    lib = _lib()
    lib.wq_internal_noalloc_flags_set.argtypes = []
    lib.wq_internal_noalloc_flags_set.restype = ctypes.c_int
    qw = mod.quantize(weight(N, K, seed=5).cuda(), bits=BITS, group=GROUP, symmetric=SYM)
    X = synth.activation(M, K, seed=6).cuda()
    lib.wq_internal_set_kernel(3)
    try:
        ref = mod.matmul_noalloc(X, qw)
        torch.cuda.synchronize()
        assert mod.get_device_error() == 0
        lib.wq_internal_timeout_test(publishing_cta(lib), 20_000_000)
        mod.matmul_noalloc(X, qw)
        assert mod.get_device_error() == 5
        lib.wq_internal_timeout_test(-1, 0)
        first = mod.matmul_noalloc(X, qw)
        second = mod.matmul_noalloc(X, qw)
        torch.cuda.synchronize()
        assert mod.get_device_error() == 0
    finally:
        lib.wq_internal_timeout_test(-1, 0)
        lib.wq_internal_set_kernel(0)
    assert torch.equal(first, ref)
    assert torch.equal(second, ref)
    assert lib.wq_internal_noalloc_flags_set() == 0
