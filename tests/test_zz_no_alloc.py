"""wq_matmul_noalloc: the matmul with the library's own fixed scratch block
instead of a caller workspace.  Two calls in a row must give the same bits
as wq_matmul with a workspace (same kernel and plan, deterministic), with
the default kernel choice and with row tiles split across CTAs (the path
that uses the scratch), and leave no error and the block's flags clear."""
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


def test_scratch_size_and_rejections():
    mod = wq()
    assert mod.lib.wq_matmul_noalloc_scratch_bytes() >= mod.lib.wq_matmul_workspace_bytes()
    qw = mod.quantize(synth.weight(256, 512).cuda())
    bad = torch.empty(2 * 512 + 8, dtype=torch.bfloat16, device="cuda")[1:513].view(1, 512)
    with pytest.raises(mod.WQError) as e:
        mod.matmul_noalloc(bad, qw)
    assert e.value.status == 3
