"""The timeout path of a device-side wait, made to run without faulting the
GPU: through an internal test hook, one CTA of the balanced kernel's split
mode never publishes its partial sums, and the CTA that adds them gives up
after 20 ms instead of 2 s.  That wait follows the completion of every copy
and product of the waiting CTA, so nothing is left in flight.  The call must
record WQ_ERR_TIMEOUT in the device status word (read by
wq_get_device_error), the context must stay usable, and once the workspace
is zero-filled again the next call must give the same bits as a clean one."""
import ctypes

import pytest
import torch

import synth
from tests.gpu_util import weight, wq

pytestmark = pytest.mark.gpu

M, N, K, BITS, GROUP, SYM = 3, 1000, 4096, 8, 32, False


def _lib():
    lib = wq().lib
    lib.wq_internal_set_kernel.argtypes = [ctypes.c_int]
    lib.wq_internal_timeout_test.argtypes = [ctypes.c_int, ctypes.c_ulonglong]
    lib.wq_internal_plan_sk.argtypes = [ctypes.c_int] * 9 + [ctypes.POINTER(ctypes.c_int64)]
    lib.wq_internal_plan_sk.restype = ctypes.c_int
    return lib


def publishing_cta(lib) -> int:
    """A CTA whose share of the split tail starts inside a tile (so it
    publishes a partial sum that an earlier CTA waits for), from the plan of
    this device."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    smem = torch.cuda.get_device_properties(0).shared_memory_per_block_optin
    out = (ctypes.c_int64 * 25)()
    assert lib.wq_internal_plan_sk(M, N, K, BITS, GROUP, int(SYM), sms, smem, 1, out) == 1
    nk, waves, ctas, split, tail_tiles = out[5], out[6], out[7], out[8], out[24]
    assert split == 1

    def tail_begin(c):
        return waves * ctas * nk + c * (tail_tiles * nk) // ctas

    for c in range(1, ctas):
        if tail_begin(c) % nk != 0 and tail_begin(c + 1) > tail_begin(c):
            return c
    raise AssertionError("no publishing CTA in this plan")


@pytest.fixture
def hooks():
    lib = _lib()
    lib.wq_internal_set_kernel(3)            # balanced kernel, split tiles
    yield lib
    lib.wq_internal_timeout_test(-1, 0)
    lib.wq_internal_set_kernel(0)


def test_timed_out_wait_is_reported_and_the_next_call_is_clean(hooks):
    mod = wq()
    lib = hooks
    qw = mod.quantize(weight(N, K, seed=5).cuda(), bits=BITS, group=GROUP, symmetric=SYM)
    X = synth.activation(M, K, seed=6).cuda()
    assert mod.get_device_error() == 0
    ref = mod.matmul(X, qw)
    torch.cuda.synchronize()
    assert mod.get_device_error() == 0

    lib.wq_internal_timeout_test(publishing_cta(lib), 20_000_000)   # 20 ms
    mod.matmul(X, qw)
    assert mod.get_device_error() == 5                              # WQ_ERR_TIMEOUT
    assert mod.get_device_error() == 0                              # read and cleared

    lib.wq_internal_timeout_test(-1, 0)
    stream = torch.cuda.current_stream().cuda_stream
    mod.workspace(torch.device("cuda", 0), stream).zero_()           # as wq.h asks
    again = mod.matmul(X, qw)
    torch.cuda.synchronize()
    assert mod.get_device_error() == 0
    assert torch.equal(again, ref)
