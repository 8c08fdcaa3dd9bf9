"""Failure detection on the GPU without a GPU fault.

Every wait of the chunked kernels on another part of the block (an mbarrier
phase: a TMA load landing, an MMA completing, another warp group's
hand-off) is bounded: after 1 s it records the failure in a device error
word, raises the block's abort flag so the other waiters leave, and the
kernel returns.  Here a dedicated self-test kernel makes that wait run out
(an mbarrier that nothing arrives at) and the host reads the status; the
context must stay usable and the next call must be clean.
"""
import time

import pytest
import torch

import oracle
from linear_attention_transformers_b200 import api, inputs
from parity_util import compare

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nthreads", [1, 608])
def test_bounded_wait_gives_up_and_reports(nthreads):
    api.load_library()
    torch.cuda.synchronize()
    api.la_get_device_error()  # start from a clean error word
    t0 = time.perf_counter()
    api.la_selftest_wait_timeout(nthreads)
    with pytest.raises(api.LinearAttentionError) as err:
        api.la_get_device_error()
    elapsed = time.perf_counter() - t0
    assert err.value.status == api.LA_ERR_DEVICE_TIMEOUT
    # the wait's limit is 1 s; the kernel returned instead of hanging
    assert 0.9 < elapsed < 10.0, elapsed
    # the error word was read and cleared: the next check is clean
    api.la_get_device_error()


def test_context_usable_after_timeout():
    api.la_selftest_wait_timeout(64)
    with pytest.raises(api.LinearAttentionError):
        api.la_get_device_error()
    q, k, v = (t.cuda() for t in inputs.make_tensors(2, 3, 300, 64, torch.bfloat16, 21))
    o = api.la_forward(q, k, v, True)
    torch.cuda.synchronize()
    api.la_get_device_error()
    compare(o, oracle.forward(q, k, v, True, oracle.PHI_ELU1)[0], torch.bfloat16, "o")
