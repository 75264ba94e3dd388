"""The timeout path of the library's bounded waits, exercised on the GPU without a fault.

Every copy barrier the kernels wait on gives up after about one second, flags
KVQ_DEV_TIMEOUT in the device status word and lets the kernel finish. The self-check entry
point waits on a barrier nothing completes; the status must carry the flag, the wait must
have lasted about the limit, and the context must still run a decode correctly afterwards.
"""
import time

import pytest
import torch

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


def test_wait_that_nothing_completes_times_out_and_flags():
    kvq = H.kvq()
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    kvq.kvq_check_bounded_wait(status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(status[0].item()) & kvq.KVQ_DEV_TIMEOUT
    assert 0.9 <= dt <= 30.0, dt
    # the context is intact: a decode still matches the oracle
    H.dense_case(B=1, Hq=8, Hkv=1, ks=synth.FP8_E4M3_PER_TENSOR, vs=synth.FP8_E4M3_PER_TENSOR, prefill=100, steps=1)


def test_misaligned_status_pointer_is_refused_on_the_host():
    kvq = H.kvq()
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    import ctypes
    st = kvq.lib.kvq_check_bounded_wait(ctypes.c_void_p(status.data_ptr() + 2), None)
    assert st == kvq.KVQ_ERR_INVALID_ARG
