"""Failure detection without a GPU fault.

Every wait inside the library's kernels is bounded: a wait that runs out sets
a bit in the device error word and its kernel returns, so a stuck pipeline is
reported instead of hanging the GPU.  The self-test entry point enqueues a
wait on a barrier that nothing completes; the test checks that the wait gives
up (after the library's 2 s limit), that the bit is reported once, and that
the context still computes correctly afterwards.  On the host, bad arguments
are rejected before anything is enqueued (tests/test_abi.py).
"""

import time

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import workloads as wl
from oracle import nf4


def test_selftest_needs_a_device_on_cpu():
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert qn.lib().qn_selftest_bounded_wait(None) == 7


@pytest.mark.gpu
def test_stuck_wait_is_reported_and_the_context_survives():
    assert qn.device_error() == 0
    t0 = time.perf_counter()
    qn.selftest_bounded_wait()
    flags = qn.device_error()                 # synchronizes the device
    elapsed = time.perf_counter() - t0
    assert flags == qn.WAIT_SELFTEST
    assert 1.5 < elapsed < 60.0               # the limit is 2 s of device time
    assert qn.device_error() == 0             # reading clears the word
    # the context is intact: a quantize / dequantize round trip is bit-exact
    W = wl.normal_bf16(torch.Generator().manual_seed(21), (128, 256), 0.02)
    w = qn.quantize(W.cuda())
    w_hat = qn.dequantize(w)
    torch.cuda.synchronize()
    ref = nf4.quantize(wl.bits(W), 128, 256)
    ref_hat = nf4.dequantize(ref["codes"], ref["qscale"], ref["step"], ref["mean"], 128, 256)
    assert np.array_equal(wl.bits(w_hat.cpu()), ref_hat)
    assert qn.device_error() == 0
