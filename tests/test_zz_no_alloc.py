"""nf4_quantize_noalloc: quantization without any device allocation.

Some callers cannot allocate device memory at the point where they quantize
a weight (their memory was planned and reserved when the program started,
or they run inside a host framework that only hands them finished buffers),
so they cannot supply the workspace nf4_quantize asks for.  The library
offers them a variant whose scratch is a fixed array built into the library.
These tests call it through the C ABI and check its results against the
workspace variant's, bit for bit (the exactness every storage test here
asks for), on two calls in a row; the second call reuses the array the
first call left filled.

This file is collected last on purpose, and each test stands alone, so it
passes both in a fresh process and after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_BLOCKS = 1 << 20      # the built-in scratch: one fp32 per block of 64 weights


def _same(a, b):
    for x, y in ((a.codes, b.codes), (a.qscale, b.qscale), (a.dq_step, b.dq_step), (a.dq_mean, b.dq_mean)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def _weight(seed, n, k):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(n, k, generator=g) * 0.02
    w[0, :64] = 0.0                                   # an all-zero block
    return w.to(torch.bfloat16).cuda()


def test_two_calls_match_workspace_variant():
    """Two different weights quantized back to back without allocation give
    exactly what nf4_quantize with a workspace gives."""
    for seed, (n, k) in ((11, (4096, 4096)), (12, (1024, 11008))):
        W = _weight(seed, n, k)
        ref = qn.quantize(W)
        got = qn.quantize_noalloc(W)
        torch.cuda.synchronize()
        _same(ref, got)
    assert qn.device_error() == 0


def test_largest_weight_that_fits():
    """n_out * k_in / 64 == 2^20 blocks: the largest weight the scratch holds."""
    W = _weight(13, 16384, 4096)
    ref = qn.quantize(W)
    got = qn.quantize_noalloc(W)
    torch.cuda.synchronize()
    _same(ref, got)


def test_too_large_is_rejected_before_any_work():
    """One block more than the scratch holds: QN_ERR_SHAPE, nothing enqueued."""
    L = qn.lib()
    n, k = 16384 + 1, 4096
    assert n * k // 64 > MAX_BLOCKS
    fake = qn._Weight(n, k, 16, 16, 16, 16)     # pointers never dereferenced
    assert L.nf4_quantize_noalloc(ctypes.c_void_p(16), ctypes.byref(fake), None) == 2


def test_matches_oracle_storage():
    """The tiny workload's weight, compared with the CPU definition as well."""
    from oracle import nf4
    t = wl.tiny()
    got = qn.quantize_noalloc(t.W.cuda())
    torch.cuda.synchronize()
    ref = nf4.quantize(wl.bits(t.W), t.n_out, t.k_in)
    assert np.array_equal(got.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(got.qscale.cpu().numpy(), ref["qscale"])
