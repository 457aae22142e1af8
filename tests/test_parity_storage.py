"""GPU parity of NF4 storage: codes, int8 scales, the fp32 second-level
step and mean, and the dequantized bf16 weight must be bit-identical to the
oracle on the same seeded inputs."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import workloads as wl
from oracle import nf4

pytestmark = pytest.mark.gpu


def _run(w_cpu):
    W = w_cpu.cuda()
    q = qn.quantize(W)
    wh = qn.dequantize(q)
    torch.cuda.synchronize()
    assert qn.device_error() == 0
    return q, wh


def _assert_exact(w_cpu, q, wh):
    n, k = w_cpu.shape
    ref = nf4.quantize(wl.bits(w_cpu), n, k)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"]), "codes"
    assert np.array_equal(q.qscale.cpu().numpy(), ref["qscale"]), "int8 scales"
    assert np.array_equal(q.dq_step.cpu().numpy().view(np.uint32), ref["step"].view(np.uint32)), "dq step"
    assert np.array_equal(q.dq_mean.cpu().numpy().view(np.uint32), ref["mean"].view(np.uint32)), "dq mean"
    ref_wh = nf4.dequantize(ref["codes"], ref["qscale"], ref["step"], ref["mean"], n, k)
    assert np.array_equal(wl.bits(wh.cpu()), ref_wh), "dequantized bf16"


def test_tiny_weight():
    w = wl.tiny().W
    q, wh = _run(w)
    _assert_exact(w, q, wh)


def test_quant_round_trip_config_outliers():
    """4096 x 4096, N(0, 0.02) with 1 % x20 outliers (the round-trip workload)."""
    w = wl.quant_weight()
    q, wh = _run(w)
    _assert_exact(w, q, wh)


@pytest.mark.parametrize("shape", [(1, 64), (3, 192), (5, 4096 + 64), (257, 320), (11008 // 16, 4096)])
def test_ragged_shapes(shape):
    g = torch.Generator().manual_seed(shape[0] * 7 + shape[1])
    w = (torch.randn(*shape, generator=g) * 0.02).to(torch.bfloat16)
    q, wh = _run(w)
    _assert_exact(w, q, wh)


def test_degenerate_blocks():
    """All-zero blocks and rows, constant blocks (absmax = every |w|), a group
    whose scales are all equal (step 0), and values near level midpoints."""
    g = torch.Generator().manual_seed(5)
    w = (torch.randn(64, 1024, generator=g) * 0.02)
    w[0] = 0.0                                    # a zero row: 16 zero blocks
    w[1, :64] = 0.0
    w[2, :] = 0.5                                 # constant blocks
    w[3, :] = -0.25
    w[4:8, :] = torch.sign(torch.randn(4, 1024, generator=g))   # +-1 only: 16 equal scales
    w[8, :64] = torch.linspace(-1, 1, 64)
    lv = torch.tensor(nf4.nf4_levels())
    w[11, :16] = lv
    w[11, 16:31] = (lv[:-1] + lv[1:]) * 0.5           # level midpoints
    w[11, 31] = 1.0
    w = w.to(torch.bfloat16)
    q, wh = _run(w)
    _assert_exact(w, q, wh)


@pytest.mark.parametrize("scale", [1e-30, 1e30])
def test_extreme_magnitudes(scale):
    """Tiny and huge weights, one second-level group of 256 blocks each."""
    g = torch.Generator().manual_seed(6)
    w = (torch.randn(16, 1024, generator=g) * scale).to(torch.bfloat16)
    q, wh = _run(w)
    _assert_exact(w, q, wh)


def test_decode_projection_weight():
    """The 4096 -> 11008 decode projection weight (704,512 blocks)."""
    w = wl.decode(11008, 4096).W
    q, wh = _run(w)
    _assert_exact(w, q, wh)


def test_quantize_is_deterministic_and_reuses_workspace():
    w = wl.quant_weight(512, 2048, seed=8).cuda()
    need = qn.lib().nf4_quantize_workspace_bytes(512, 2048)
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device="cuda")
    a = qn.quantize(w, workspace=ws)
    b = qn.quantize(w, workspace=ws)
    torch.cuda.synchronize()
    for x, y in ((a.codes, b.codes), (a.qscale, b.qscale), (a.dq_step, b.dq_step), (a.dq_mean, b.dq_mean)):
        assert torch.equal(x, y)
