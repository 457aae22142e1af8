"""Sibling linears (q, k, v sharing x) run as one joined layer: parity of the
joined forward and backward against the oracle applied to each sibling.

[LoRA y QLoRA en Profundidad, "Módulos Objetivo"]: LoRA on the attention
projections; each is a frozen NF4 linear with its own adapter.
"""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import siblings
from bit_nf4_quantized_28_b200 import workloads as wl
from oracle import linear
from parity_util import check_close, oracle_storage, to_np

pytestmark = pytest.mark.gpu


def _siblings(m, n, k, r, alpha, count=3, seed=8000):
    """`count` sibling layers sharing x (drawn by the first) and dy blocks."""
    ts = [wl.make_linear(seed + i, n, k, m, r, alpha, a_std=1.0 / k) for i in range(count)]
    x = ts[0].x
    return ts, x


@pytest.mark.parametrize("m", [300, 12])
def test_joined_forward_backward(m):
    n, k, r, alpha = 256, 1024, 16, 32.0
    ts, x = _siblings(m, n, k, r, alpha)
    ws = [qn.quantize(t.W.cuda()) for t in ts]
    s = siblings.join(ws, [t.A.cuda() for t in ts], [t.B.cuda() for t in ts], alpha)
    xd = x.cuda()
    y, u = qn.linear_fwd(xd, s.w, s.A, s.B, s.alpha)
    dy = torch.cat([t.dy[:m] if t.dy.shape[0] >= m else t.dy for t in ts], dim=1).cuda()
    dx, dA, dB = qn.linear_bwd(dy, xd, s.w, s.A, s.B, s.alpha, u)
    torch.cuda.synchronize()
    ys = siblings.split_rows(y, s.n)
    dys = siblings.split_rows(dy, s.n)
    dAs, dBs = siblings.split_grads(s, dA, dB)
    dx_ref = 0.0
    for i, t in enumerate(ts):
        w_hat = oracle_storage(None, t.W)["w_hat"]
        y_ref, _ = linear.forward(wl.bits(x), w_hat, wl.bits(t.A), wl.bits(t.B), alpha, r)
        check_close(to_np(ys[i]), y_ref, f"y[{i}]")
        dxi, dAi, dBi = linear.backward(wl.bits(dys[i].cpu()), wl.bits(x), w_hat, wl.bits(t.A), wl.bits(t.B), alpha, r)
        dx_ref = dx_ref + dxi
        check_close(to_np(dAs[i]), dAi, f"dA[{i}]")
        check_close(to_np(dBs[i]), dBi, f"dB[{i}]")
    check_close(to_np(dx), dx_ref, "dx (sum over siblings)")


def test_joined_equals_separate_forward():
    """Each sibling's block of the joined output against its own call."""
    m, n, k, r, alpha = 300, 256, 1024, 16, 32.0
    ts, x = _siblings(m, n, k, r, alpha)
    ws = [qn.quantize(t.W.cuda()) for t in ts]
    s = siblings.join(ws, [t.A.cuda() for t in ts], [t.B.cuda() for t in ts], alpha)
    y, _ = qn.linear_fwd(x.cuda(), s.w, s.A, s.B, s.alpha)
    for i, t in enumerate(ts):
        yi, _ = qn.linear_fwd(x.cuda(), ws[i], t.A.cuda(), t.B.cuda(), alpha)
        check_close(to_np(siblings.split_rows(y, s.n)[i]), to_np(yi).astype(np.float64), f"joined vs own y[{i}]")


def test_join_weights_is_the_stacked_quantization():
    """Joining stored NF4 weights gives the storage of the stacked weight
    (whole groups of 256 block scales per sibling)."""
    ts, _ = _siblings(4, 256, 1024, 16, 32.0)
    ws = [qn.quantize(t.W.cuda()) for t in ts]
    joined = siblings.join_weights(ws)
    stacked = qn.quantize(torch.cat([t.W for t in ts]).cuda())
    for a, b in ((joined.codes, stacked.codes), (joined.qscale, stacked.qscale),
                 (joined.dq_step, stacked.dq_step), (joined.dq_mean, stacked.dq_mean)):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
