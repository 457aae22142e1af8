"""Sibling linears (q, k, v sharing x; gate and up) run as one call: parity of
the sibling forward and backward against the oracle applied to each sibling
on its own.

[LoRA y QLoRA en Profundidad, "Módulos Objetivo"]: LoRA on the attention
projections and on the MLP's gate and up; each is a frozen NF4 linear with
its own adapter of rank r.  Each sibling's y_i, dA_i and dB_i, and the sum of
the siblings' dx, are compared with the oracle's linear forward / backward of
that sibling alone (y and dx on sampled rows at the full sizes, dA and dB in
full).
"""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import siblings
from bit_nf4_quantized_28_b200 import workloads as wl
from parity_util import bits_of, check_close, oracle_backward, oracle_forward, oracle_storage, to_np

pytestmark = pytest.mark.gpu


def _layers(m, ns, k, r, alpha, seed, with_dy=True):
    """Sibling layers sharing x (drawn by the first); dy blocks of their own."""
    ts = [wl.make_linear(seed + i, n, k, m, r, alpha, a_std=1.0 / k, with_dy=with_dy) for i, n in enumerate(ns)]
    return ts, ts[0].x


def _rows(m, n=64, seed=0):
    g = np.random.default_rng(seed)
    return np.sort(g.choice(m, size=min(n, m), replace=False))


def _run(m, ns, k, r, alpha, seed=8000, backward=True, rows=None):
    ts, x = _layers(m, ns, k, r, alpha, seed, with_dy=backward)
    ws = [qn.quantize(t.W.cuda()) for t in ts]
    s = siblings.join(ws, [t.A.cuda() for t in ts], [t.B.cuda() for t in ts], alpha)
    xd = x.cuda()
    y, u = siblings.forward(xd, s)
    if backward:
        dy = torch.cat([t.dy for t in ts], dim=1)
        dx, dA, dB = siblings.backward(dy.cuda(), xd, s, u)
    torch.cuda.synchronize()
    assert qn.device_error() == 0
    sel = slice(None) if rows is None else rows
    ys = siblings.split_rows(y, s.n)
    xb = bits_of(x)
    dx_ref = 0.0
    if backward:
        dAs, dBs = siblings.split_grads(s, dA, dB)
        dys = siblings.split_rows(dy, s.n)
    for i, t in enumerate(ts):
        w_hat = oracle_storage(None, t.W)["w_hat"]
        a_bits, b_bits = bits_of(t.A), bits_of(t.B)
        y_ref, u_ref = oracle_forward(xb[sel], w_hat, a_bits, b_bits, alpha, r)
        check_close(to_np(ys[i])[sel], y_ref, f"y[{i}]")
        check_close(to_np(u[:, i * r:(i + 1) * r])[sel], u_ref, f"u[{i}]")
        if backward:
            dyb = bits_of(dys[i])
            dxi, _, _ = oracle_backward(dyb[sel], xb[sel], w_hat, a_bits, b_bits, alpha, r)
            dx_ref = dx_ref + dxi
            _, dAi, dBi = oracle_backward(dyb, xb, w_hat, a_bits, b_bits, alpha, r)
            check_close(to_np(dAs[i]), dAi, f"dA[{i}]")
            check_close(to_np(dBs[i]), dBi, f"dB[{i}]")
    if backward:
        check_close(to_np(dx)[sel], dx_ref, "dx (sum over siblings)")
    return s


@pytest.mark.parametrize("m", [300, 12])
def test_three_siblings(m):
    """q, k, v at 256 x 1024, rank 16, alpha 32: the GEMM path (m = 300) and
    the decode path (m = 12)."""
    _run(m, [256, 256, 256], 1024, 16, 32.0)


@pytest.mark.parametrize("m", [200, 8])
def test_uneven_groups(m):
    """Siblings of unequal height (k and v narrower than q, as with grouped
    attention heads), rank 8, four groups."""
    _run(m, [768, 256, 256, 512], 512, 8, 16.0, seed=8100)


def test_sibling_calls_equal_separate_calls():
    """Each sibling's block of the sibling call against its own layer call."""
    m, ns, k, r, alpha = 300, [256, 512, 256], 1024, 16, 32.0
    ts, x = _layers(m, ns, k, r, alpha, 8200, with_dy=False)
    ws = [qn.quantize(t.W.cuda()) for t in ts]
    s = siblings.join(ws, [t.A.cuda() for t in ts], [t.B.cuda() for t in ts], alpha)
    y, _ = siblings.forward(x.cuda(), s)
    for i, t in enumerate(ts):
        yi, _ = qn.linear_fwd(x.cuda(), ws[i], t.A.cuda(), t.B.cuda(), alpha)
        check_close(to_np(siblings.split_rows(y, s.n)[i]), to_np(yi).astype(np.float64), f"sibling vs own y[{i}]")


def test_join_weights_is_the_stacked_quantization():
    """Joining stored NF4 weights gives the storage of the stacked weight
    (whole groups of 256 block scales per sibling)."""
    ts, _ = _layers(4, [256, 256, 256], 1024, 16, 32.0, 8000, with_dy=False)
    ws = [qn.quantize(t.W.cuda()) for t in ts]
    joined = siblings.join_weights(ws)
    stacked = qn.quantize(torch.cat([t.W for t in ts]).cuda())
    for a, b in ((joined.codes, stacked.codes), (joined.qscale, stacked.qscale),
                 (joined.dq_step, stacked.dq_step), (joined.dq_mean, stacked.dq_mean)):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


# ------------------------------------------------------------------ full sizes

def test_qkv_full_size_decode():
    """q, k, v of a 4096-wide attention block at decode: 3 x 4096 x 4096, one
    token, rank 16, alpha 32 (the sibling decode the benchmark times)."""
    _run(1, [4096, 4096, 4096], 4096, 16, 32.0, seed=900, backward=False)


def test_qkv_full_size_train():
    """The same siblings over 2048 tokens, forward and backward; y and dx on
    64 sampled rows, u, dA and dB in full."""
    _run(2048, [4096, 4096, 4096], 4096, 16, 32.0, seed=900, rows=_rows(2048))


@pytest.mark.parametrize("m", [1, 2048])
def test_gate_up_full_size(m):
    """gate and up of a 7B MLP: 2 x 11008 x 4096, rank 16, alpha 16; decode
    (one token, forward) and 2048 tokens (forward and backward, sampled rows)."""
    _run(m, [11008, 11008], 4096, 16, 16.0, seed=950, backward=m > 1, rows=_rows(m) if m > 1 else None)
