"""GPU parity of LoRA dropout against the oracle.

The keep mask and x_drop are compared bit for bit (integer work); y, u, dx,
dA and dB within the layer's tolerance (max |err| <= 2e-2 rms, mean relative
error <= 5e-3).  The mask the kernels drew is checked against the oracle's
Philox draw first, and the layer's outputs are then compared with the
oracle run on that same mask.  Shapes cover several tiles, ragged rows,
columns that end in half a tile, ranks that are not multiples of 16, and the
full training shape (rows sampled for y and dx)."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import workloads as wl
from oracle import dropout as od
from parity_util import bits_of, check_close, oracle_storage, to_np

pytestmark = pytest.mark.gpu


def _keep_np(keep_t):
    return keep_t.cpu().numpy().view(np.uint32)


def _check_mask(x, x_drop, keep, p, seed, offset, rows=None):
    m, k = x.shape
    ref = od.keep_mask(m, k, p, seed, offset)
    assert np.array_equal(_keep_np(keep), od.pack_keep(ref))
    assert np.array_equal(bits_of(x_drop), od.apply_bits(bits_of(x), ref))
    return ref


@pytest.mark.parametrize("m,k", [(1, 32), (3, 64), (37, 192), (16, 4096), (300, 320)])
def test_mask_bit_exact(m, k):
    g = torch.Generator().manual_seed(m * 1000 + k)
    x = wl.normal_bf16(g, (m, k), 1.0).cuda()
    seed, offset = 0x0123456789ABCDEF, 0xFEDCBA9876543210
    x_drop, keep = qn.dropout(x, 0.05, seed, offset)
    torch.cuda.synchronize()
    _check_mask(x, x_drop, keep, 0.05, seed, offset)


@pytest.mark.parametrize("p", [0.0, 0.1, 0.5, 0.999])
def test_mask_rates(p):
    g = torch.Generator().manual_seed(3)
    x = wl.normal_bf16(g, (64, 1024), 1.0).cuda()
    x_drop, keep = qn.dropout(x, p, seed=17, offset=5)
    torch.cuda.synchronize()
    ref = _check_mask(x, x_drop, keep, p, 17, 5)
    if p == 0.0:
        assert ref.all() and torch.equal(x_drop, x)


def _layer_case(t, p, seed, offset, rows=None, use_u=True):
    w = qn.quantize(t.W.cuda())
    x, dy, A, B = t.x.cuda(), t.dy.cuda(), t.A.cuda(), t.B.cuda()
    y, u, x_drop, keep = qn.linear_fwd_dropout(x, w, A, B, t.alpha, p, seed, offset)
    dx, dA, dB = qn.linear_bwd_dropout(dy, x_drop, keep, w, A, B, t.alpha, p, u if use_u else None)
    torch.cuda.synchronize()
    assert qn.device_error() == 0
    keep_ref = _check_mask(x, x_drop, keep, p, seed, offset)
    st = oracle_storage((t.n_out, t.k_in, id(t.W)), t.W)
    sel = slice(None) if rows is None else rows
    xb, ab, bb, dyb = bits_of(t.x), bits_of(t.A), bits_of(t.B), bits_of(t.dy)
    y_ref, u_ref = od.forward(xb[sel], st["w_hat"], ab, bb, t.alpha, t.r, p, keep_ref[sel])
    check_close(to_np(y)[sel], y_ref, "y")
    # u_save holds x_drop A^T; the definition's u = dropout(x) A^T carries the 1 / (1 - p)
    check_close(to_np(u)[sel] / (1.0 - float(np.float32(p))), u_ref, "u")
    dx_ref, _, _ = od.backward(dyb[sel], xb[sel], st["w_hat"], ab, bb, t.alpha, t.r, p, keep_ref[sel])
    check_close(to_np(dx)[sel], dx_ref, "dx")
    _, dA_ref, dB_ref = od.backward(dyb, xb, st["w_hat"], ab, bb, t.alpha, t.r, p, keep_ref)
    check_close(to_np(dA), dA_ref, "dA")
    check_close(to_np(dB), dB_ref, "dB")
    return dict(y=y, u=u, dx=dx, dA=dA, dB=dB, x_drop=x_drop, keep=keep, w=w)


def test_tiny():
    """256 x 256, 16 tokens, r 8, p = 0.05 (the lesson's rate)."""
    t = wl.tiny()
    _layer_case(t, 0.05, seed=42, offset=0)


@pytest.mark.parametrize("m,n,k,r,p", [(37, 192, 320, 24, 0.1), (300, 256, 448, 16, 0.05),
                                       (130, 128, 256, 128, 0.3), (2304, 4096, 256, 16, 0.05)])
def test_shapes(m, n, k, r, p):
    """Ragged rows, half-tile columns, r not a multiple of 16, r = 128, and a
    GEMM that leaves no SMs idle (u then runs before it on every SM)."""
    t = wl.make_linear(m + n + k, n, k, m, r, 2.0 * r, a_std=1.0 / k)
    _layer_case(t, p, seed=m * 7 + 1, offset=r)


def test_recomputed_u_matches_saved_u():
    t = wl.make_linear(9, 256, 512, 96, 16, 32.0, a_std=1.0 / 512)
    a = _layer_case(t, 0.05, seed=3, offset=1, use_u=True)
    b = _layer_case(t, 0.05, seed=3, offset=1, use_u=False)
    assert torch.allclose(a["dA"], b["dA"], rtol=1e-5, atol=1e-7)
    assert torch.allclose(a["dB"], b["dB"], rtol=1e-5, atol=1e-7)


def test_p_zero_forward_is_the_plain_layer():
    """p = 0 keeps every element and s_d = s: the forward's launches see the
    same inputs as the plain GEMM forward, so y and u are bit-identical."""
    t = wl.make_linear(12, 256, 256, 64, 16, 32.0, a_std=1.0 / 256)
    w = qn.quantize(t.W.cuda())
    x, A, B = t.x.cuda(), t.A.cuda(), t.B.cuda()
    y, u, x_drop, keep = qn.linear_fwd_dropout(x, w, A, B, t.alpha, 0.0, seed=5)
    y0, u0 = qn.linear_fwd_gemm(x, w, A, B, t.alpha)
    torch.cuda.synchronize()
    assert torch.equal(x_drop, x)
    assert bool((keep == -1).all())
    assert torch.equal(y, y0) and torch.equal(u, u0)


def test_no_dx():
    t = wl.make_linear(13, 128, 256, 32, 8, 16.0, a_std=1.0 / 256)
    w = qn.quantize(t.W.cuda())
    x, dy, A, B = t.x.cuda(), t.dy.cuda(), t.A.cuda(), t.B.cuda()
    y, u, x_drop, keep = qn.linear_fwd_dropout(x, w, A, B, t.alpha, 0.1, seed=8)
    dx, dA, dB = qn.linear_bwd_dropout(dy, x_drop, None, w, A, B, t.alpha, 0.1, u, need_dx=False)
    dx1, dA1, dB1 = qn.linear_bwd_dropout(dy, x_drop, keep, w, A, B, t.alpha, 0.1, u)
    torch.cuda.synchronize()
    assert dx is None
    assert torch.allclose(dA, dA1, rtol=1e-5, atol=1e-7) and torch.allclose(dB, dB1, rtol=1e-5, atol=1e-7)


def test_training_shape():
    """x 2048 x 4096, W 4096 x 4096, r 16, alpha 32, p = 0.05: the mask in
    full, y and dx on 64 seeded rows, dA and dB in full."""
    t = wl.train()
    rows = np.sort(np.random.default_rng(0).choice(t.m, 64, replace=False))
    _layer_case(t, 0.05, seed=2024, offset=7, rows=rows)
