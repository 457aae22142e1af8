"""GPU parity of the QLoRA linear (forward on both paths, backward) against
the oracle: y, dx, dA, dB within max|err| <= 2e-2 rms and mean relative
error <= 5e-3.  Sizes span several tiles with ragged tails; the full-size
workloads are checked on seeded row samples (y, dx are row-separable) and in
full for dA, dB."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import workloads as wl
from parity_util import bits_of, check_close, oracle_backward, oracle_forward, oracle_storage, to_np

pytestmark = pytest.mark.gpu


def _gpu_layer(t):
    W = t.W.cuda()
    w = qn.quantize(W)
    return w


def _fwd_bwd(t, path="auto", rows=None, b_zero=False, r_override=None):
    """Runs forward + backward on the GPU and the oracle; compares."""
    w = _gpu_layer(t)
    x, dy = t.x.cuda(), t.dy.cuda() if t.dy is not None else None
    A, B = t.A.cuda(), t.B.cuda()
    if b_zero:
        B = torch.zeros_like(B)
    fwd = {"auto": qn.linear_fwd, "gemm": qn.linear_fwd_gemm, "gemv": qn.linear_fwd_gemv}[path]
    y, u = fwd(x, w, A, B, t.alpha)
    out = {"y": y, "u": u}
    if dy is not None:
        dx, dA, dB = qn.linear_bwd(dy, x, w, A, B, t.alpha, u)
        out.update(dx=dx, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert qn.device_error() == 0

    st = oracle_storage((t.n_out, t.k_in, id(t.W)), t.W)
    b_bits = bits_of(B)
    sel = slice(None) if rows is None else rows
    y_ref, u_ref = oracle_forward(bits_of(t.x)[sel], st["w_hat"], bits_of(t.A), b_bits, t.alpha, t.r)
    check_close(to_np(y)[sel], y_ref, "y")
    if u is not None:
        check_close(to_np(u)[sel], u_ref, "u")
    if dy is not None:
        dx_ref, _, _ = oracle_backward(bits_of(t.dy)[sel], bits_of(t.x)[sel], st["w_hat"], bits_of(t.A),
                                       b_bits, t.alpha, t.r)
        check_close(to_np(out["dx"])[sel], dx_ref, "dx")
        _, dA_ref, dB_ref = oracle_backward(bits_of(t.dy), bits_of(t.x), st["w_hat"], bits_of(t.A),
                                            b_bits, t.alpha, t.r)
        if b_zero:
            assert torch.count_nonzero(out["dA"]) == 0
        else:
            check_close(to_np(out["dA"]), dA_ref, "dA")
        check_close(to_np(out["dB"]), dB_ref, "dB")
    return out


# ------------------------------------------------------------------ tiny workload

@pytest.mark.parametrize("path", ["auto", "gemm", "gemv"])
def test_tiny(path):
    """256 x 256, 16 tokens, r 8, alpha 16 (seed 0)."""
    _fwd_bwd(wl.tiny(), path=path)


@pytest.mark.parametrize("path", ["gemm", "gemv"])
def test_tiny_b_zero_equals_base(path):
    """B = 0 (LoRA start): y equals the base-only output exactly, dA = 0."""
    t = wl.tiny()
    out = _fwd_bwd(t, path=path, b_zero=True)
    w = _gpu_layer(t)
    fwd = qn.linear_fwd_gemm if path == "gemm" else qn.linear_fwd_gemv
    y0, _ = fwd(t.x.cuda(), w)
    dx0, _, _ = qn.linear_bwd(t.dy.cuda(), t.x.cuda(), w)
    torch.cuda.synchronize()
    assert torch.equal(out["y"].float(), y0.float())
    assert torch.equal(out["dx"].float(), dx0.float())


# ------------------------------------------------------------------ tiles and tails

@pytest.mark.parametrize("m,n,k,r", [
    (300, 384, 320, 16),      # ragged M vs the 256-row tile, 3 N tiles, 5 k-blocks
    (17, 128, 64, 8),         # one k-block, smallest GEMM M above the decode path
    (512, 256, 1024, 64),
    (257, 640, 192, 128),     # two LoRA k-blocks
    (64, 192, 128, 0),        # no LoRA
])
def test_gemm_tiles(m, n, k, r):
    t = wl.make_linear(1000 + m + n + k + r, n, k, m, max(r, 8), 2.0 * max(r, 8), a_std=1.0 / k)
    if r == 0:
        w = _gpu_layer(t)
        y, _ = qn.linear_fwd(t.x.cuda(), w)
        dx, _, _ = qn.linear_bwd(t.dy.cuda(), t.x.cuda(), w)
        torch.cuda.synchronize()
        st = oracle_storage((n, k, id(t.W)), t.W)
        y_ref, _ = oracle_forward(bits_of(t.x), st["w_hat"], None, None, 0.0, 0)
        dx_ref, _, _ = oracle_backward(bits_of(t.dy), bits_of(t.x), st["w_hat"], None, None, 0.0, 0)
        check_close(to_np(y), y_ref, "y")
        check_close(to_np(dx), dx_ref, "dx")
    else:
        _fwd_bwd(t)


def test_backward_recomputes_u():
    """Without the forward's u, the backward computes u = x A^T itself (with
    v, before the dx GEMM).  Those launches may split their reductions
    differently from the ones that run beside a GEMM, so u and v can round
    differently: both sets of gradients must meet the oracle."""
    t = wl.make_linear(77, 256, 512, 96, 16, 32.0, a_std=1.0 / 512)
    w = _gpu_layer(t)
    x, dy, A, B = t.x.cuda(), t.dy.cuda(), t.A.cuda(), t.B.cuda()
    y, u = qn.linear_fwd(x, w, A, B, t.alpha)
    g1 = qn.linear_bwd(dy, x, w, A, B, t.alpha, u)
    g2 = qn.linear_bwd(dy, x, w, A, B, t.alpha, None)
    torch.cuda.synchronize()
    assert qn.device_error() == 0
    st = oracle_storage((t.n_out, t.k_in, id(t.W)), t.W)
    dx_ref, dA_ref, dB_ref = oracle_backward(bits_of(t.dy), bits_of(t.x), st["w_hat"], bits_of(t.A),
                                             bits_of(t.B), t.alpha, t.r)
    for g in (g1, g2):
        check_close(to_np(g[0]), dx_ref, "dx")
        check_close(to_np(g[1]), dA_ref, "dA")
        check_close(to_np(g[2]), dB_ref, "dB")


def test_dx_skipped():
    t = wl.make_linear(78, 256, 256, 64, 8, 16.0, a_std=1.0 / 256)
    w = _gpu_layer(t)
    dx, dA, dB = qn.linear_bwd(t.dy.cuda(), t.x.cuda(), w, t.A.cuda(), t.B.cuda(), t.alpha, None,
                               need_dx=False)
    torch.cuda.synchronize()
    assert dx is None and dA is not None


# ------------------------------------------------------------------ decode path

@pytest.mark.parametrize("t_tok", [1, 2, 4, 7, 8, 9, 16])
def test_gemv_tokens(t_tok):
    t = wl.make_linear(2000 + t_tok, 512, 1024, t_tok, 64, 16.0, a_std=1.0 / 1024, with_dy=False)
    _fwd_bwd(t, path="gemv")


@pytest.mark.parametrize("t_tok,k", [(4, 4352), (16, 4352), (1, 11008)])
def test_gemv_split_k(t_tok, k):
    """Long K: more k-ranges of 256 than warps in a CTA (17 and 43 of them),
    so warps change k-range within the main loop and the parked tiles of a
    row group span many warps."""
    t = wl.make_linear(3000 + t_tok + k, 256, k, t_tok, 32, 16.0, a_std=1.0 / k, with_dy=False)
    _fwd_bwd(t, path="gemv")


def test_gemv_matches_gemm_path():
    t = wl.make_linear(4000, 768, 2048, 12, 16, 32.0, a_std=1.0 / 2048, with_dy=False)
    w = _gpu_layer(t)
    a = qn.linear_fwd_gemv(t.x.cuda(), w, t.A.cuda(), t.B.cuda(), t.alpha)[0]
    b = qn.linear_fwd_gemm(t.x.cuda(), w, t.A.cuda(), t.B.cuda(), t.alpha)[0]
    torch.cuda.synchronize()
    check_close(to_np(a), to_np(b).astype(np.float64), "gemv vs gemm")


# ------------------------------------------------------------------ full-size workloads

def _rows(m, n=64, seed=0):
    g = np.random.default_rng(seed)
    return np.sort(g.choice(m, size=min(n, m), replace=False))


def test_train_config_full_size():
    """d_in = d_out = 4096, x 2048 x 4096, r 16, alpha 32 (seed 2): y and dx
    on 64 sampled rows, dA and dB in full."""
    t = wl.train()
    _fwd_bwd(t, rows=_rows(t.m))


@pytest.mark.parametrize("shape", wl.DECODE_SHAPES)
def test_decode_config_full_size(shape):
    """4096 -> 11008 and 11008 -> 4096, T = 1, 4, 16, r 64, alpha 16 (seed 3)."""
    n, k = shape
    base = wl.decode(n, k)
    w = _gpu_layer(base)
    st = oracle_storage((n, k, id(base.W)), base.W)
    A, B = base.A.cuda(), base.B.cuda()
    for T in wl.DECODE_TOKENS:
        x = base.x[:T]
        y, _ = qn.linear_fwd(x.cuda(), w, A, B, base.alpha)
        torch.cuda.synchronize()
        y_ref, _ = oracle_forward(bits_of(x), st["w_hat"], bits_of(base.A), bits_of(base.B), base.alpha, base.r)
        check_close(to_np(y), y_ref, f"y T={T}")
    assert qn.device_error() == 0


@pytest.mark.parametrize("name", ["q", "gate", "up", "down"])
def test_block7b_linear_full_size(name):
    """The 7B block's linear shapes at M = 8192 (r 16, alpha 16): q (as k, v
    and o, 4096 x 4096), gate and up (11008 x 4096) and down (4096 x 11008);
    y and dx on sampled rows, dA and dB in full."""
    t = wl.block7b_layer(name)
    _fwd_bwd(t, rows=_rows(t.m, seed=1))
