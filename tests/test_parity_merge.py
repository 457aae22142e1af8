"""GPU parity of the LoRA merge (W_hat + (alpha/r) B A -> bf16) against the oracle.

[LoRA y QLoRA en Profundidad, "Cómo Funciona LoRA"]: W_final = W + (alpha/r) B @ A;
[QLoRA glossary, "Compromessi"]: the 4-bit base is dequantized before merging.

The kernel accumulates B A in fp32 and rounds the fp32 sum once to bf16; the
oracle rounds the exact fp64 value.  The two can differ only where the value
lies within a few fp32 ulps of a bf16 rounding boundary: the test asks for
bit equality everywhere else and for at most one bf16 ulp at such points.
"""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import workloads as wl
from oracle import merge as omerge
from oracle import nf4
from parity_util import bits_of, oracle_storage

pytestmark = pytest.mark.gpu

TIE = 1e-4       # in bf16 ulps: far above the fp32 accumulation error, far below a rounding step


def _ulps(a_bits, b_bits):
    """Distance in bf16 ulps of same-sign finite values (as ordered integers)."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(key(a_bits) - key(b_bits))


def _check(t, r, rows=None, b_zero=False):
    w = qn.quantize(t.W.cuda())
    A = t.A.cuda() if r else None
    B = (torch.zeros_like(t.B) if b_zero else t.B).cuda() if r else None
    got = bits_of(qn.merge(w, A, B, t.alpha))
    torch.cuda.synchronize()
    q = oracle_storage(None, t.W)
    what = q["w_hat"]
    a_bits = wl.bits(t.A) if r else None
    b_bits = (np.zeros_like(wl.bits(t.B)) if b_zero else wl.bits(t.B)) if r else None
    if rows is not None:
        got, what = got[rows], what[rows]
        b_bits = b_bits[rows] if r else None
    exact = omerge.merge_f64(what, a_bits, b_bits, t.alpha, r)
    ref = omerge.f64_to_bf16_bits(exact)
    d = _ulps(got, ref)
    near_tie = omerge.tie_margin(exact) < TIE
    assert np.all(d[~near_tie] == 0), f"{int((d[~near_tie] != 0).sum())} mismatches away from ties"
    assert np.all(d <= 1)
    return what, got


def test_tiny():
    _check(wl.tiny(), 8)


def test_rank_zero_and_b_zero_equal_dequantize():
    """r = 0 and B = 0 both give W_hat, bit for bit (the dequantized weight)."""
    t = wl.tiny()
    w = qn.quantize(t.W.cuda())
    wh = bits_of(qn.dequantize(w))
    assert np.array_equal(bits_of(qn.merge(w)), wh)
    assert np.array_equal(bits_of(qn.merge(w, t.A.cuda(), torch.zeros_like(t.B).cuda(), t.alpha)), wh)


@pytest.mark.parametrize("n,k,r", [(128, 320, 16), (64, 256, 128), (192, 448, 24), (64, 128, 8)])
def test_shapes(n, k, r):
    """Ragged column tiles (k % 128 != 0), the largest rank, r % 16 == 8."""
    t = wl.make_linear(6000 + n + k + r, n, k, 4, r, 16.0, a_std=1.0 / k, with_dy=False)
    _check(t, r)


def test_requantize_is_quantize_of_the_merge():
    t = wl.tiny()
    w = qn.quantize(t.W.cuda())
    m = qn.merge(w, t.A.cuda(), t.B.cuda(), t.alpha)
    q1 = qn.merge(w, t.A.cuda(), t.B.cuda(), t.alpha, requantize=True)
    q2 = qn.quantize(m)
    for a, b in ((q1.codes, q2.codes), (q1.qscale, q2.qscale), (q1.dq_step, q2.dq_step), (q1.dq_mean, q2.dq_mean)):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def test_full_size_sampled_rows():
    """The training weight 4096 x 4096, rank 16, on seeded sampled rows."""
    t = wl.train()
    rows = np.sort(np.random.default_rng(7).choice(t.n_out, 96, replace=False))
    _check(t, t.r, rows=rows)
