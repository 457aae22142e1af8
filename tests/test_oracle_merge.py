"""Pins of the LoRA merge oracle (CPU).

[LoRA y QLoRA en Profundidad, "Cómo Funciona LoRA"]: W_final = W + (alpha/r) B @ A;
[QLoRA glossary, "Compromessi"]: the 4-bit base is dequantized before merging.
"""

import numpy as np
import torch

from bit_nf4_quantized_28_b200 import workloads as wl
from oracle import linear, merge, nf4


def _layer(seed=5, n=64, k=128, r=8, b_zero=False):
    t = wl.make_linear(seed, n, k, 4, r, 16.0, a_std=1.0 / k, with_dy=False)
    q = nf4.quantize(wl.bits(t.W), n, k)
    what = nf4.dequantize(q["codes"], q["qscale"], q["step"], q["mean"], n, k)
    a = wl.bits(t.A)
    b = np.zeros_like(wl.bits(t.B)) if b_zero else wl.bits(t.B)
    return t, what, a, b


def test_b_zero_gives_the_dequantized_weight():
    """B = 0 (the LoRA start): the merge is W_hat itself, bit for bit."""
    t, what, a, b = _layer(b_zero=True)
    assert np.array_equal(merge.merge(what, a, b, t.alpha, t.r), what)


def test_rank_zero_is_the_dequantized_weight():
    t, what, a, b = _layer()
    assert np.array_equal(merge.merge(what, None, None, t.alpha, 0), what)


def test_matches_brute_force_loops():
    """W_hat + s B @ A against textbook loops (tiny shape), before rounding."""
    t, what, a, b = _layer(n=16, k=64, r=8)
    w = nf4.bf16_bits_to_f64(what)
    ba = np.array(linear.matmul_loops(nf4.bf16_bits_to_f64(b).tolist(), nf4.bf16_bits_to_f64(a).tolist()))
    ref = w + linear.lora_scale(t.alpha, t.r) * ba
    assert np.allclose(merge.merge_f64(what, a, b, t.alpha, t.r), ref, rtol=0, atol=1e-15)


def test_one_hot_adapter():
    """A = e_j rows, B = columns of constants: each row of W_hat moves by s * c
    at the columns the one-hot rows select (a closed form)."""
    n, k, r, alpha = 8, 64, 8, 16.0
    what = wl.bits(torch.randn(n, k, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16) * 0.02)
    a = np.zeros((r, k), np.float32)
    for j in range(r):
        a[j, 3 * j] = 1.0
    b = np.full((n, r), 0.5, np.float32)
    a_bits = nf4.f32_to_bf16_bits(a)
    b_bits = nf4.f32_to_bf16_bits(b)
    got = merge.merge_f64(what, a_bits, b_bits, alpha, r)
    want = nf4.bf16_bits_to_f64(what).copy()
    want[:, [3 * j for j in range(r)]] += (alpha / r) * 0.5
    assert np.array_equal(got, want)


def test_rounding_is_nearest_even():
    """f64 -> bf16 rounding on hand-picked values: exact bf16 values, halfway
    cases (to even) and just off halfway."""
    one = 1.0
    ulp = 2.0 ** -7
    vals = np.array([one, one + ulp / 2, one + 3 * ulp / 2, one + ulp / 2 + 1e-12, -(one + ulp / 2), 0.0])
    got = nf4.bf16_bits_to_f64(merge.f64_to_bf16_bits(vals))
    assert list(got) == [1.0, 1.0, 1.0 + 2 * ulp, 1.0 + ulp, -1.0, 0.0]


def test_tie_margin():
    ulp = 2.0 ** -7
    m = merge.tie_margin(np.array([1.0, 1.0 + ulp / 2, 1.0 + ulp / 4]))
    assert np.allclose(m, [0.5, 0.0, 0.25])
