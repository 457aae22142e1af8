"""Pins of the oracle's frozen linear (forward and backward) — no GPU.

Checks: brute-force triple loops on tiny shapes, central finite differences of
<dy, y> (exact up to rounding because y is linear in each argument), the
B = 0 start of LoRA (update is zero), and the LoRA parameter counts the pages
print.
"""

import numpy as np
import pytest

from oracle import linear, nf4
from bit_nf4_quantized_28_b200 import workloads as wl


def _tiny(seed=1, m=4, k=8, n=6, r=2):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((m, k)), rng.standard_normal((n, k)),
            rng.standard_normal((r, k)), rng.standard_normal((n, r)),
            rng.standard_normal((m, n)))


def test_forward_brute_force_loops():
    x, w, a, b, _ = _tiny()
    s = 1.75
    y, u = linear.forward_f64(x, w, a, b, s)
    base = linear.matmul_loops(x.tolist(), w.T.tolist())
    uu = linear.matmul_loops(x.tolist(), a.T.tolist())
    up = linear.matmul_loops(uu, b.T.tolist())
    ref = np.array(base) + s * np.array(up)
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(u, np.array(uu), rtol=1e-13, atol=1e-13)


def test_backward_brute_force_loops():
    x, w, a, b, dy = _tiny(2)
    s = 0.5
    dx, da, db = linear.backward_f64(dy, x, w, a, b, s)
    v = np.array(linear.matmul_loops(dy.tolist(), b.tolist()))
    ref_dx = np.array(linear.matmul_loops(dy.tolist(), w.tolist())) + s * np.array(
        linear.matmul_loops(v.tolist(), a.tolist()))
    ref_da = s * np.array(linear.matmul_loops(v.T.tolist(), x.tolist()))
    u = np.array(linear.matmul_loops(x.tolist(), a.T.tolist()))
    ref_db = s * np.array(linear.matmul_loops(dy.T.tolist(), u.tolist()))
    assert np.allclose(dx, ref_dx, rtol=1e-13, atol=1e-13)
    assert np.allclose(da, ref_da, rtol=1e-13, atol=1e-13)
    assert np.allclose(db, ref_db, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("which", ["x", "a", "b"])
def test_gradients_match_finite_differences(which):
    """Central differences of L = <dy, y(x, A, B)> on 16x64x64, r = 4."""
    x, w, a, b, dy = _tiny(3, m=16, k=64, n=64, r=4)
    s = 2.0
    dx, da, db = linear.backward_f64(dy, x, w, a, b, s)
    params = {"x": x, "a": a, "b": b}
    grads = {"x": dx, "a": da, "b": db}
    p = params[which]
    rng = np.random.default_rng(7)
    h = 1e-3
    for _ in range(12):
        idx = tuple(rng.integers(0, d) for d in p.shape)
        old = p[idx]
        p[idx] = old + h
        lp = np.sum(dy * linear.forward_f64(x, w, a, b, s)[0])
        p[idx] = old - h
        lm = np.sum(dy * linear.forward_f64(x, w, a, b, s)[0])
        p[idx] = old
        fd = (lp - lm) / (2 * h)
        assert abs(fd - grads[which][idx]) <= 1e-8 * max(1.0, abs(fd))


def test_b_zero_gives_base_output_and_zero_da():
    """B = 0 at LoRA start: the update B @ A is zero, so y equals the base
    output exactly and dA = 0 [skyvanguard lesson, "Inicialización"]."""
    t = wl.tiny()
    q = nf4.quantize(wl.bits(t.W), t.n_out, t.k_in)
    wh = nf4.dequantize(q["codes"], q["qscale"], q["step"], q["mean"], t.n_out, t.k_in)
    zero_b = np.zeros((t.n_out, t.r), np.uint16)
    y0, _ = linear.forward(wl.bits(t.x), wh, None, None, t.alpha, 0)
    y1, _ = linear.forward(wl.bits(t.x), wh, wl.bits(t.A), zero_b, t.alpha, t.r)
    assert np.array_equal(y0, y1)
    dx0, _, _ = linear.backward(wl.bits(t.dy), wl.bits(t.x), wh, None, None, t.alpha, 0)
    dx1, da, db = linear.backward(wl.bits(t.dy), wl.bits(t.x), wh, wl.bits(t.A), zero_b, t.alpha, t.r)
    assert np.array_equal(dx0, dx1)
    assert np.all(da == 0)
    assert np.any(db != 0)


def test_lora_scale():
    assert linear.lora_scale(16, 8) == 2.0
    assert linear.lora_scale(32, 16) == 2.0
    assert linear.lora_scale(16, 64) == 0.25
    assert linear.lora_scale(16, 16) == 1.0


def test_lora_parameter_counts(golden):
    g = golden("lora_params.txt")
    assert 4096 * 4096 == int(g["full_4096"])
    for r in (8, 16, 32, 64):
        t = wl.make_linear(0, 32, 4096, 1, r, 2.0 * r)
        assert t.A.numel() + 4096 * r == int(g[f"lora_r{r}"])
    assert round(100 * (1 - 131072 / 16777216), 1) == float(g["reduction_percent"])
