"""Pins of the 8-bit AdamW oracle (CPU).

[LoRA y QLoRA en Profundidad, "Optimizadores Paginados": optim =
"paged_adamw_8bit", Adam with 8-bit states.]  The E4M3 grid and rounding are
pinned by torch's own float8_e4m3fn conversion, the quantization by its
error bound, and the step by torch.optim.AdamW run in fp64 (states at full
precision) and by Adam's first-step closed form.
"""

import numpy as np
import pytest
import torch

from oracle import adamw8


def _torch_codes(x):
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return np.where((t & 0x7F) == 0, 0, t).astype(np.uint8)     # zero stored as +0


def test_grid_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    grid = adamw8.e4m3_grid()
    assert grid.size == 127 and grid[-1] == 448.0 and grid[1] == 2.0 ** -9
    assert np.array_equal(codes[:127], grid)
    assert np.array_equal(codes[128:255], -grid)
    assert np.isnan(codes[127]) and np.isnan(codes[255])
    assert np.array_equal(adamw8.e4m3_decode(np.arange(127, dtype=np.uint8)), grid.astype(np.float32))


def test_encode_matches_torch_rounding():
    rng = np.random.default_rng(0)
    mags = np.exp2(rng.uniform(-14, np.log2(448.0), 20000)).astype(np.float32)
    x = mags * np.where(rng.random(mags.size) < 0.5, -1, 1).astype(np.float32)
    grid = adamw8.e4m3_grid()
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)           # exact ties
    x = np.concatenate([x, mids, -mids, np.float32([0.0, -0.0, 448.0, 448.00003, 2.0 ** -10, 2.0 ** -11])])
    assert np.array_equal(adamw8.e4m3_encode(x), _torch_codes(x))


def test_quantize_error_bound_and_ragged_blocks():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(1000) * np.exp2(rng.uniform(-12, 0, 1000))).astype(np.float32)
    x[256:512] = 0.0                                  # an all-zero block: scale 0, codes 0
    codes, scales = adamw8.quantize(x)
    assert scales.shape == (4,) and scales[1] == 0 and not codes[256:512].any()
    y = adamw8.dequantize(codes, scales)
    s = np.repeat(scales, 256)[:1000].astype(np.float64)
    # half an ulp of a 3-bit mantissa, or half the subnormal spacing (2^-9 scale)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(y - x) <= bound)
    for b in (0, 2, 3):
        blk = x[256 * b:256 * (b + 1)]
        assert scales[b] == np.float32(np.abs(blk).max() / np.float32(448))
        assert np.abs(y[256 * b:256 * (b + 1)]).max() == pytest.approx(np.abs(blk).max(), rel=1e-6)


def test_codes_are_the_nearest_grid_value():
    """Brute force: each code's value times the scale is a nearest grid
    point to x (no other E4M3 value is closer), for fp64 inputs."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal(512) * np.exp2(rng.uniform(-20, 5, 512))
    codes, scales = adamw8.quantize(x)
    grid = adamw8.e4m3_grid()
    allv = np.concatenate([grid, -grid[1:]])
    for b in range(2):
        s = float(scales[b])
        for i in range(256 * b, 256 * (b + 1)):
            y = x[i] / s
            best = np.abs(allv - y).min()
            got = adamw8.e4m3_decode(codes[i:i + 1])[0]
            assert abs(got - y) == best or (abs(y) >= 448 and abs(got) == 448)


def test_tiny_blocks():
    """Blocks near the bottom of fp32's range still get finite codes that
    decode within the bound (no NaN or infinite codes)."""
    x = (np.linspace(-1, 1, 256) * 1e-37).astype(np.float32)
    codes, scales = adamw8.quantize(x)
    assert scales[0] > 0
    assert (codes & 0x7F).max() <= 126
    y = adamw8.dequantize(codes, scales)
    assert np.all(np.abs(y - x) <= np.maximum(np.abs(x) * 2.0 ** -4, float(scales[0]) * 2.0 ** -10) * (1 + 1e-6)
                  + 1e-45)


HP = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _torch_adamw_f64(p0, grads):
    """torch.optim.AdamW in fp64 with the fp32 values of the hyperparameters
    (what the oracle's caller passes through the fp32 interface)."""
    lr, b1, b2, eps, wd = adamw8.hyper(**HP)
    tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([tp], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd, foreach=False)
    for g in grads:
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
    st = opt.state[tp]
    return tp.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()


def _oracle_f64(p0, grads):
    lr, b1, b2, eps, wd = adamw8.hyper(**HP)
    p, m, v = p0.astype(np.float64), np.zeros(p0.size), np.zeros(p0.size)
    for t, g in enumerate(grads, start=1):
        p, m, v = adamw8.adamw_step(p, g, m, v, lr, b1, b2, eps, wd, t)
    return p, m, v


def test_full_precision_steps_match_torch_adamw():
    rng = np.random.default_rng(2)
    p0 = rng.standard_normal(700).astype(np.float32) * 0.02
    grads = [rng.standard_normal(700).astype(np.float32) * 1e-3 for _ in range(5)]
    tp, tm, tv = _torch_adamw_f64(p0, grads)
    p, m, v = _oracle_f64(p0, grads)
    # both in fp64, differing only in rounding order: far below one step (lr)
    assert np.allclose(p, tp, rtol=0, atol=HP["lr"] * 1e-10)
    assert np.allclose(m, tm, rtol=1e-12, atol=0)
    assert np.allclose(v, tv, rtol=1e-12, atol=0)


def test_first_step_closed_form():
    """From zero states Adam's first bias-corrected moments are g and g^2, so
    the update is lr g / (|g| + eps), after the decoupled decay."""
    rng = np.random.default_rng(3)
    p = rng.standard_normal(512).astype(np.float32)
    g = (rng.standard_normal(512) * 1e-2).astype(np.float32)
    z8, z32 = np.zeros(512, np.uint8), np.zeros(2, np.float32)
    lr, b1, b2, eps, wd = adamw8.hyper(**HP)
    p2, m, v, mc, ms, vc, vs = adamw8.step(p, g, z8, z32, z8, z32, t=1, **HP)
    g64 = g.astype(np.float64)
    want = p.astype(np.float64) * (1 - lr * wd) - lr * g64 / (np.abs(g64) + eps)
    assert np.allclose(p2, want, rtol=1e-13, atol=0)
    # the stored moments are (1 - beta1) g and (1 - beta2) g^2, 8-bit
    m_want = (1 - b1) * g64
    v_want = (1 - b2) * g64 * g64
    assert np.allclose(m, m_want, rtol=1e-15, atol=0) and np.allclose(v, v_want, rtol=1e-15, atol=0)
    assert np.allclose(adamw8.dequantize(mc, ms), m_want, rtol=2.0 ** -4, atol=ms.max() * 2.0 ** -10)
    assert np.allclose(adamw8.dequantize(vc, vs), v_want, rtol=2.0 ** -4, atol=vs.max() * 2.0 ** -10)


def test_zero_gradient_only_decays():
    p = np.linspace(-1, 1, 300, dtype=np.float32)
    z8, z32 = np.zeros(300, np.uint8), np.zeros(2, np.float32)
    lr, b1, b2, eps, wd = adamw8.hyper(**HP)
    p2, m, v, mc, ms, vc, vs = adamw8.step(p, np.zeros(300, np.float32), z8, z32, z8, z32, t=4, **HP)
    assert np.array_equal(p2, p.astype(np.float64) * (1 - lr * wd))
    assert not mc.any() and not vc.any() and not ms.any() and not vs.any()


def test_eight_bit_states_track_full_precision():
    """Ten steps with 8-bit states stay close to the same steps with full
    precision states (the 8-bit error is relative to each block's largest
    moment)."""
    rng = np.random.default_rng(4)
    n = 1024
    p = rng.standard_normal(n).astype(np.float32) * 0.02
    grads = [(rng.standard_normal(n) * 1e-3).astype(np.float32) for _ in range(10)]
    mc, vc = np.zeros(n, np.uint8), np.zeros(n, np.uint8)
    ms, vs = np.zeros(4, np.float32), np.zeros(4, np.float32)
    p8 = p.astype(np.float64)
    for t, g in enumerate(grads, start=1):
        p8, _, _, mc, ms, vc, vs = adamw8.step(p8, g, mc, ms, vc, vs, t=t, **HP)
    pf, _, _ = _oracle_f64(p, grads)
    # each step moves a weight by about lr; the 8-bit states change a step by a few per cent
    assert np.abs(p8 - pf).max() < 0.15 * 10 * HP["lr"]
    assert np.abs(p8 - pf).mean() < 0.02 * 10 * HP["lr"]
