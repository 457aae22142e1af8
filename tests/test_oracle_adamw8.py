"""Pins of the 8-bit AdamW oracle (CPU).

[LoRA y QLoRA en Profundidad, "Optimizadores Paginados": optim =
"paged_adamw_8bit", Adam with 8-bit states.]  The E4M3 grid and rounding are
pinned by torch's own float8_e4m3fn conversion, the quantization by its
error bound, and the step by torch.optim.AdamW (states at full precision)
and by Adam's first-step closed form.
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
    s = np.repeat(scales, 256)[:1000]
    # half an ulp of a 3-bit mantissa, or half the subnormal spacing (2^-9 scale)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(y - x) <= bound)
    for b in (0, 2, 3):
        blk = x[256 * b:256 * (b + 1)]
        assert scales[b] == np.float32(np.abs(blk).max() / np.float32(448))
        assert np.abs(y[256 * b:256 * (b + 1)]).max() == pytest.approx(np.abs(blk).max(), rel=1e-6)


def test_tiny_blocks_use_the_division():
    """Where 448 / absmax overflows fp32, the codes come from x / scale and
    still decode to x within the bound (no NaN or infinite codes)."""
    x = (np.linspace(-1, 1, 256) * 1e-37).astype(np.float32)
    codes, scales = adamw8.quantize(x)
    with np.errstate(over="ignore"):
        assert np.isinf(np.float32(448) / np.abs(x).max()) and scales[0] > 0
    assert (codes & 0x7F).max() <= 126
    y = adamw8.dequantize(codes, scales)
    assert np.all(np.abs(y - x) <= np.maximum(np.abs(x) * 2.0 ** -4, scales[0] * 2.0 ** -10) * (1 + 1e-6) + 1e-45)


# hyperparameters exact in fp32 (the C ABI passes fp32), so that torch's fp64
# scalars and the oracle's fp32 ones are the same numbers
HP = dict(lr=2.0 ** -12, beta1=0.875, beta2=1 - 2.0 ** -10, eps=2.0 ** -27, weight_decay=2.0 ** -6)


def test_full_precision_steps_match_torch_adamw():
    rng = np.random.default_rng(2)
    p0 = rng.standard_normal(700).astype(np.float32) * 0.02
    grads = [rng.standard_normal(700).astype(np.float32) * 1e-3 for _ in range(5)]
    tp = torch.nn.Parameter(torch.tensor(p0))
    opt = torch.optim.AdamW([tp], lr=HP["lr"], betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"],
                            weight_decay=HP["weight_decay"], foreach=False)
    p, m, v = p0, np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g)
        opt.step()
        c = adamw8.constants(HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t)
        p, m, v = adamw8.step_f32(p, g, m, v, c)
    # the two differ only in rounding order (torch forms m by lerp and divides by
    # sqrt(bc2) after the root): a few fp32 ulps, far below one step's lr
    assert np.allclose(p, tp.detach().numpy(), rtol=0, atol=HP["lr"] / 4000)
    st = opt.state[tp]
    assert np.allclose(m, st["exp_avg"].numpy(), rtol=0, atol=1e-6 * np.abs(m).max())
    assert np.allclose(v, st["exp_avg_sq"].numpy(), rtol=0, atol=1e-6 * np.abs(v).max())


def test_first_step_closed_form():
    """From zero states, Adam's first update is lr * g / (|g| + eps / ...):
    about lr * sign(g) for |g| >> eps, after the decoupled decay."""
    rng = np.random.default_rng(3)
    p = rng.standard_normal(512).astype(np.float32)
    g = (rng.standard_normal(512) * 1e-2).astype(np.float32)
    z8, z32 = np.zeros(512, np.uint8), np.zeros(2, np.float32)
    p2, pb, mc, ms, vc, vs = adamw8.step(p, g, z8, z32, z8, z32, t=1, **HP)
    want = p * np.float32(1 - HP["lr"] * HP["weight_decay"]) - HP["lr"] * g / (np.abs(g) + HP["eps"])
    assert np.allclose(p2, want, rtol=0, atol=1e-7 * HP["lr"] + 1e-7)
    # the stored moments are (1 - beta1) g and (1 - beta2) g^2, 8-bit
    m_want = (1 - HP["beta1"]) * g
    v_want = (1 - HP["beta2"]) * g * g
    assert np.allclose(adamw8.dequantize(mc, ms), m_want, rtol=2.0 ** -4, atol=ms.max() * 2.0 ** -10)
    assert np.allclose(adamw8.dequantize(vc, vs), v_want, rtol=2.0 ** -4, atol=vs.max() * 2.0 ** -10)


def test_zero_gradient_only_decays():
    p = np.linspace(-1, 1, 300, dtype=np.float32)
    z8, z32 = np.zeros(300, np.uint8), np.zeros(2, np.float32)
    p2, _, mc, ms, vc, vs = adamw8.step(p, np.zeros(300, np.float32), z8, z32, z8, z32, t=4, **HP)
    assert np.array_equal(p2, p * np.float32(1 - HP["lr"] * HP["weight_decay"]))
    assert not mc.any() and not vc.any() and not ms.any() and not vs.any()


def test_eight_bit_states_track_full_precision():
    """Ten steps with 8-bit states stay close to the same steps with fp32
    states (the 8-bit error is relative to each block's largest moment)."""
    rng = np.random.default_rng(4)
    n = 1024
    p = rng.standard_normal(n).astype(np.float32) * 0.02
    pf, mf, vf = p.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    mc, vc = np.zeros(n, np.uint8), np.zeros(n, np.uint8)
    ms, vs = np.zeros(4, np.float32), np.zeros(4, np.float32)
    for t in range(1, 11):
        g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
        p, _, mc, ms, vc, vs = adamw8.step(p, g, mc, ms, vc, vs, t=t, **HP)
        c = adamw8.constants(HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t)
        pf, mf, vf = adamw8.step_f32(pf, g, mf, vf, c)
    # each step moves a weight by about lr; the 8-bit states change a step by a few per cent
    assert np.abs(p - pf).max() < 0.15 * 10 * HP["lr"]
    assert np.abs(p - pf).mean() < 0.02 * 10 * HP["lr"]
