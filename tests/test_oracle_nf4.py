"""Pins of the oracle's NF4 storage against what the pages and mathematics fix.

No GPU.  Each test checks the oracle against something other than itself: the
values the NF4 snippet prints, closed forms, the normal CDF evaluated through
math.erf (independent of the inverse routine the oracle uses), exact-arithmetic
nearest-level optimality, torch's own bf16 rounding, and invariants.
"""

import math

import numpy as np
import pytest
import torch

from oracle import nf4
from bit_nf4_quantized_28_b200 import workloads as wl


def phi(x):
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def phi_inverse_bisect(p):
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


# ------------------------------------------------------------------ level table

def test_levels_invariants():
    lv = nf4.nf4_levels()
    assert lv.dtype == np.float32 and lv.shape == (16,)
    assert np.all(np.diff(lv) > 0), "strictly sorted"
    assert lv[0] == -1.0 and lv[15] == 1.0
    assert np.count_nonzero(lv == 0.0) == 1 and lv[7] == 0.0
    assert np.count_nonzero(lv < 0) == 7 and np.count_nonzero(lv > 0) == 8
    assert np.all(np.abs(lv) <= 1.0)


def test_levels_are_normal_quantiles():
    """Each unnormalised level sits at its stated probability under the normal
    CDF (checked with erf; the scale is found by bisection on erf)."""
    top = phi_inverse_bisect(0.9677083)
    lv = nf4.nf4_levels_f64()
    p_pos = np.linspace(0.9677083, 0.5, 9)[:-1]
    p_neg = np.linspace(0.9677083, 0.5, 8)[:-1]
    pos = lv[8:][::-1]            # largest first, matching p_pos order
    neg = -lv[:7]                 # |negative| largest first, matching p_neg
    for v, p in zip(pos, p_pos):
        assert abs(phi(v * top) - p) < 1e-12
    for v, p in zip(neg, p_neg):
        assert abs(phi(v * top) - p) < 1e-12


def test_levels_fp32_is_rounded_fp64():
    assert np.array_equal(nf4.nf4_levels(), nf4.nf4_levels_f64().astype(np.float32))


def test_int4_levels_evenly_spaced():
    lv = nf4.int4_levels().astype(np.float64)
    assert lv[0] == -1 and lv[-1] == 1 and len(lv) == 16
    assert np.allclose(np.diff(lv), 2.0 / 15, atol=1e-7)
    assert not np.any(lv == 0.0), "evenly spaced 16 levels have no exact zero"


# ------------------------------------------------------------------ worked example

def test_snippet_printed_errors(golden):
    """The NF4 snippet prints 3.395e-06 (NF4) and 4.053e-06 (evenly spaced)."""
    g = golden("snippet_mse.txt")
    w = wl.snippet_weights().numpy()
    e_nf4 = nf4.blockwise_mse(w, nf4.nf4_levels())
    e_int4 = nf4.blockwise_mse(w, nf4.int4_levels())
    assert f"{e_nf4:.3e}" == g["nf4"]
    assert f"{e_int4:.3e}" == g["int4"]
    assert round(100 * (1 - e_nf4 / e_int4)) == int(g["lower_percent"])


# ------------------------------------------------------------------ encode

def _random_blocks(seed, nb=512):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(nb, 64, generator=g) * 0.02
    w[::7, ::5] *= 20.0                                   # outliers
    return w.to(torch.bfloat16).float().numpy()


def test_encode_is_nearest_level_in_exact_arithmetic():
    """|w/a - L[c]| is minimal over all 16 levels, with the quotient in fp64
    (far more precise than the fp32 decision); slack covers fp32 rounding."""
    w = _random_blocks(11)
    lv = nf4.nf4_levels().astype(np.float64)
    codes, absmax = nf4.encode_blocks(w, nf4.nf4_levels())
    x = w.astype(np.float64) / absmax.astype(np.float64)[:, None]
    d = np.abs(x[..., None] - lv)
    chosen = np.take_along_axis(d, codes[..., None].astype(np.int64), -1)[..., 0]
    assert np.all(chosen <= d.min(-1) + 2e-7)


def test_encode_brute_force_tiny():
    """Every code checked against every level by loops on a tiny input: the
    chosen level is no farther than any other (fp32 distances), and on an
    exact tie the lower index wins."""
    w = _random_blocks(5, nb=4)
    lv = [float(v) for v in nf4.nf4_levels()]
    codes, absmax = nf4.encode_blocks(w, nf4.nf4_levels())
    for b in range(w.shape[0]):
        for i in range(64):
            x = np.float32(w[b, i]) / np.float32(absmax[b])
            ds = [abs(np.float32(x) - np.float32(l)) for l in lv]
            c = int(codes[b, i])
            assert all(ds[c] <= dj for dj in ds)
            assert all(ds[j] > ds[c] for j in range(c))


def test_encode_round_trip_levels_and_extremes():
    lv = nf4.nf4_levels()
    # a block holding every level exactly (absmax = 1) encodes to its indices
    blk = np.tile(lv, 4)[None, :].astype(np.float32)
    codes, absmax = nf4.encode_blocks(blk, lv)
    assert absmax[0] == 1.0
    assert np.array_equal(codes[0], np.tile(np.arange(16), 4))
    # +absmax -> 15, -absmax -> 0, 0 -> 7
    blk = np.zeros((1, 64), np.float32)
    blk[0, 0], blk[0, 1] = 0.5, -0.5
    codes, absmax = nf4.encode_blocks(blk, lv)
    assert codes[0, 0] == 15 and codes[0, 1] == 0 and np.all(codes[0, 2:] == 7)


def test_encode_zero_block():
    codes, absmax = nf4.encode_blocks(np.zeros((3, 64), np.float32), nf4.nf4_levels())
    assert np.all(absmax == 0) and np.all(codes == 7)


def test_encode_tie_goes_to_lower_index():
    """x exactly halfway between two levels (in fp32) takes the lower index.
    With absmax 1 and levels -1 and L[1], the midpoint is representable."""
    lv = nf4.nf4_levels()
    # search for a float32 x whose fp32 distances to L[i] and L[i+1] are equal
    found = 0
    for i in range(15):
        mid = np.float32((np.float64(lv[i]) + np.float64(lv[i + 1])) / 2)
        for cand in (mid, np.nextafter(mid, np.float32(2)), np.nextafter(mid, np.float32(-2))):
            d0 = abs(np.float32(cand - lv[i]))
            d1 = abs(np.float32(cand - lv[i + 1]))
            if d0 == d1:
                blk = np.zeros((1, 64), np.float32)
                blk[0, 0] = 1.0
                blk[0, 1] = cand
                codes, _ = nf4.encode_blocks(blk, lv)
                assert codes[0, 1] == i
                found += 1
    assert found > 0


# ------------------------------------------------------------------ packing

def test_pack_nibble_order():
    codes = np.array([[1, 2, 3, 4, 15, 0]], np.uint8)
    assert nf4.pack_codes(codes).tolist() == [[0x21, 0x43, 0x0F]]
    assert np.array_equal(nf4.unpack_codes(nf4.pack_codes(codes)), codes)


# ------------------------------------------------------------------ bf16 rounding

def test_bf16_rounding_matches_torch():
    g = torch.Generator().manual_seed(3)
    f = torch.randn(100000, generator=g) * torch.logspace(-30, 30, 100000)
    f[:16] = torch.tensor([0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.0e38, -3.0e38,
                           1e-40, -1e-40, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 65504.0, 2**-126,
                           1.0 + 2**-8 + 2**-20, 0.5])
    ours = nf4.f32_to_bf16_bits(f.numpy())
    ref = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(nf4.bf16_bits_to_f32(ref), f.to(torch.bfloat16).float().numpy())


# ------------------------------------------------------------------ double quant

def test_double_quant_bits_per_param(golden):
    g = golden("double_quant_bits.txt")
    # fp32 scale per block of 64, no second level
    assert 32 / 64 == float(g["overhead_without_dq_bits"])
    # int8 per block plus one fp32 constant per 256 blocks, as the page counts it
    closed = nf4.storage_bits_per_param(4096, 4096, with_mean=False)
    assert closed == 8 / 64 + 32 / (64 * 256)
    assert round(closed, 3) == float(g["overhead_with_dq_bits"])
    # as built: a second fp32 constant (the group mean) per 256 blocks
    assert nf4.storage_bits_per_param(4096, 4096) == 8 / 64 + 64 / (64 * 256)
    saving_65b_gb = 65e9 * (0.5 - closed) / 8 / 1e9
    assert round(saving_65b_gb) == int(g["saving_65b_gb"])
    assert abs((0.5 - closed) - float(g["saving_bits_module4"])) < 0.01


def test_double_quant_error_bound_and_range():
    w = wl.quant_weight(256, 4096, seed=9)
    q = nf4.quantize(wl.bits(w), 256, 4096)
    s = q["absmax"]
    shat = nf4.restore_scales(q["qscale"], q["step"], q["mean"])
    grp = np.arange(s.shape[0]) // nf4.DQ_GROUP
    step = q["step"][grp].astype(np.float64)
    err = np.abs(shat.astype(np.float64) - s.astype(np.float64))
    assert np.all(err <= step / 2 + 4 * np.spacing(np.abs(s).astype(np.float32)).astype(np.float64) + 1e-12)
    assert q["qscale"].min() >= -127 and q["qscale"].max() <= 127
    # in every group the scale farthest from the mean codes to +-127
    for g_ in range(q["step"].shape[0]):
        sl = slice(g_ * 256, (g_ + 1) * 256)
        d = np.abs(s[sl].astype(np.float64) - q["mean"][g_])
        assert abs(int(q["qscale"][sl][np.argmax(d)])) == 127
    # the stored mean is the group mean
    for g_ in range(q["step"].shape[0]):
        sl = slice(g_ * 256, (g_ + 1) * 256)
        assert abs(q["mean"][g_] - s[sl].astype(np.float64).mean()) <= 1e-7 * abs(q["mean"][g_])


def test_double_quant_constant_group_and_tail():
    s = np.full(300, 0.03125, np.float32)     # one full group and a tail of 44
    q, step, mean = nf4.double_quant(s)
    assert step.shape == (2,) and np.all(step == 0) and np.all(q == 0)
    assert np.array_equal(nf4.restore_scales(q, step, mean), s)


# ------------------------------------------------------------------ whole weight

def test_dequantize_error_bound():
    """|W_hat - W| <= (half the widest level gap) * s_hat + scale error + bf16
    rounding: the restore is the level times the block scale."""
    w = wl.quant_weight(128, 1024, seed=4)
    wb = wl.bits(w)
    q = nf4.quantize(wb, 128, 1024)
    wh = nf4.bf16_bits_to_f32(nf4.dequantize(q["codes"], q["qscale"], q["step"], q["mean"], 128, 1024))
    w32 = nf4.bf16_bits_to_f32(wb).reshape(-1, 64).astype(np.float64)
    shat = nf4.restore_scales(q["qscale"], q["step"], q["mean"]).astype(np.float64)
    s = q["absmax"].astype(np.float64)
    gap = np.max(np.diff(nf4.nf4_levels().astype(np.float64))) / 2
    bound = gap * shat[:, None] + np.abs(shat - s)[:, None] + np.abs(wh.reshape(-1, 64)) * 2**-8 + 1e-12
    assert np.all(np.abs(wh.reshape(-1, 64) - w32) <= bound)


def test_dequantize_exact_levels_single_group():
    """A weight whose 64-blocks all have absmax 1 and hold bf16-exact levels:
    the scales are all 1 (step 0), so W_hat is bf16(level) exactly."""
    lv = nf4.nf4_levels()
    lvb = torch.from_numpy(lv).to(torch.bfloat16)
    row = lvb.repeat(8)                               # 128 values, two blocks
    w = row.repeat(4, 1)                              # [4, 128]
    wb = wl.bits(w)
    q = nf4.quantize(wb, 4, 128)
    assert np.all(q["step"] == 0) and np.all(q["mean"] == 1.0)
    wh = nf4.dequantize(q["codes"], q["qscale"], q["step"], q["mean"], 4, 128)
    assert np.array_equal(wh, wb)


def test_quantize_shapes():
    w = wl.quant_weight(64, 256, seed=2)
    q = nf4.quantize(wl.bits(w), 64, 256)
    assert q["codes"].shape == (64, 128) and q["codes"].dtype == np.uint8
    assert q["qscale"].shape == (256,) and q["qscale"].dtype == np.int8
    assert q["step"].shape == (1,) and q["mean"].shape == (1,)


def test_outliers_mse_below_int4():
    """On N(0, 0.02) weights with 1 % x20 outliers, NF4 error stays below the
    evenly spaced table's, as the snippet shows for plain normal blocks."""
    w = wl.quant_weight(256, 4096, seed=1).float().numpy().reshape(-1, 64)
    assert nf4.blockwise_mse(w, nf4.nf4_levels()) < nf4.blockwise_mse(w, nf4.int4_levels())


@pytest.mark.parametrize("shape", [(64, 64), (3, 192), (257, 64)])
def test_quantize_dequantize_roundtrip_shapes(shape):
    n, k = shape
    g = torch.Generator().manual_seed(n * k)
    w = (torch.randn(n, k, generator=g) * 0.02).to(torch.bfloat16)
    q = nf4.quantize(wl.bits(w), n, k)
    wh = nf4.dequantize(q["codes"], q["qscale"], q["step"], q["mean"], n, k)
    assert wh.shape == (n, k)
    rel = np.abs(nf4.bf16_bits_to_f32(wh) - w.float().numpy()).max() / np.abs(w.float().numpy()).max()
    assert rel < 0.2
