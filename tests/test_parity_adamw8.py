"""GPU parity of the 8-bit AdamW step against the oracle's fp64 definition.

Each step starts both sides from the same state (the parameters and 8-bit
states the GPU holds), so that errors do not compound across steps.  The
kernel computes in fp32, the oracle in fp64, so the comparison is a bound
derived from the kernel's arithmetic (eps = 2^-24, the fp32 unit roundoff):

* p: the two fp32 roundings of p (1 - lr wd) and of the subtraction give at
  most 2 ulp of p; the update lr m_hat / (sqrt(v_hat) + eps) carries about
  nine roundings (moments, root, bias constants, division, product), bounded
  by 24 eps of its size; and m itself, formed as beta1 m0 + (1 - beta1) g,
  can lose relative accuracy to cancellation, so its error bound
  4 eps (|beta1 m0| + |(1 - beta1) g|) + eps |m| (plus three roundings'
  worth of fp32's smallest subnormal, for moments that underflow) passes
  through the update's factor lr / (1 - beta1^t) / (sqrt(v_hat) + eps)
  (times 2 for safety).
* the bf16 copy is the round-to-nearest-even of the kernel's own fp32 p.
* block scales: fl32(absmax / 448) on both sides; the absmaxes differ by at
  most the block's moment error bound, so the scales by that / 448 plus 2 ulp.
* codes: decoded, each within one E4M3 grid step (at that magnitude) plus
  the moment error bound of the oracle's, since both round to the nearest
  grid point moments that differ by at most that bound; and at most 1 in
  10^4 codes differ at all (a code changes only where a moment sits within a
  few fp32 ulps of a rounding boundary of the 3-bit mantissa).

Covered: ragged sizes, one LoRA pair of the training shape, and every adapter
of a 7B model (all seven linears, rank 16) in one array, with an all-zero
block and blocks of tiny values."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from oracle import adamw8
from oracle.nf4 import f32_to_bf16_bits

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
EPS32 = 2.0 ** -24
TINY32 = 2.0 ** -149      # fp32's smallest subnormal: the absolute error of a rounding near zero

# adapters of one 7B decoder layer at rank 16: q, k, v, o (4096 x 4096),
# gate, up (11008 x 4096), down (4096 x 11008): r (d_in + d_out) each
ADAPTERS_7B = 32 * (4 * 16 * (4096 + 4096) + 3 * 16 * (4096 + 11008))


def _grads(n, steps, seed):
    """Gradients whose magnitude varies by block (1e-6 .. 1e-1), with an
    all-zero block and blocks of tiny values when n allows."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(steps):
        g = rng.standard_normal(n).astype(np.float32)
        scale = np.repeat(np.exp(rng.uniform(np.log(1e-6), np.log(1e-1), (n + 255) // 256)), 256)[:n]
        g = (g * scale).astype(np.float32)
        if n > 768:
            g[256:512] = 0.0
            g[512:768] *= np.float32(1e-30)
        if n > 1024:
            g[768:1024] *= np.float32(1e-35)      # moments that underflow in fp32
        out.append(g)
    return out


def _ulp32(x):
    return np.spacing(np.abs(np.asarray(x, dtype=np.float64)).astype(np.float32)).astype(np.float64)


def _e4m3_step(y):
    """Spacing of the E4M3 grid at magnitude |y| (y in units of the scale)."""
    a = np.abs(y)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))


def _block_max(x, n):
    nb = (n + 255) // 256
    pad = np.zeros(nb * 256)
    pad[:n] = x
    return pad.reshape(nb, 256).max(axis=1)


def _check_states(codes_g, scale_g, codes_o, scale_o, err, n, what):
    nb = (n + 255) // 256
    sg = scale_g[:nb].astype(np.float64)
    so = scale_o.astype(np.float64)
    s_tol = 2 * _ulp32(so) + _block_max(err, n) / 448.0
    assert np.all(np.abs(sg - so) <= s_tol), f"{what} scales"
    dg = adamw8.dequantize(codes_g, scale_g[:nb])
    do = adamw8.dequantize(codes_o, scale_o)
    sgr, sor = np.repeat(sg, 256)[:n], np.repeat(so, 256)[:n]
    yg = np.divide(np.abs(dg), sgr, out=np.zeros(n), where=sgr > 0)
    yo = np.divide(np.abs(do), sor, out=np.zeros(n), where=sor > 0)
    tol = np.maximum(_e4m3_step(yg), _e4m3_step(yo)) * np.maximum(sgr, sor) * (1 + 2.0 ** -18) \
        + 448.0 * np.abs(sgr - sor) + err
    assert np.all(np.abs(dg - do) <= tol), f"{what} codes beyond one E4M3 step"
    differ = np.count_nonzero(codes_g != codes_o)
    assert differ <= max(2, n // 10000), f"{what}: {differ} of {n} codes differ"


def _one_step(p_host, g, mc, ms, vc, vs, t, with_bf16):
    """Runs one step on the GPU and on the oracle from the same state and
    compares them; returns the GPU's new state."""
    n = p_host.size
    nb = (n + 255) // 256
    p = torch.tensor(p_host, device="cuda")
    st = qn.AdamW8State(torch.tensor(mc, device="cuda"), torch.tensor(ms, device="cuda"),
                        torch.tensor(vc, device="cuda"), torch.tensor(vs, device="cuda"))
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda") if with_bf16 else None
    qn.adamw8_step(p, torch.tensor(g, device="cuda"), st, t, param_bf16=pb, **HP)
    torch.cuda.synchronize()
    p_g = p.cpu().numpy()
    mc_g, ms_g = st.m_codes.cpu().numpy(), st.m_scale.cpu().numpy()
    vc_g, vs_g = st.v_codes.cpu().numpy(), st.v_scale.cpu().numpy()

    p_o, m_o, v_o, mc_o, ms_o, vc_o, vs_o = adamw8.step(p_host, g, mc, ms[:nb], vc, vs[:nb], t=t, **HP)

    lr, b1, b2, eps, wd = adamw8.hyper(**HP)
    m0 = adamw8.dequantize(mc, ms[:nb])
    v0 = adamw8.dequantize(vc, vs[:nb])
    g64 = g.astype(np.float64)
    mag_m = np.abs(b1 * m0) + np.abs((1 - b1) * g64)
    err_m = 4 * EPS32 * mag_m + EPS32 * np.abs(m_o) + 3 * TINY32
    err_v = 6 * EPS32 * (np.abs(b2 * v0) + np.abs((1 - b2) * g64 * g64)) + 3 * TINY32
    ss = lr / (1 - b1 ** t)
    den = np.sqrt(v_o / (1 - b2 ** t)) + eps
    upd = ss * m_o / den
    tol_p = 2 * _ulp32(p_o) + 24 * EPS32 * np.abs(upd) + 2 * ss * err_m / den
    bad = np.abs(p_g.astype(np.float64) - p_o) > tol_p
    assert not bad.any(), f"p at step {t}: {np.count_nonzero(bad)} beyond the bound"
    if with_bf16:
        assert np.array_equal(pb.cpu().view(torch.int16).numpy().view(np.uint16), f32_to_bf16_bits(p_g))
    _check_states(mc_g, ms_g, mc_o, ms_o, err_m, n, f"m at step {t}")
    _check_states(vc_g, vs_g, vc_o, vs_o, err_v, n, f"v at step {t}")
    return p_g, mc_g, ms_g, vc_g, vs_g


def _run(n, steps=3, seed=0, with_bf16=True):
    rng = np.random.default_rng(seed + 1)
    p = (rng.standard_normal(n) * 0.02).astype(np.float32)
    nb = max((n + 255) // 256, 1)
    mc, vc = np.zeros(n, np.uint8), np.zeros(n, np.uint8)
    ms, vs = np.zeros(nb, np.float32), np.zeros(nb, np.float32)
    for t, g in enumerate(_grads(n, steps, seed), start=1):
        p, mc, ms, vc, vs = _one_step(p, g, mc, ms, vc, vs, t, with_bf16)


@pytest.mark.parametrize("n", [1, 8, 250, 1000, 4096 + 24])
def test_ragged_sizes(n):
    _run(n, steps=3, seed=n)


def test_training_shape_pair():
    """A [16, 4096] and B [4096, 16] of the training-shape layer, one array."""
    _run(2 * 16 * 4096, steps=4, seed=7)


def test_without_bf16_copy():
    _run(3000, steps=2, seed=9, with_bf16=False)


def test_hyperparameters_are_checked():
    p = torch.zeros(16, device="cuda")
    st = qn.AdamW8State.zeros(16)
    for bad in (dict(beta1=1.0), dict(beta2=-0.1), dict(eps=0.0), dict(lr=float("nan"))):
        kw = dict(HP, **bad)
        with pytest.raises(qn.QNError):
            qn.adamw8_step(p, p, st, 1, **kw)
    with pytest.raises(qn.QNError):
        qn.adamw8_step(p, p, st, 0, **HP)


def test_all_adapters_of_a_7b_model():
    """39,976,960 parameters (every linear of 32 layers at rank 16) in one
    call, as the benchmark times it: two steps, compared in full."""
    _run(ADAPTERS_7B, steps=2, seed=11)
