"""Planted mistakes in the oracle (CPU only) must each fail a pin.

Every case swaps one oracle function for a plausible wrong version (a dropped
term, a wrong index, a wrong sign, the other nibble order...) and checks that
the pin written for that part raises.  This shows the pins are not vacuous.
"""

import statistics

import numpy as np
import pytest

from oracle import adamw8, dropout, linear, nf4
import test_oracle_adamw8 as ta
import test_oracle_dropout as td
import test_oracle_linear as tl
import test_oracle_nf4 as tn

# originals, captured before any monkeypatching
ORIG_LEVELS = nf4.nf4_levels_f64
ORIG_DQ = nf4.double_quant
ORIG_BWD = linear.backward_f64
ORIG_PHILOX = dropout.philox
ORIG_DROP_BWD = dropout.backward
ORIG_E4M3 = adamw8.e4m3_encode


def _levels_wrong_count():
    normal = statistics.NormalDist()
    p_pos = np.linspace(0.9677083, 0.5, 8)[:-1].tolist() + [0.55]   # 8 not 9 steps
    p_neg = np.linspace(0.9677083, 0.5, 8)[:-1]
    v = sorted([-normal.inv_cdf(p) for p in p_neg] + [0.0] + [normal.inv_cdf(p) for p in p_pos])
    return np.array([x / max(v) for x in v])


def _levels_unnormalised():
    return ORIG_LEVELS() * 1.5


def _encode_last_tie(w32, levels, chunk=8192):
    w32 = np.asarray(w32, np.float32)
    levels = np.asarray(levels, np.float32)
    absmax = np.max(np.abs(w32), axis=1).astype(np.float32)
    x = (w32 / np.where(absmax == 0, 1, absmax)[:, None]).astype(np.float32)
    d = np.abs(x[..., None] - levels)[..., ::-1]
    codes = (15 - np.argmin(d, axis=-1)).astype(np.uint8)
    return codes, absmax


def _encode_signed_max(w32, levels, chunk=8192):
    w32 = np.asarray(w32, np.float32)
    absmax = np.max(w32, axis=1).astype(np.float32)          # forgot abs
    x = (w32 / absmax[:, None]).astype(np.float32)
    codes = np.argmin(np.abs(x[..., None] - np.asarray(levels, np.float32)), -1).astype(np.uint8)
    return codes, absmax


def _pack_swapped(codes):
    c = np.asarray(codes, np.uint8)
    return (c[..., 1::2] | (c[..., 0::2] << 4)).astype(np.uint8)


def _dq_no_mean(absmax):
    s = np.asarray(absmax, np.float32)
    ng = (len(s) + 255) // 256
    q = np.zeros(len(s), np.int8)
    step = np.zeros(ng, np.float32)
    mean = np.zeros(ng, np.float32)
    for g in range(ng):
        grp = s[g * 256:(g + 1) * 256]
        st = np.float32(np.max(np.abs(grp)) / np.float32(127))
        q[g * 256:g * 256 + len(grp)] = np.clip(np.rint(grp / st), -127, 127).astype(np.int8)
        step[g] = st
    return q, step, mean


def _dq_step_128(absmax):
    q, step, mean = ORIG_DQ(absmax)
    s = np.asarray(absmax, np.float32)
    grp = np.arange(len(s)) // 256
    st = (step * np.float32(127) / np.float32(128)).astype(np.float32)
    d = (s - mean[grp]).astype(np.float32)
    q2 = np.clip(np.rint(d / np.where(st[grp] == 0, 1, st[grp])), -127, 127).astype(np.int8)
    return q2, st, mean


def _bf16_truncate(x):
    f = np.ascontiguousarray(np.asarray(x, np.float32))
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def _fwd_no_scale(x, w, a, b, s):
    y = x @ w.T
    if a is None:
        return y, None
    u = x @ a.T
    return y + (u @ b.T), u


def _bwd_wrong_sign(dy, x, w, a, b, s):
    dx, da, db = ORIG_BWD(dy, x, w, a, b, s)
    if da is None:
        return dx, da, db
    return dy @ w - s * ((dy @ b) @ a), da, db


def _bwd_transposed_db(dy, x, w, a, b, s):
    dx, da, db = ORIG_BWD(dy, x, w, a, b, s)
    if db is None:
        return dx, da, db
    return dx, da, s * (dy.T @ (x @ a.T))[:, ::-1].copy()


def _bwd_dropped_lora_dx(dy, x, w, a, b, s):
    dx, da, db = ORIG_BWD(dy, x, w, a, b, s)
    return dy @ w, da, db


def _philox_words_swapped(ctr, key, width=32, rounds=10):
    # x1 and x3 exchanged in the round's output
    mask = (1 << width) - 1
    m0, m1 = dropout.PHILOX_MULT[width]
    w0, w1 = dropout.PHILOX_WEYL[width]
    x0, x1, x2, x3 = ctr
    k0, k1 = key
    for i in range(rounds):
        if i > 0:
            k0, k1 = (k0 + w0) & mask, (k1 + w1) & mask
        p0, p1 = x0 * m0, x2 * m1
        x0, x1, x2, x3 = (p1 >> width) ^ x3 ^ k0, p1 & mask, (p0 >> width) ^ x1 ^ k1, p0 & mask
    return x0, x1, x2, x3


def _philox_nine_rounds(ctr, key, width=32, rounds=10):
    return ORIG_PHILOX(ctr, key, width, rounds - 1)


def _drop_bwd_unscaled_dx(dy, x, w, a, b, alpha, r, p, keep):
    dx, da, db = ORIG_DROP_BWD(dy, x, w, a, b, alpha, r, p, keep)
    base = nf4.bf16_bits_to_f64(dy) @ nf4.bf16_bits_to_f64(w)
    return base + (dx - base) * (1.0 - float(np.float32(p))), da, db


def _drop_bwd_da_from_x(dy, x, w, a, b, alpha, r, p, keep):
    dx, da, db = ORIG_DROP_BWD(dy, x, w, a, b, alpha, r, p, np.ones_like(keep))
    dx2, _, db2 = ORIG_DROP_BWD(dy, x, w, a, b, alpha, r, p, keep)
    return dx2, da, db2


def _pack_keep_msb_first(keep):
    m, k = keep.shape
    bits = keep.reshape(m, k // 32, 32).astype(np.uint64)
    return (bits << np.arange(31, -1, -1, dtype=np.uint64)).sum(axis=2).astype(np.uint32)


def _e4m3_ties_down(x):
    x = np.asarray(x, dtype=np.float32)
    grid = adamw8.e4m3_grid()
    a = np.abs(x).astype(np.float64)
    hi = np.minimum(np.searchsorted(grid, a, side="left"), len(grid) - 1)
    lo = np.maximum(hi - 1, 0)
    idx = np.where(grid[hi] - a < a - grid[lo], hi, lo)          # ties to the smaller magnitude
    sign = (np.signbit(x) & (idx != 0)).astype(np.uint8) << 7
    return (idx.astype(np.uint8) | sign).astype(np.uint8)


def _quantize_int8_range(x):
    x = np.asarray(x, dtype=np.float32)
    nb = (x.size + 255) // 256
    codes = np.zeros(x.size, np.uint8)
    scales = np.zeros(nb, np.float32)
    for b in range(nb):
        blk = x[256 * b:256 * (b + 1)]
        s = np.float32(np.abs(blk).max() / np.float32(127))      # int8's range, not E4M3's
        scales[b] = s
        if s > 0:
            codes[256 * b:256 * (b + 1)] = ORIG_E4M3(blk * np.float32(127 / np.abs(blk).max()))
    return codes, scales


def _step_no_bias_correction(p, g, m0, v0, lr, beta1, beta2, eps, weight_decay, t):
    p, g, m0, v0 = (np.asarray(x, dtype=np.float64) for x in (p, g, m0, v0))
    m = beta1 * m0 + (1.0 - beta1) * g
    v = beta2 * v0 + (1.0 - beta2) * g * g
    return p * (1.0 - lr * weight_decay) - lr * m / (np.sqrt(v) + eps), m, v


def _step_coupled_decay(p, g, m0, v0, lr, beta1, beta2, eps, weight_decay, t):
    # L2 regularisation folded into the gradient instead of a decoupled decay
    g = np.asarray(g, np.float64) + weight_decay * np.asarray(p, np.float64)
    return ORIG_ADAMW_STEP(p, g, m0, v0, lr, beta1, beta2, eps, 0.0, t)


def _step_eps_inside_root(p, g, m0, v0, lr, beta1, beta2, eps, weight_decay, t):
    p, g, m0, v0 = (np.asarray(x, dtype=np.float64) for x in (p, g, m0, v0))
    m = beta1 * m0 + (1.0 - beta1) * g
    v = beta2 * v0 + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** int(t))
    v_hat = v / (1.0 - beta2 ** int(t))
    return p * (1.0 - lr * weight_decay) - lr * m_hat / np.sqrt(v_hat + eps), m, v


ORIG_ADAMW_STEP = adamw8.adamw_step

MUTANTS = [
    ("levels: 8 positive steps", nf4, "nf4_levels_f64", _levels_wrong_count,
     [tn.test_levels_are_normal_quantiles]),
    ("levels: not divided by the max", nf4, "nf4_levels_f64", _levels_unnormalised,
     [tn.test_levels_invariants]),
    ("encode: ties to the higher index", nf4, "encode_blocks", _encode_last_tie,
     [tn.test_encode_tie_goes_to_lower_index]),
    ("encode: max without abs", nf4, "encode_blocks", _encode_signed_max,
     [tn.test_dequantize_error_bound]),
    ("pack: nibbles swapped", nf4, "pack_codes", _pack_swapped,
     [tn.test_pack_nibble_order]),
    ("double quant: no mean", nf4, "double_quant", _dq_no_mean,
     [tn.test_double_quant_error_bound_and_range]),
    ("double quant: step max/128", nf4, "double_quant", _dq_step_128,
     [tn.test_double_quant_error_bound_and_range]),
    ("bf16: truncation", nf4, "f32_to_bf16_bits", _bf16_truncate,
     [tn.test_bf16_rounding_matches_torch]),
    ("forward: alpha/r dropped", linear, "forward_f64", _fwd_no_scale,
     [lambda: tl.test_gradients_match_finite_differences("a")]),
    ("backward: LoRA dx sign", linear, "backward_f64", _bwd_wrong_sign,
     [lambda: tl.test_gradients_match_finite_differences("x")]),
    ("backward: dB transposed", linear, "backward_f64", _bwd_transposed_db,
     [lambda: tl.test_gradients_match_finite_differences("b")]),
    ("backward: LoRA term of dx dropped", linear, "backward_f64", _bwd_dropped_lora_dx,
     [tl.test_backward_brute_force_loops]),
    ("philox: round words exchanged", dropout, "philox", _philox_words_swapped,
     [lambda: td.test_philox4x32_known_answers(*td.KAT_4X32_10[2])]),
    ("philox: nine rounds", dropout, "philox", _philox_nine_rounds,
     [lambda: td.test_philox4x32_known_answers(*td.KAT_4X32_10[0]),
      td.test_philox_rounds_match_numpy_philox4x64]),
    ("dropout: dx without 1/(1-p)", dropout, "backward", _drop_bwd_unscaled_dx,
     [td.test_backward_matches_autograd]),
    ("dropout: dA from x, not dropout(x)", dropout, "backward", _drop_bwd_da_from_x,
     [td.test_backward_matches_autograd]),
    ("dropout: mask bits MSB first", dropout, "pack_keep", _pack_keep_msb_first,
     [td.test_pack_keep_bit_order]),
    ("adamw8: E4M3 ties to the smaller value", adamw8, "e4m3_encode", _e4m3_ties_down,
     [ta.test_encode_matches_torch_rounding]),
    ("adamw8: block scale absmax/127", adamw8, "quantize", _quantize_int8_range,
     [ta.test_quantize_error_bound_and_ragged_blocks]),
    ("adamw8: no bias correction", adamw8, "adamw_step", _step_no_bias_correction,
     [ta.test_full_precision_steps_match_torch_adamw, ta.test_first_step_closed_form]),
    ("adamw8: decay coupled into the gradient", adamw8, "adamw_step", _step_coupled_decay,
     [ta.test_full_precision_steps_match_torch_adamw]),
    ("adamw8: eps inside the root", adamw8, "adamw_step", _step_eps_inside_root,
     [ta.test_full_precision_steps_match_torch_adamw]),
]


@pytest.mark.parametrize("label,mod,name,mutant,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, label, mod, name, mutant, pins):
    monkeypatch.setattr(mod, name, mutant)
    if name == "nf4_levels_f64":
        monkeypatch.setattr(nf4, "nf4_levels", lambda: mutant().astype(np.float32))
    for pin in pins:
        with pytest.raises(AssertionError):
            pin()
