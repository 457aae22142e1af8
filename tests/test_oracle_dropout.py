"""Pins of the LoRA dropout oracle (CPU).

[LoRA y QLoRA en Profundidad, "Dropout (lora_dropout)"]: the LoRA layers'
dropout zeroes randomly chosen elements during training.  The random draw is
Philox4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3",
SC 2011); it is pinned by the generator's published known-answer vectors and,
for the round structure, by numpy's own Philox4x64-10.  The gradients are
pinned by autograd, the p = 0 case by the plain linear.
"""

import math

import numpy as np
import pytest
import torch

from bit_nf4_quantized_28_b200 import workloads as wl
from oracle import dropout, linear, nf4


# Known-answer vectors of Philox4x32-10 (counter, key) -> output, as published
# with the reference implementation of the SC 2011 paper (Random123).
KAT_4X32_10 = [
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("ctr,key,want", KAT_4X32_10)
def test_philox4x32_known_answers(ctr, key, want):
    assert tuple(dropout.philox(ctr, key, 32)) == want
    # the vectorized form (numpy uint64 words) gives the same words
    got = dropout.philox(tuple(np.array([c], dtype=np.uint64) for c in ctr), key, 32)
    assert tuple(int(w[0]) for w in got) == want


def test_philox_rounds_match_numpy_philox4x64():
    """The same routine at 64-bit words against numpy.random.Philox (4x64-10),
    which advances its counter by one before each block of four words."""
    key = (0x0123456789ABCDEF, 0x0F1E2D3C4B5A6978)
    start = 41
    bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array([start, 0, 0, 0], dtype=np.uint64))
    raw = [int(v) for v in bg.random_raw(12)]
    mine = []
    for c in range(start + 1, start + 4):
        mine.extend(dropout.philox((c, 0, 0, 0), key, 64))
    assert mine == raw


def test_threshold():
    assert dropout.threshold(0.0) == 0
    assert dropout.threshold(0.5) == 2 ** 31
    assert dropout.threshold(0.25) == 2 ** 30
    assert dropout.threshold(0.05) == math.floor(float(np.float32(0.05)) * 2 ** 32)
    for bad in (1.0, -0.1, 1.5):
        with pytest.raises(ValueError):
            dropout.threshold(bad)


def test_element_to_counter_mapping():
    """Element e takes word e % 4 of the block with counter e // 4 (scalar
    Python-int Philox, independent of the vectorized path)."""
    m, k, seed, offset = 2, 32, 0x1122334455667788, 0x99AABBCCDDEEFF00
    words = dropout.random_words(m * k, seed, offset)
    for e in range(m * k):
        q = e // 4
        blk = dropout.philox((q & 0xFFFFFFFF, q >> 32, offset & 0xFFFFFFFF, offset >> 32),
                             (seed & 0xFFFFFFFF, seed >> 32), 32)
        assert int(words[e]) == blk[e % 4]
    t = dropout.threshold(0.3)
    keep = dropout.keep_mask(m, k, 0.3, seed, offset)
    assert np.array_equal(keep.reshape(-1), words >= t)


def test_keep_rate_and_p_zero():
    m, k = 256, 4096
    for p in (0.05, 0.1):
        keep = dropout.keep_mask(m, k, p, seed=7, offset=3)
        n = keep.size
        drop = 1.0 - keep.mean()
        sigma = math.sqrt(p * (1 - p) / n)
        assert abs(drop - p) < 5 * sigma, (p, drop)
        # rows and columns carry no structure: per-row drop rates spread like a binomial
        row_rates = 1.0 - keep.mean(axis=1)
        assert abs(row_rates.std() - math.sqrt(p * (1 - p) / k)) < 0.25 * math.sqrt(p * (1 - p) / k)
    assert dropout.keep_mask(16, 64, 0.0, seed=7, offset=3).all()


def test_seed_and_offset_select_independent_masks():
    a = dropout.keep_mask(64, 256, 0.5, seed=1, offset=0)
    b = dropout.keep_mask(64, 256, 0.5, seed=2, offset=0)
    c = dropout.keep_mask(64, 256, 0.5, seed=1, offset=1)
    assert np.array_equal(a, dropout.keep_mask(64, 256, 0.5, seed=1, offset=0))
    for other in (b, c):
        agree = (a == other).mean()
        assert 0.45 < agree < 0.55


def test_pack_keep_bit_order():
    keep = np.zeros((2, 64), dtype=bool)
    keep[0, 0] = keep[0, 31] = keep[0, 32] = True
    keep[1, 63] = True
    words = dropout.pack_keep(keep)
    assert words.dtype == np.uint32 and words.shape == (2, 2)
    assert words.tolist() == [[0x80000001, 0x00000001], [0, 0x80000000]]


def test_apply_bits():
    x = np.array([[0x3F80, 0x8000, 0xC040, 0x0001]], dtype=np.uint16)   # 1, -0, -3, tiny
    keep = np.array([[True, True, False, False]])
    assert dropout.apply_bits(x, keep).tolist() == [[0x3F80, 0x8000, 0, 0]]


def _layer(seed=11, m=6, k=64, n=32, r=8):
    t = wl.make_linear(seed, n, k, m, r, 16.0, a_std=0.1, b_std=0.1, w_std=0.1)
    return wl.bits(t.x), wl.bits(t.W), wl.bits(t.A), wl.bits(t.B), wl.bits(t.dy), t


def test_p_zero_is_the_plain_linear():
    x, w, a, b, dy, t = _layer()
    keep = np.ones(x.shape, dtype=bool)
    y, u = dropout.forward(x, w, a, b, t.alpha, t.r, 0.0, keep)
    y0, u0 = linear.forward(x, w, a, b, t.alpha, t.r)
    assert np.array_equal(y, y0) and np.array_equal(u, u0)
    g = dropout.backward(dy, x, w, a, b, t.alpha, t.r, 0.0, keep)
    g0 = linear.backward(dy, x, w, a, b, t.alpha, t.r)
    for p_, q_ in zip(g, g0):
        assert np.allclose(p_, q_, rtol=1e-14, atol=1e-14)


def test_all_kept_scales_the_lora_path():
    """Nothing dropped: the LoRA path is scaled by 1 / (1 - p)."""
    x, w, a, b, dy, t = _layer()
    p = 0.1
    keep = np.ones(x.shape, dtype=bool)
    y, _ = dropout.forward(x, w, a, b, t.alpha, t.r, p, keep)
    s = linear.lora_scale(t.alpha, t.r) / (1.0 - float(np.float32(p)))
    y_ref, _ = linear.forward_f64(nf4.bf16_bits_to_f64(x), nf4.bf16_bits_to_f64(w), nf4.bf16_bits_to_f64(a),
                                  nf4.bf16_bits_to_f64(b), s)
    assert np.allclose(y, y_ref, rtol=1e-13, atol=1e-13)


def test_backward_matches_autograd():
    """dx, dA, dB against torch autograd (fp64, CPU) of <dy, y> with the mask fixed."""
    x, w, a, b, dy, t = _layer()
    p = 0.25
    keep = dropout.keep_mask(x.shape[0], x.shape[1], p, seed=5, offset=9)
    assert 0 < keep.sum() < keep.size
    s = linear.lora_scale(t.alpha, t.r)
    f = lambda bits: torch.tensor(nf4.bf16_bits_to_f64(bits), dtype=torch.float64)
    X = f(x).requires_grad_()
    A = f(a).requires_grad_()
    B = f(b).requires_grad_()
    W, DY = f(w), f(dy)
    K = torch.tensor(keep, dtype=torch.float64)
    y = X @ W.T + s * (torch.nn.functional.linear(X * K / (1 - float(np.float32(p))), A) @ B.T)
    (y * DY).sum().backward()
    dx, da, db = dropout.backward(dy, x, w, a, b, t.alpha, t.r, p, keep)
    y_o, _ = dropout.forward(x, w, a, b, t.alpha, t.r, p, keep)
    assert np.allclose(y_o, y.detach().numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dx, X.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(da, A.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(db, B.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_dropped_inputs_do_not_reach_the_lora_path():
    """A column of x dropped in every row changes neither u nor dA's column."""
    x, w, a, b, dy, t = _layer()
    keep = np.ones(x.shape, dtype=bool)
    keep[:, 5] = False
    x2 = x.copy()
    x2[:, 5] = 0x4500   # a different value in the dropped column
    _, u1 = dropout.forward(x, w, a, b, t.alpha, t.r, 0.05, keep)
    _, u2 = dropout.forward(x2, w, a, b, t.alpha, t.r, 0.05, keep)
    assert np.array_equal(u1, u2)
    _, da, _ = dropout.backward(dy, x, w, a, b, t.alpha, t.r, 0.05, keep)
    assert np.all(da[:, 5] == 0)
