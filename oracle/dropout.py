"""LoRA dropout on the LoRA path's input, forward and backward, in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

[LoRA y QLoRA en Profundidad, "Dropout (lora_dropout)"]: during training the
LoRA layers' dropout sets randomly chosen elements to zero as regularisation
(rates 0, 0.05 -- the default of the lesson's config -- or 0.1).  The LoRA
path of the frozen linear (see `linear`) then reads dropout(x) instead of x:

    y  = x W_hat^T + s (dropout(x) A^T) B^T,   s = fl32(alpha / r)
    dropout(x) = x * keep / (1 - p)

Readings taken where the pages are silent:
  * Inverted dropout: kept elements are scaled by 1 / (1 - p) so that the
    expectation is x, and only the LoRA path sees the dropout (the base path
    reads x itself), as the lesson's "capas LoRA" says.
  * The random draw is Philox4x32-10 (Salmon, Moraes, Dror and Shaw,
    "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011), a counter-based
    generator, so that the backward can redraw or re-read the same mask.
    Element e = i * k + j of x [m, k] takes word e % 4 of
    Philox(counter = (lo32(e // 4), hi32(e // 4), lo32(offset), hi32(offset)),
           key = (lo32(seed), hi32(seed))),
    and is kept iff that word >= floor(p * 2^32) (p the fp32 rate), so the
    drop probability is p to within 2^-32.
  * The keep mask is stored one bit per element: bit (j % 32) of word
    i * (k / 32) + j // 32, row-major.

The backward of <dy, y> with the mask fixed:
    dx = dy W_hat + s / (1 - p) * keep * ((dy B) A)
    dA = s (dy B)^T dropout(x)
    dB = s dy^T (dropout(x) A^T)
"""

import math

import numpy as np

from .linear import lora_scale
from .nf4 import bf16_bits_to_f64

# Philox constants of the SC 2011 paper: round multipliers and key increments
# (the Weyl sequence), for 32- and 64-bit words.
PHILOX_MULT = {32: (0xD2511F53, 0xCD9E8D57), 64: (0xD2E7470EE14C6C93, 0xCA5A826395121157)}
PHILOX_WEYL = {32: (0x9E3779B9, 0xBB67AE85), 64: (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)}


def philox(ctr, key, width=32, rounds=10):
    """Philox4xW-rounds of the SC 2011 paper on a 4-word counter and a 2-word key.

    Each round multiplies words 0 and 2 by the round multipliers, keeping
    both halves of the double-width products; the new words are
    (hi(M1 x2) ^ x1 ^ k0, lo(M1 x2), hi(M0 x0) ^ x3 ^ k1, lo(M0 x0)); the key
    advances by the Weyl increments between rounds.  Words may be Python
    ints or, for width 32, numpy uint64 arrays (products < 2^64 are exact).
    """
    mask = (1 << width) - 1
    m0, m1 = PHILOX_MULT[width]
    w0, w1 = PHILOX_WEYL[width]
    x0, x1, x2, x3 = ctr
    k0, k1 = key
    for i in range(rounds):
        if i > 0:
            k0 = (k0 + w0) & mask
            k1 = (k1 + w1) & mask
        p0 = x0 * m0
        p1 = x2 * m1
        x0, x1, x2, x3 = (p1 >> width) ^ x1 ^ k0, p1 & mask, (p0 >> width) ^ x3 ^ k1, p0 & mask
    return x0, x1, x2, x3


def threshold(p):
    """floor(p * 2^32) for the fp32 rate p in [0, 1): a word below it drops."""
    p32 = float(np.float32(p))
    if not 0.0 <= p32 < 1.0:
        raise ValueError("dropout rate must be in [0, 1)")
    return int(math.floor(p32 * 2.0 ** 32))


def random_words(count, seed, offset):
    """The 32-bit words of elements 0 .. count-1 (count % 4 == 0)."""
    assert count % 4 == 0
    m32 = 0xFFFFFFFF
    q = np.arange(count // 4, dtype=np.uint64)
    seed, offset = int(seed), int(offset)
    words = philox((q & np.uint64(m32), q >> np.uint64(32), offset & m32, offset >> 32),
                   (seed & m32, seed >> 32))
    return np.stack([np.asarray(w, dtype=np.uint64) for w in words], axis=1).reshape(-1)


def keep_mask(m, k, p, seed, offset):
    """bool [m, k]: which elements of x [m, k] the dropout keeps."""
    return (random_words(m * k, seed, offset) >= threshold(p)).reshape(m, k)


def pack_keep(keep):
    """bool [m, k] -> uint32 [m, k / 32], bit j % 32 of word j // 32 of a row."""
    m, k = keep.shape
    assert k % 32 == 0
    bits = keep.reshape(m, k // 32, 32).astype(np.uint64)
    return (bits << np.arange(32, dtype=np.uint64)).sum(axis=2).astype(np.uint32)


def apply_bits(x_bits, keep):
    """x * keep as bf16 bit patterns (dropped elements are +0)."""
    return np.where(keep, x_bits, np.uint16(0)).astype(np.uint16)


def dropout_f64(x, keep, p):
    """dropout(x) = x * keep / (1 - p) on fp64 values (p the fp32 rate)."""
    return x * keep / (1.0 - float(np.float32(p)))


def forward(x_bits, w_hat_bits, a_bits, b_bits, alpha, r, p, keep):
    """y = x W_hat^T + s (dropout(x) A^T) B^T; returns (y, u) with
    u = dropout(x) A^T, both fp64.  r > 0."""
    x = bf16_bits_to_f64(x_bits)
    w = bf16_bits_to_f64(w_hat_bits)
    a = bf16_bits_to_f64(a_bits)
    b = bf16_bits_to_f64(b_bits)
    s = lora_scale(alpha, r)
    u = dropout_f64(x, keep, p) @ a.T
    return x @ w.T + s * (u @ b.T), u


def backward(dy_bits, x_bits, w_hat_bits, a_bits, b_bits, alpha, r, p, keep):
    """(dx, dA, dB) of <dy, y> for the forward above, fp64, mask fixed."""
    dy = bf16_bits_to_f64(dy_bits)
    x = bf16_bits_to_f64(x_bits)
    w = bf16_bits_to_f64(w_hat_bits)
    a = bf16_bits_to_f64(a_bits)
    b = bf16_bits_to_f64(b_bits)
    s = lora_scale(alpha, r)
    xd = dropout_f64(x, keep, p)
    v = dy @ b
    dx = dy @ w + (s / (1.0 - float(np.float32(p)))) * (keep * (v @ a))
    return dx, s * (v.T @ xd), s * (dy.T @ (xd @ a.T))
