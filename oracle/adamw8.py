"""8-bit AdamW step on the LoRA matrices, in plain numpy, fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

[LoRA y QLoRA en Profundidad, "Optimizadores Paginados": QLoRA trains with
optim="paged_adamw_8bit", Adam with 8-bit states (paging moves the states to
CPU memory when the GPU runs short; paging is not built here).  "Cálculo de
Memoria": an 8-bit optimizer holds its states in a fraction of fp32 Adam's
8 bytes per parameter.  Módulo 4: QLoRA, 4.4: only the LoRA matrices train.]

The step is the textbook definition, written out in the order its authors
give it and evaluated in fp64:
  * Adam (Kingma and Ba) with decoupled weight decay (Loshchilov and Hutter):
        m = beta1 m0 + (1 - beta1) g          v = beta2 v0 + (1 - beta2) g^2
        m_hat = m / (1 - beta1^t)             v_hat = v / (1 - beta2^t)
        p <- p (1 - lr wd) - lr m_hat / (sqrt(v_hat) + eps)
    The hyperparameters are the fp32 values a caller passes; everything after
    that is fp64.
The pages give no format for the 8-bit states.  Readings taken:
  * both moments in blocks of 256 consecutive values (the block of the
    pages' double quantization); a block stores one fp32 scale, the block's
    absmax / 448 rounded to fp32, and per value the FP8 E4M3 code nearest
    to value / scale (ties to the even code, saturating at 448, zero stored
    as +0).  A floating 8-bit code keeps small second moments that a
    fixed-point int8 code would flush to zero (and so turn into a division
    by eps);
  * the update uses the new m and v at full precision; only then are they
    stored in 8 bits; the next step starts from the stored codes;
  * parameters are fp32 masters; the bf16 copy the layer reads is their
    bf16 rounding (nearest, ties to even).
"""

import numpy as np

BLOCK = 256
E4M3_MAX = 448.0


def e4m3_grid():
    """The 127 finite non-negative E4M3 values, in code order (code = index).

    E4M3 ("fn"): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no
    infinities, only S.1111.111 is NaN.  Exponent field 0 is subnormal:
    m / 8 * 2^-6; otherwise (1 + m / 8) * 2^(e - 7)."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            vals.append(m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


_GRID = e4m3_grid()


def e4m3_encode(x):
    """Real values (fp32 or fp64 arrays) -> E4M3 codes (uint8): the nearest
    grid value, ties to the even code, magnitudes at or past 448 saturate to
    448; a result of magnitude 0 is +0."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    hi = np.searchsorted(_GRID, a, side="left")          # first grid value >= a
    hi = np.minimum(hi, len(_GRID) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _GRID[lo]
    d_hi = _GRID[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(a >= _GRID[-1], len(_GRID) - 1, np.where(pick_hi, hi, lo))
    sign = (np.signbit(x) & (idx != 0)).astype(np.uint8) << 7
    return (idx.astype(np.uint8) | sign).astype(np.uint8)


def e4m3_decode(codes):
    """E4M3 codes (no NaN codes) -> their values (fp64, exact)."""
    c = np.asarray(codes, dtype=np.uint8)
    v = _GRID[(c & 0x7F).astype(np.int64)]
    return np.where(c & 0x80, -v, v)


def quantize(x):
    """Real values [n] -> (codes uint8 [n], scales fp32 [ceil(n / 256)]).
    Per block: scale = fl32(absmax / 448); code = E4M3 nearest to
    x / scale (the division in fp64); a block whose scale is 0 gets all-zero
    codes.  (The last block is zero padded, which changes neither its absmax
    nor its codes.)"""
    x = np.asarray(x, dtype=np.float64)
    n = x.size
    nb = (n + BLOCK - 1) // BLOCK
    blocks = np.zeros(nb * BLOCK, dtype=np.float64)
    blocks[:n] = x
    blocks = blocks.reshape(nb, BLOCK)
    absmax = np.abs(blocks).max(axis=1)
    scales = (absmax / E4M3_MAX).astype(np.float32)
    safe = np.where(scales > 0, scales, np.float32(1)).astype(np.float64)
    codes = np.where(scales[:, None] > 0, e4m3_encode(blocks / safe[:, None]), np.uint8(0))
    return codes.reshape(-1)[:n].astype(np.uint8), scales


def dequantize(codes, scales):
    """code value * block scale, exact in fp64 (a 4-bit by 24-bit product)."""
    c = np.asarray(codes, dtype=np.uint8)
    s = np.repeat(np.asarray(scales, dtype=np.float32).astype(np.float64), BLOCK)[:c.size]
    return e4m3_decode(c) * s


def hyper(lr, beta1, beta2, eps, weight_decay):
    """The hyperparameters as a caller of the fp32 interface passes them."""
    return tuple(float(np.float32(v)) for v in (lr, beta1, beta2, eps, weight_decay))


def adamw_step(p, g, m0, v0, lr, beta1, beta2, eps, weight_decay, t):
    """One AdamW step with full-precision states, fp64: returns the new
    (p, m, v).  The formulas of the module docstring, one line each."""
    p, g, m0, v0 = (np.asarray(a, dtype=np.float64) for a in (p, g, m0, v0))
    m = beta1 * m0 + (1.0 - beta1) * g
    v = beta2 * v0 + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** int(t))
    v_hat = v / (1.0 - beta2 ** int(t))
    p = p * (1.0 - lr * weight_decay) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return p, m, v


def step(p, g, m_codes, m_scales, v_codes, v_scales, lr, beta1, beta2, eps, weight_decay, t):
    """One 8-bit AdamW step: decode the stored states, step in fp64, store
    the new states in 8 bits.  Returns (p, m, v, m_codes, m_scales, v_codes,
    v_scales): p, m and v in fp64 (before any rounding to a stored format)."""
    lr, beta1, beta2, eps, weight_decay = hyper(lr, beta1, beta2, eps, weight_decay)
    m0 = dequantize(m_codes, m_scales)
    v0 = dequantize(v_codes, v_scales)
    p2, m, v = adamw_step(p, g, m0, v0, lr, beta1, beta2, eps, weight_decay, t)
    mc, ms = quantize(m)
    vc, vs = quantize(v)
    return p2, m, v, mc, ms, vc, vs
