"""8-bit AdamW step on the LoRA matrices, in plain numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring).

[LoRA y QLoRA en Profundidad, "Optimizadores Paginados": QLoRA trains with
optim="paged_adamw_8bit", Adam with 8-bit states (paging moves the states to
CPU memory when the GPU runs short; paging is not built here).  "Cálculo de
Memoria": an 8-bit optimizer holds its states in a fraction of fp32 Adam's
8 bytes per parameter.  Módulo 4: QLoRA, 4.4: only the LoRA matrices train.]

The pages give no format for the 8-bit states.  Readings taken:
  * AdamW: Adam (Kingma and Ba) with decoupled weight decay (Loshchilov and
    Hutter): p <- p (1 - lr wd), then p <- p - lr m_hat / (sqrt(v_hat) + eps)
    with m_hat = m / (1 - beta1^t), v_hat = v / (1 - beta2^t), evaluated as
    p - (lr / (1 - beta1^t)) m / (sqrt(v) / sqrt(1 - beta2^t) + eps), the
    bias corrections folded into two per-step constants; the update uses the
    new m and v at full fp32 precision, and only then are they stored in 8
    bits.
  * 8-bit states: both moments in blocks of 256 consecutive values (the
    block of the pages' double quantization), each block with one fp32 scale
    = absmax / 448 and one 8-bit FP8 E4M3 code per value (x * (448 / absmax)
    rounded to nearest, ties to even; zero stored as +0).  A floating 8-bit code
    keeps small second moments that a fixed-point int8 code would flush to
    zero (and so turn into a division by eps).
  * Parameters: fp32 master copies; the bf16 copy the layer reads is
    written by the same step (bf16 round to nearest even).
  * Arithmetic: fp32, one IEEE operation at a time in the order written in
    `step_f32` and `quantize`; the host-side constants (1 - beta, the two
    bias-correction factors, the decay factor) are computed in fp64 and
    rounded once to fp32.
"""

import numpy as np

from .nf4 import f32_to_bf16_bits

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
    """fp32 values with |x| <= 448 (a hair above rounds to 448) -> E4M3 codes
    (uint8), round to nearest, ties to the even code; a result of magnitude 0
    is +0."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
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
    """E4M3 codes (no NaN codes) -> fp32 values (exact)."""
    c = np.asarray(codes, dtype=np.uint8)
    v = _GRID[(c & 0x7F).astype(np.int64)]
    return np.where(c & 0x80, -v, v).astype(np.float32)


def quantize(x):
    """fp32 [n] -> (codes uint8 [n], scales fp32 [ceil(n / 256)]), per block:
    scale = fl32(absmax / 448), code = e4m3(fl32(x * fl32(448 / absmax))),
    or e4m3(fl32(x / scale)) where 448 / absmax overflows fp32 (absmax below
    about 1.3e-36); a block whose scale is 0 gets all-zero codes.  (The last
    block is zero padded, which changes neither its absmax nor its codes.)"""
    x = np.asarray(x, dtype=np.float32)
    n = x.size
    nb = (n + BLOCK - 1) // BLOCK
    blocks = np.zeros(nb * BLOCK, dtype=np.float32)
    blocks[:n] = x
    blocks = blocks.reshape(nb, BLOCK)
    absmax = np.abs(blocks).max(axis=1).astype(np.float32)
    scales = (absmax / np.float32(E4M3_MAX)).astype(np.float32)
    with np.errstate(over="ignore"):
        inv = (np.float32(E4M3_MAX) / np.where(absmax > 0, absmax, np.float32(1))).astype(np.float32)
    safe = np.where(scales > 0, scales, np.float32(1)).astype(np.float32)
    q = np.where(np.isfinite(inv)[:, None], blocks * np.where(np.isfinite(inv), inv, np.float32(1))[:, None],
                 blocks / safe[:, None]).astype(np.float32)
    codes = np.where(scales[:, None] > 0, e4m3_encode(q), np.uint8(0))
    return codes.reshape(-1)[:n].astype(np.uint8), scales


def dequantize(codes, scales):
    """fl32(e4m3 value * block scale)."""
    c = np.asarray(codes, dtype=np.uint8)
    s = np.repeat(np.asarray(scales, dtype=np.float32), BLOCK)[:c.size]
    return (e4m3_decode(c) * s).astype(np.float32)


def constants(lr, beta1, beta2, eps, weight_decay, step):
    """The fp32 scalars of one step.  The hyperparameters are fp32 values (as
    a caller passes them); 1 - beta, the step size lr / (1 - beta1^t), the
    factor 1 / sqrt(1 - beta2^t) and the decay factor 1 - lr wd are formed
    from them in fp64 and rounded once."""
    f = np.float32
    lr, beta1, beta2, eps, weight_decay = (float(f(v)) for v in (lr, beta1, beta2, eps, weight_decay))
    bc1 = 1.0 - beta1 ** int(step)
    bc2 = 1.0 - beta2 ** int(step)
    return dict(b1=f(beta1), omb1=f(1.0 - beta1), b2=f(beta2), omb2=f(1.0 - beta2),
                step_size=f(lr / bc1), rsqrt_bc2=f(1.0 / np.sqrt(bc2)),
                decay=f(1.0 - lr * weight_decay), eps=f(eps))


def step_f32(p, g, m0, v0, c):
    """One AdamW step on fp32 arrays (states at full precision): returns the
    new (p, m, v).  Every operation is one fp32 rounding."""
    f = np.float32
    p, g, m0, v0 = (np.asarray(a, dtype=np.float32) for a in (p, g, m0, v0))
    m = f(c["b1"]) * m0 + f(c["omb1"]) * g
    v = f(c["b2"]) * v0 + f(c["omb2"]) * (g * g)
    p1 = p * f(c["decay"])
    den = np.sqrt(v) * f(c["rsqrt_bc2"]) + f(c["eps"])
    p2 = p1 - f(c["step_size"]) * (m / den)
    return p2.astype(np.float32), m.astype(np.float32), v.astype(np.float32)


def step(p, g, m_codes, m_scales, v_codes, v_scales, lr, beta1, beta2, eps, weight_decay, t):
    """One 8-bit AdamW step: dequantize the states, step in fp32, store the
    new states in 8 bits.  Returns (p, p_bf16_bits, m_codes, m_scales,
    v_codes, v_scales)."""
    c = constants(lr, beta1, beta2, eps, weight_decay, t)
    m0 = dequantize(m_codes, m_scales)
    v0 = dequantize(v_codes, v_scales)
    p2, m, v = step_f32(p, g, m0, v0, c)
    mc, ms = quantize(m)
    vc, vs = quantize(v)
    return p2, f32_to_bf16_bits(p2), mc, ms, vc, vs
