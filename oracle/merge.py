"""LoRA merge: the adapter folded back into the dequantized weight, in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

[LoRA y QLoRA en Profundidad, "Cómo Funciona LoRA"]: for inference the LoRA
matrices are merged, W_final = W + (alpha / r) B @ A, with W (d_out x d_in),
A (r x d_in), B (d_out x r).  [QLoRA glossary, "Compromessi"]: merging an
adapter into the 4-bit base model first dequantizes it to 16 bits; "QLoRA e
metodi correlati": the merged 16-bit weights are often quantized again for
deployment.

Reading taken where the pages are silent: W is the dequantized bf16 weight
W_hat of this library, the scale is s = fl32(alpha / r) (the value the layer
uses), B @ A and the sum are exact in fp64, and the result is rounded once to
bf16 (the compute dtype of the QLoRA config).  Re-quantizing the merged
weight is plain NF4 quantization of it (`nf4.quantize`).
"""

import numpy as np

from .linear import lora_scale
from .nf4 import bf16_bits_to_f64, f32_to_bf16_bits


def merge_f64(w_hat_bits, a_bits, b_bits, alpha, r):
    """W_hat + s B @ A in fp64 (no rounding).  w_hat [n, k], A [r, k], B [n, r]."""
    w = bf16_bits_to_f64(w_hat_bits)
    if r == 0:
        return w
    a = bf16_bits_to_f64(a_bits)
    b = bf16_bits_to_f64(b_bits)
    return w + lora_scale(alpha, r) * (b @ a)


def f64_to_bf16_bits(v):
    """Round fp64 values to bf16 (nearest, ties to even) in one step: scale
    by the bf16 ulp of each value (a power of two, so exact), round the
    quotient half-to-even, scale back (exactly representable in bf16).
    Values here are finite and far from the bf16 range limits."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.exp2(e - 7)                       # 8 significant bits
    r = np.where(a > 0, np.rint(v / ulp) * ulp, 0.0)
    return f32_to_bf16_bits(r.astype(np.float32))   # exact: r is a bf16 value


def merge(w_hat_bits, a_bits, b_bits, alpha, r):
    """bf16 bits of W_hat + s B @ A, rounded once from the exact fp64 value."""
    return f64_to_bf16_bits(merge_f64(w_hat_bits, a_bits, b_bits, alpha, r))


def tie_margin(values):
    """Distance of each value from the nearest bf16 rounding boundary, in
    units of its bf16 ulp (0 = exactly on a tie, 0.5 = on a bf16 value)."""
    v = np.abs(np.asarray(values, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    ulp = np.exp2(e - 7)
    frac = (v / ulp) % 1.0
    return np.abs(frac - 0.5)
