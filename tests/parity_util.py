"""Shared helpers of the GPU parity tests: the tolerance rule and cached
oracle results (the oracle always quantizes from the seeded bf16 weight
itself; nothing it uses comes from the CUDA path)."""

import hashlib

import numpy as np
import torch

from oracle import linear, nf4
from bit_nf4_quantized_28_b200 import workloads as wl

# y, dx, dA, dB: max |g - o| <= 2e-2 * rms(o) and sum|g - o| / sum|o| <= 5e-3.
MAX_ABS_REL_RMS = 2e-2
MEAN_REL = 5e-3


def check_close(got, ref, what=""):
    g = np.asarray(got, dtype=np.float64)
    o = np.asarray(ref, dtype=np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - o)
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.abs(o).sum())
    mean_rel = float(err.sum() / denom) if denom > 0 else float(err.sum())
    assert max_abs <= MAX_ABS_REL_RMS * rms + 1e-30, f"{what}: max|err| {max_abs:.3e} > 2e-2 * rms {rms:.3e}"
    assert mean_rel <= MEAN_REL, f"{what}: mean relative error {mean_rel:.3e} > 5e-3"
    return max_abs / max(rms, 1e-30), mean_rel


def to_np(t):
    """GPU/CPU tensor -> numpy (bf16 as float32 values, exact)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def bits_of(t):
    return wl.bits(t.detach().cpu())


_oracle_cache = {}


def oracle_storage(_unused_key, w_bf16):
    """Oracle quantization (and W_hat bits) of a CPU bf16 weight, cached by
    the weight's contents."""
    b = wl.bits(w_bf16)
    key = (b.shape, hashlib.sha1(b.tobytes()).hexdigest())
    if key not in _oracle_cache:
        n, k = w_bf16.shape
        q = nf4.quantize(b, n, k)
        q["w_hat"] = nf4.dequantize(q["codes"], q["qscale"], q["step"], q["mean"], n, k)
        _oracle_cache[key] = q
    return _oracle_cache[key]


def oracle_forward(x_bits, w_hat_bits, a_bits, b_bits, alpha, r):
    return linear.forward(x_bits, w_hat_bits, a_bits, b_bits, alpha, r)


def oracle_backward(dy_bits, x_bits, w_hat_bits, a_bits, b_bits, alpha, r):
    return linear.backward(dy_bits, x_bits, w_hat_bits, a_bits, b_bits, alpha, r)
