"""The frozen QLoRA linear layer with its LoRA path, forward and backward, in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Shapes follow [LoRA y QLoRA en Profundidad, "Cómo Funciona LoRA"]: W is
(d_out x d_in), A is (r x d_in), B is (d_out x r), delta_W = B @ A, and the
update is scaled by alpha / r ["Alpha (lora_alpha)"].  The forward adds the
LoRA path's output to the base path computed with the dequantized weight; the
backward sends the gradient through the dequantized weight to the input and
gives gradients to A and B only [QLoRA glossary, "Come funziona QLoRA"].

Inputs are bf16 bit patterns (uint16); they are widened exactly and every
product and sum below is fp64 (numpy matmul on fp64 arrays).  The scale is
s = fl32(alpha / r), the value the kernels use.  u = x A^T is kept in fp64
(the pages do not say whether the LoRA intermediate is rounded).
"""

import numpy as np

from .nf4 import bf16_bits_to_f64


def lora_scale(alpha, r):
    """s = alpha / r, rounded to fp32.  [LoRA y QLoRA en Profundidad, "Alpha"]"""
    return float(np.float32(np.float32(alpha) / np.float32(r)))


def forward(x_bits, w_hat_bits, a_bits, b_bits, alpha, r):
    """y = x W_hat^T + s (x A^T) B^T, returned with u = x A^T (both fp64).

    x: [M, d_in], W_hat: [d_out, d_in] (the dequantized bf16 weight), A:
    [r, d_in], B: [d_out, r].  A or B may be None (base path only).
    """
    x = bf16_bits_to_f64(x_bits)
    w = bf16_bits_to_f64(w_hat_bits)
    if a_bits is None or b_bits is None or r == 0:
        return forward_f64(x, w, None, None, 0.0)
    return forward_f64(x, w, bf16_bits_to_f64(a_bits), bf16_bits_to_f64(b_bits),
                       lora_scale(alpha, r))


def forward_f64(x, w, a, b, s):
    """The forward on fp64 arrays (a, b may be None); returns (y, u)."""
    y = x @ w.T
    if a is None or b is None:
        return y, None
    u = x @ a.T
    return y + s * (u @ b.T), u


def backward(dy_bits, x_bits, w_hat_bits, a_bits, b_bits, alpha, r):
    """Gradients of <dy, y> for the forward above, in fp64.

    dx = dy W_hat + s (dy B) A;  dA = s (dy B)^T x;  dB = s dy^T (x A^T).
    The frozen weight gets no gradient.  [QLoRA glossary, "Come funziona
    QLoRA"; Módulo 4: QLoRA, 4.4 (only the LoRA parameters are trained)]
    """
    dy = bf16_bits_to_f64(dy_bits)
    x = bf16_bits_to_f64(x_bits)
    w = bf16_bits_to_f64(w_hat_bits)
    if a_bits is None or b_bits is None or r == 0:
        return backward_f64(dy, x, w, None, None, 0.0)
    return backward_f64(dy, x, w, bf16_bits_to_f64(a_bits), bf16_bits_to_f64(b_bits),
                        lora_scale(alpha, r))


def backward_f64(dy, x, w, a, b, s):
    """The backward on fp64 arrays; returns (dx, dA, dB), dA = dB = None
    without a LoRA path."""
    dx = dy @ w
    if a is None or b is None:
        return dx, None, None
    v = dy @ b
    dx = dx + s * (v @ a)
    d_a = s * (v.T @ x)
    d_b = s * (dy.T @ (x @ a.T))
    return dx, d_a, d_b


def matmul_loops(p, q):
    """Textbook triple loop in Python floats, for tiny brute-force checks."""
    n, k = len(p), len(p[0])
    m = len(q[0])
    out = [[0.0] * m for _ in range(n)]
    for i in range(n):
        for j in range(m):
            acc = 0.0
            for t in range(k):
                acc += p[i][t] * q[t][j]
            out[i][j] = acc
    return out
