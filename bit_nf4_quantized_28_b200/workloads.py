"""Seeded synthetic inputs for the QLoRA NF4 linear workloads.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, so both the CUDA path's tests and the CPU oracle can take
their inputs from it.  Draws use a CPU ``torch.Generator`` seeded per workload,
fp32 normals scaled by the stated standard deviation, then rounded to bf16 on
the host.  Every "N(0, s)" below names the standard deviation s, as the QLoRA
glossary's NF4 snippet draws its weights (``randn * 0.02``).  Draw order is
W, x, A, B, dy.

Workloads (shapes of the layer W [d_out, d_in], x [M, d_in], A [r, d_in],
B [d_out, r]):

* ``tiny``      W 256x256 ~N(0,0.02); x 16x256 ~N(0,1); r 8, alpha 16;
                A ~N(0,1/256); B ~N(0,0.02) and a B = 0 copy; dy ~N(0,1); seed 0
* ``quant``     W 4096x4096 ~N(0,0.02) with 1% of entries scaled x20; seed 1
* ``train``     d_in = d_out = 4096; x 2048x4096 ~N(0,1); r 16, alpha 32;
                A ~N(0,1/4096); B ~N(0,0.02); dy ~N(0,1); seed 2
* ``decode``    4096->11008 and 11008->4096, T in {1, 4, 16}; r 64, alpha 16;
                A ~N(0,1/d_in); B ~N(0,0.02); seed 3
* ``block7b``   q/k/v/o 4096x4096, gate/up 4096->11008, down 11008->4096;
                M = 8192; r 16, alpha 16; each linear its own x, dy and
                generator (seed 400 + index)
"""

from dataclasses import dataclass

import torch


def normal_bf16(gen, shape, std):
    """fp32 standard normals times ``std``, rounded to bf16 (CPU tensor)."""
    t = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t = t * std
    return t.to(torch.bfloat16)


def bits(t):
    """bf16 CPU tensor -> its uint16 bit patterns as a numpy array."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclass
class Linear:
    n_out: int
    k_in: int
    m: int
    r: int
    alpha: float
    W: torch.Tensor
    x: torch.Tensor
    A: torch.Tensor
    B: torch.Tensor
    dy: torch.Tensor


def make_linear(seed, n_out, k_in, m, r, alpha, a_std=None, b_std=0.02, w_std=0.02,
                with_dy=True, gen=None):
    """One seeded linear layer's inputs in the fixed draw order W, x, A, B, dy."""
    g = gen if gen is not None else torch.Generator().manual_seed(seed)
    W = normal_bf16(g, (n_out, k_in), w_std)
    x = normal_bf16(g, (m, k_in), 1.0)
    A = normal_bf16(g, (r, k_in), a_std if a_std is not None else 1.0 / k_in)
    B = normal_bf16(g, (n_out, r), b_std)
    dy = normal_bf16(g, (m, n_out), 1.0) if with_dy else None
    return Linear(n_out, k_in, m, r, alpha, W, x, A, B, dy)


def tiny():
    """256x256 layer, 16 tokens, r 8, alpha 16, seed 0 (plus B = 0 via zero_b)."""
    return make_linear(0, 256, 256, 16, 8, 16.0, a_std=1.0 / 256)


def quant_weight(n_out=4096, k_in=4096, seed=1, outlier_frac=0.01, outlier_mult=20.0):
    """W ~N(0, 0.02) with a seeded 1% of entries multiplied by 20."""
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(n_out, k_in, generator=g, dtype=torch.float32) * 0.02
    n = n_out * k_in
    idx = torch.randperm(n, generator=g)[: int(n * outlier_frac)]
    flat = w.view(-1)
    flat[idx] = flat[idx] * outlier_mult
    return w.to(torch.bfloat16)


def train(m=2048, d=4096, seed=2):
    """d_in = d_out = 4096, x 2048 tokens, r 16, alpha 32, A ~N(0, 1/4096)."""
    return make_linear(seed, d, d, m, 16, 32.0, a_std=1.0 / d)


DECODE_SHAPES = ((11008, 4096), (4096, 11008))   # (d_out, d_in): up and down projections
DECODE_TOKENS = (1, 4, 16)


def decode(n_out, k_in, seed=3):
    """One decode projection drawn for 16 tokens; r 64, alpha 16, A ~N(0, 1/d_in).

    The T = 1 and T = 4 cases use the first T rows of x.  Each projection has
    its own generator, seeded with ``seed`` plus its index in DECODE_SHAPES.
    """
    i = DECODE_SHAPES.index((n_out, k_in)) if (n_out, k_in) in DECODE_SHAPES else 0
    g = torch.Generator().manual_seed(seed + 100 * i)
    return make_linear(seed, n_out, k_in, max(DECODE_TOKENS), 64, 16.0, a_std=1.0 / k_in,
                       with_dy=False, gen=g)


BLOCK7B = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
           ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))


def block7b_layer(name, m=8192, seed=4):
    """One linear of a 7B-shaped decoder block with its own x and dy; each
    layer has its own generator, seeded with 100 * seed + its index."""
    i = [b[0] for b in BLOCK7B].index(name)
    _, n, k = BLOCK7B[i]
    g = torch.Generator().manual_seed(100 * seed + i)
    return make_linear(seed, n, k, m, 16, 16.0, a_std=1.0 / k, gen=g)


def block7b(m=8192, seed=4):
    """The seven linears of a 7B-shaped decoder block, in order."""
    return [(name, block7b_layer(name, m, seed)) for name, _, _ in BLOCK7B]


def snippet_weights(seed=0):
    """The NF4 snippet's input: randn(4096, 64) * 0.02 in fp32 after seed 0."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(4096, 64, generator=g, dtype=torch.float32) * 0.02)
