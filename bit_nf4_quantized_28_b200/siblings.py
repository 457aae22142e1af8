"""Sibling linears run as one: linears that read the same input (q, k and v
of attention; gate and up of the MLP) share one forward and one backward.

[LoRA y QLoRA en Profundidad, "Módulos Objetivo": LoRA on the attention
projections q_proj, k_proj, v_proj, o_proj or on every linear layer,
including the MLP's gate_proj, up_proj and down_proj; QLoRA glossary, "Come
funziona QLoRA": each such layer is the frozen NF4 weight plus its LoRA
path.]

Siblings W_i [n_i, k] with adapters A_i [r, k], B_i [n_i, r] and the same
alpha / r are one linear with
    W = [W_1; W_2; ...]            (rows stacked, [sum n_i, k])
    A = [A_1; A_2; ...]            ([sum r, k])
    B = blockdiag(B_1, B_2, ...)   ([sum n_i, sum r], zero off the blocks)
    alpha' = alpha * (sum r) / r   (so that alpha' / (sum r) = alpha / r)
because row block i of y = x W^T + s (x A^T) B^T only meets u_i = x A_i^T.
The off-diagonal blocks of B add exact zeros, so each sibling's outputs are
the ones its own call gives.  This module only lays the data out (once, at
load time) and splits the results; every step of the layer runs in the
library's kernels.

The NF4 weights are joined as stored (codes and block scales stacked, and
the double-quantization groups of 256 block scales concatenated), which is
the storage of the stacked weight exactly when every sibling but the last
holds a whole number of groups (n_i * k / 64 a multiple of 256, e.g. any
n_i that is a multiple of 256 at k = 4096).
"""

from dataclasses import dataclass

import torch

from . import NF4Weight


@dataclass
class Siblings:
    """The joined weight and adapters of sibling linears."""
    w: NF4Weight
    A: torch.Tensor            # [sum r, k]
    B: torch.Tensor            # [sum n_i, sum r], block diagonal
    alpha: float               # alpha' of the joined layer
    n: list                    # n_i
    r: int                     # rank of each sibling


def join_weights(ws):
    """Stacks NF4 weights with the same k_in (see the module docstring)."""
    k = ws[0].k_in
    for i, w in enumerate(ws):
        if w.k_in != k:
            raise ValueError("siblings must share k_in")
        if i + 1 < len(ws) and (w.n_out * w.k_in // 64) % 256 != 0:
            raise ValueError("every sibling but the last must hold whole groups of 256 block scales")
    n = sum(w.n_out for w in ws)
    return NF4Weight(n, k, torch.cat([w.codes for w in ws]), torch.cat([w.qscale for w in ws]),
                     torch.cat([w.dq_step for w in ws]), torch.cat([w.dq_mean for w in ws]))


def join(ws, As, Bs, alpha):
    """Joins sibling NF4 weights and their adapters (equal rank and alpha)."""
    r = As[0].shape[0]
    if any(a.shape[0] != r for a in As) or any(b.shape[1] != r for b in Bs):
        raise ValueError("siblings must share the rank")
    n = [w.n_out for w in ws]
    B = torch.zeros(sum(n), r * len(ws), dtype=Bs[0].dtype, device=Bs[0].device)
    row = 0
    for i, b in enumerate(Bs):
        B[row:row + n[i], i * r:(i + 1) * r] = b
        row += n[i]
    return Siblings(join_weights(ws), torch.cat(As).contiguous(), B, float(alpha) * len(ws), n, r)


def split_rows(y, n):
    """Column blocks of y [m, sum n_i] (or row blocks of [sum n_i, ...] with dim=0)."""
    return list(torch.split(y, n, dim=-1))


def split_grads(s, dA, dB):
    """dA [sum r, k] -> the siblings' dA_i; dB [sum n_i, sum r] -> the
    diagonal blocks dB_i (the off-diagonal entries of B are structurally zero
    and take no update)."""
    dAs = list(torch.split(dA, s.r, dim=0))
    dBs, row = [], 0
    for i, ni in enumerate(s.n):
        dBs.append(dB[row:row + ni, i * s.r:(i + 1) * s.r])
        row += ni
    return dAs, dBs
