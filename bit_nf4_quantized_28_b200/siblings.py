"""Sibling linears run as one: linears that read the same input (q, k and v
of attention; gate and up of the MLP) share one forward and one backward.

[LoRA y QLoRA en Profundidad, "Módulos Objetivo": LoRA on the attention
projections q_proj, k_proj, v_proj, o_proj or on every linear layer,
including the MLP's gate_proj, up_proj and down_proj; QLoRA glossary, "Come
funziona QLoRA": each such layer is the frozen NF4 weight plus its LoRA
path.]

Siblings W_i [n_i, k] with adapters A_i [r, k], B_i [n_i, r] of the same
rank and alpha are stored once, stacked: W = [W_1; W_2; ...] as NF4,
A = [A_1; A_2; ...] ([G r, k]) and B = [B_1; B_2; ...] ([sum n_i, r]).  The
library's sibling calls (qlora_siblings_fwd / _bwd) take the row counts n_i
and run every sibling's LoRA path at its own rank r: u = x A^T once for all
siblings, and output rows of sibling i take their LoRA product from its r
columns of u.  This module lays the data out (once, at load time), calls
them and splits the results; every step of the layer runs in the library's
kernels.

The NF4 weights are joined as stored (codes and block scales stacked, and
the double-quantization groups of 256 block scales concatenated), which is
the storage of the stacked weight exactly when every sibling but the last
holds a whole number of groups (n_i * k / 64 a multiple of 256, e.g. any
n_i that is a multiple of 256 at k = 4096).  The library requires each n_i
to be a multiple of 256.
"""

import ctypes
from dataclasses import dataclass

import torch

from . import NF4Weight, _check, _ptr, _stream, lib


@dataclass
class Siblings:
    """The joined weight and adapters of sibling linears."""
    w: NF4Weight
    A: torch.Tensor            # [G r, k], the A_i stacked
    B: torch.Tensor            # [sum n_i, r], the B_i stacked
    alpha: float               # the siblings' alpha (s = alpha / r)
    n: list                    # n_i
    r: int                     # rank of each sibling

    def rows(self):
        return (ctypes.c_int64 * len(self.n))(*self.n)


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
    if any(b.shape[0] != ni for b, ni in zip(Bs, n)):
        raise ValueError("B_i must have n_i rows")
    return Siblings(join_weights(ws), torch.cat(As).contiguous(), torch.cat(Bs).contiguous(), float(alpha), n, r)


def workspace_bytes(m, s):
    return lib().qlora_siblings_workspace_bytes(m, s.w.n_out, s.w.k_in, len(s.n), s.r)


def make_workspace(m, s, device="cuda"):
    """Workspace of a sibling call; zeroed once (its last 256 bytes hold the
    decode path's counters, which every call leaves zero)."""
    return torch.zeros(max(workspace_bytes(m, s), 256), dtype=torch.uint8, device=device)


def forward(x, s, save_u=True, y=None, workspace=None):
    """y = [y_1 | y_2 | ...] bf16 [m, sum n_i] and u = x A^T bf16 [m, G r]
    (None unless save_u)."""
    m = x.shape[0]
    y = y if y is not None else torch.empty(m, s.w.n_out, dtype=torch.bfloat16, device=x.device)
    u = torch.empty(m, len(s.n) * s.r, dtype=torch.bfloat16, device=x.device) if save_u else None
    ws = workspace if workspace is not None else make_workspace(m, s, x.device)
    st = s.w.struct()
    _check(lib().qlora_siblings_fwd(_ptr(x), m, ctypes.byref(st), len(s.n), s.rows(), _ptr(s.A), _ptr(s.B),
                                    s.r, float(s.alpha), _ptr(y), _ptr(u), _ptr(ws), ws.numel(), _stream()),
           "qlora_siblings_fwd")
    return y, u


def backward(dy, x, s, u=None, need_dx=True, out=None, workspace=None):
    """(dx, dA, dB): dx bf16 [m, k] (the siblings' sum; None if not needed),
    dA fp32 [G r, k] and dB fp32 [sum n_i, r] (the siblings' gradients
    stacked)."""
    m = dy.shape[0]
    dev = dy.device
    if out is not None:
        dx, dA, dB = out
    else:
        dx = torch.empty(m, s.w.k_in, dtype=torch.bfloat16, device=dev) if need_dx else None
        dA = torch.empty(len(s.n) * s.r, s.w.k_in, dtype=torch.float32, device=dev)
        dB = torch.empty(s.w.n_out, s.r, dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else make_workspace(m, s, dev)
    st = s.w.struct()
    _check(lib().qlora_siblings_bwd(_ptr(dy), _ptr(x), m, ctypes.byref(st), len(s.n), s.rows(), _ptr(s.A),
                                    _ptr(s.B), s.r, float(s.alpha), _ptr(u), _ptr(dx), _ptr(dA), _ptr(dB),
                                    _ptr(ws), ws.numel(), _stream()),
           "qlora_siblings_bwd")
    return dx, dA, dB


def split_rows(y, n):
    """Column blocks of y [m, sum n_i]."""
    return list(torch.split(y, n, dim=-1))


def split_grads(s, dA, dB):
    """dA [G r, k] -> the siblings' dA_i; dB [sum n_i, r] -> their dB_i."""
    return list(torch.split(dA, s.r, dim=0)), list(torch.split(dB, s.n, dim=0))
