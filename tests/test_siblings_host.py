"""Host logic of sibling linears, on the CPU.

[LoRA y QLoRA en Profundidad, "Módulos Objetivo": q, k, v (and gate, up)
read the same x.]  `siblings.join` lays out siblings for the library's
sibling calls (stacked NF4 storage, stacked A, stacked B, the siblings'
alpha); these tests check the layout with the oracle: the joined storage is
the storage of the stacked weight bit for bit, A and B are the siblings'
adapters stacked, and `split_grads` and `split_rows` return each sibling's
own blocks of stacked results that the oracle computes sibling by sibling.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_28_b200 import NF4Weight, siblings
from bit_nf4_quantized_28_b200 import workloads as wl
from oracle import linear, nf4


def _oracle_weight(W):
    n, k = W.shape
    q = nf4.quantize(wl.bits(W), n, k)
    return NF4Weight(n, k, torch.from_numpy(q["codes"]), torch.from_numpy(q["qscale"]),
                     torch.from_numpy(q["step"]), torch.from_numpy(q["mean"]))


def _siblings(ns, k=256, r=8, seed=3):
    g = torch.Generator().manual_seed(seed)
    Ws = [wl.normal_bf16(g, (n, k), 0.02) for n in ns]
    As = [wl.normal_bf16(g, (r, k), 1.0 / k) for _ in ns]
    Bs = [wl.normal_bf16(g, (n, r), 0.02) for n in ns]
    return Ws, As, Bs


def test_joined_storage_is_the_stacked_weights_storage():
    """Siblings of whole groups of 256 block scales (n * k / 64 % 256 == 0)."""
    Ws, _, _ = _siblings([64, 128, 64], k=256)
    joined = siblings.join_weights([_oracle_weight(W) for W in Ws])
    stacked = _oracle_weight(torch.cat(Ws))
    for f in ("codes", "qscale", "dq_step", "dq_mean"):
        assert torch.equal(getattr(joined, f), getattr(stacked, f)), f
    assert (joined.n_out, joined.k_in) == (256, 256)


def test_partial_group_is_rejected_unless_last():
    Ws, _, _ = _siblings([64, 32], k=256)            # 64 * 256 / 64 = 256 scales, then 128
    siblings.join_weights([_oracle_weight(W) for W in Ws])
    with pytest.raises(ValueError):
        siblings.join_weights([_oracle_weight(W) for W in reversed(Ws)])


def test_join_stacks_the_adapters_and_keeps_alpha():
    ns, k, r, alpha = [64, 128, 64], 256, 8, 16.0
    Ws, As, Bs = _siblings(ns, k, r)
    s = siblings.join([_oracle_weight(W) for W in Ws], As, Bs, alpha)
    assert s.A.shape == (r * len(ns), k) and s.B.shape == (sum(ns), r)
    assert s.alpha == alpha and s.r == r and s.n == ns
    assert torch.equal(s.A, torch.cat(As)) and torch.equal(s.B, torch.cat(Bs))
    with pytest.raises(ValueError):
        siblings.join([_oracle_weight(W) for W in Ws], As, [Bs[0][:, :4]] + Bs[1:], alpha)


def test_split_returns_each_siblings_results():
    """Stacked results computed sibling by sibling by the oracle come back
    per sibling: y blocks by columns, dA by rank rows, dB by output rows."""
    ns, k, r, alpha, m = [64, 128, 64], 256, 8, 16.0, 12
    Ws, As, Bs = _siblings(ns, k, r)
    ows = [_oracle_weight(W) for W in Ws]
    s = siblings.join(ows, As, Bs, alpha)
    g = torch.Generator().manual_seed(9)
    x = wl.normal_bf16(g, (m, k), 1.0)
    dys = [wl.normal_bf16(g, (m, n), 1.0) for n in ns]
    res = []
    for i, n in enumerate(ns):
        q = ows[i]
        wi = nf4.dequantize(q.codes.numpy(), q.qscale.numpy(), q.dq_step.numpy(), q.dq_mean.numpy(), n, k)
        yi, _ = linear.forward(wl.bits(x), wi, wl.bits(As[i]), wl.bits(Bs[i]), alpha, r)
        _, dAi, dBi = linear.backward(wl.bits(dys[i]), wl.bits(x), wi, wl.bits(As[i]), wl.bits(Bs[i]), alpha, r)
        res.append((yi, dAi, dBi))
    y = torch.from_numpy(np.concatenate([t[0] for t in res], axis=1))
    dA = torch.from_numpy(np.concatenate([t[1] for t in res], axis=0))
    dB = torch.from_numpy(np.concatenate([t[2] for t in res], axis=0))
    ys = siblings.split_rows(y, ns)
    dAs, dBs = siblings.split_grads(s, dA, dB)
    for i in range(len(ns)):
        assert np.array_equal(ys[i].numpy(), res[i][0])
        assert np.array_equal(dAs[i].numpy(), res[i][1])
        assert np.array_equal(dBs[i].numpy(), res[i][2])
