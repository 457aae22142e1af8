"""Host logic of fused sibling linears, on the CPU.

[LoRA y QLoRA en Profundidad, "Módulos Objetivo": q, k, v (and gate, up)
read the same x.]  `siblings.join` lays out siblings as one layer (stacked
NF4 storage, stacked A, block-diagonal B, alpha scaled by the number of
siblings); these tests check the layout with the oracle: the joined storage
is the storage of the stacked weight bit for bit, the joined layer's forward
is the siblings' forwards side by side, and `split_grads` returns each
sibling's own dA and dB.
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


def test_joined_forward_and_gradients_are_the_siblings():
    ns, k, r, alpha, m = [64, 128, 64], 256, 8, 16.0, 12
    Ws, As, Bs = _siblings(ns, k, r)
    ows = [_oracle_weight(W) for W in Ws]
    s = siblings.join(ows, As, Bs, alpha)
    assert s.B.shape == (sum(ns), r * len(ns)) and s.alpha == alpha * len(ns)
    # off-diagonal blocks of B are zero
    row = 0
    for i, n in enumerate(ns):
        blk = s.B[row:row + n]
        assert torch.count_nonzero(torch.cat([blk[:, :i * r], blk[:, (i + 1) * r:]], 1)) == 0
        row += n
    g = torch.Generator().manual_seed(9)
    x = wl.normal_bf16(g, (m, k), 1.0)
    dys = [wl.normal_bf16(g, (m, n), 1.0) for n in ns]
    w_hat = nf4.dequantize(s.w.codes.numpy(), s.w.qscale.numpy(), s.w.dq_step.numpy(), s.w.dq_mean.numpy(),
                           sum(ns), k)
    y, _ = linear.forward(wl.bits(x), w_hat, wl.bits(s.A), wl.bits(s.B), s.alpha, r * len(ns))
    dy = torch.cat(dys, 1)
    dx, dA, dB = linear.backward(wl.bits(dy), wl.bits(x), w_hat, wl.bits(s.A), wl.bits(s.B), s.alpha, r * len(ns))
    ys = siblings.split_rows(torch.from_numpy(y), ns)
    dAs, dBs = siblings.split_grads(s, torch.from_numpy(dA), torch.from_numpy(dB))
    dx_sum = 0
    row = 0
    for i, n in enumerate(ns):
        wi = w_hat[row:row + n]
        yi, _ = linear.forward(wl.bits(x), wi, wl.bits(As[i]), wl.bits(Bs[i]), alpha, r)
        dxi, dAi, dBi = linear.backward(wl.bits(dys[i]), wl.bits(x), wi, wl.bits(As[i]), wl.bits(Bs[i]), alpha, r)
        assert np.allclose(ys[i].numpy(), yi, rtol=1e-12, atol=1e-12)
        assert np.allclose(dAs[i].numpy(), dAi, rtol=1e-12, atol=1e-12)
        assert np.allclose(dBs[i].numpy(), dBi, rtol=1e-12, atol=1e-12)
        dx_sum = dx_sum + dxi
        row += n
    # dx of the joined layer is the sum of the siblings' dx
    assert np.allclose(dx, dx_sum, rtol=1e-12, atol=1e-12)
