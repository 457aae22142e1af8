"""GPU parity of the 8-bit AdamW step against the oracle: parameters (fp32
and bf16), E4M3 state codes and block scales, bit for bit, over several
steps (each side carries its own states), for ragged sizes, one LoRA pair of
the training shape, and every adapter of a 7B model (all seven linears,
rank 16) in one array."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_28_b200 as qn
from oracle import adamw8

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)

# adapters of one 7B decoder layer at rank 16: q, k, v, o (4096 x 4096),
# gate, up (11008 x 4096), down (4096 x 11008): r (d_in + d_out) each
ADAPTERS_7B = 32 * (4 * 16 * (4096 + 4096) + 3 * 16 * (4096 + 11008))


def _grads(n, steps, seed):
    """Gradients whose magnitude varies by block (1e-6 .. 1e-1), with an
    all-zero block and blocks of tiny values when n allows."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(steps):
        g = rng.standard_normal(n).astype(np.float32)
        scale = np.repeat(np.exp(rng.uniform(np.log(1e-6), np.log(1e-1), (n + 255) // 256)), 256)[:n]
        g = (g * scale).astype(np.float32)
        if n > 768:
            g[256:512] = 0.0
            g[512:768] *= np.float32(1e-30)
        if n > 1024:
            g[768:1024] *= np.float32(1e-35)      # moments where 448 / absmax overflows, and subnormals
        out.append(g)
    return out


def _run(n, steps=3, seed=0, with_bf16=True):
    rng = np.random.default_rng(seed + 1)
    p_host = (rng.standard_normal(n) * 0.02).astype(np.float32)
    grads = _grads(n, steps, seed)
    p = torch.tensor(p_host, device="cuda")
    st = qn.AdamW8State.zeros(n)
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda") if with_bf16 else None
    nb = (n + 255) // 256
    op, omc, oms, ovc, ovs = p_host, np.zeros(n, np.uint8), np.zeros(nb, np.float32), np.zeros(n, np.uint8), \
        np.zeros(nb, np.float32)
    for t, g in enumerate(grads, start=1):
        qn.adamw8_step(p, torch.tensor(g, device="cuda"), st, t, param_bf16=pb, **HP)
        op, opb, omc, oms, ovc, ovs = adamw8.step(op, g, omc, oms, ovc, ovs, t=t, **HP)
        torch.cuda.synchronize()
        assert np.array_equal(p.cpu().numpy().view(np.uint32), op.view(np.uint32)), f"p at step {t}"
        assert np.array_equal(st.m_codes.cpu().numpy(), omc), f"m codes at step {t}"
        assert np.array_equal(st.v_codes.cpu().numpy(), ovc), f"v codes at step {t}"
        assert np.array_equal(st.m_scale.cpu().numpy()[:nb].view(np.uint32), oms.view(np.uint32))
        assert np.array_equal(st.v_scale.cpu().numpy()[:nb].view(np.uint32), ovs.view(np.uint32))
        if with_bf16:
            assert np.array_equal(pb.cpu().view(torch.int16).numpy().view(np.uint16), opb)
    return op


@pytest.mark.parametrize("n", [1, 8, 250, 1000, 4096 + 24])
def test_ragged_sizes(n):
    _run(n, steps=3, seed=n)


def test_training_shape_pair():
    """A [16, 4096] and B [4096, 16] of the training-shape layer, one array."""
    _run(2 * 16 * 4096, steps=4, seed=7)


def test_without_bf16_copy():
    _run(3000, steps=2, seed=9, with_bf16=False)


def test_hyperparameters_are_checked():
    p = torch.zeros(16, device="cuda")
    st = qn.AdamW8State.zeros(16)
    for bad in (dict(beta1=1.0), dict(beta2=-0.1), dict(eps=0.0), dict(lr=float("nan"))):
        kw = dict(HP, **bad)
        with pytest.raises(qn.QNError):
            qn.adamw8_step(p, p, st, 1, **kw)
    with pytest.raises(qn.QNError):
        qn.adamw8_step(p, p, st, 0, **HP)


def test_all_adapters_of_a_7b_model():
    """39,976,960 parameters (every linear of 32 layers at rank 16) in one
    call, as the benchmark times it: one step, compared in full."""
    _run(ADAPTERS_7B, steps=1, seed=11)
