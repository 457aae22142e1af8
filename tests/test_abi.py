"""The C ABI without a GPU: the library loads, exports every function that
include/qlora_nf4.h declares, computes the same NF4 table as the oracle, and
rejects bad arguments before touching the device."""

import ctypes
import os
import re

import numpy as np
import pytest

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import build
from oracle import nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return qn.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            name = m.group(1)
            if name not in ("if", "sizeof", "defined"):
                names.append(name)
    return sorted(set(names))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for call in ("nf4_quantize", "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd"):
        assert call in names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(L, name), f"{name} declared in include/ but not exported"


def test_abi_version(L):
    assert L.qn_abi_version() == 1


def test_levels_match_oracle(L):
    assert np.array_equal(np.array(qn.levels(), np.float32), nf4.nf4_levels())


def test_status_strings(L):
    for s, text in qn.QN_STATUS.items():
        assert L.qn_status_string(s).decode() == text


def test_workspace_sizes(L):
    assert L.nf4_quantize_workspace_bytes(4096, 4096) >= 4096 * 64 * 4
    assert L.nf4_quantize_workspace_bytes(0, 64) == 0
    small = L.qlora_workspace_bytes(16, 256, 256, 8)
    big = L.qlora_workspace_bytes(2048, 4096, 4096, 16)
    assert 0 < small < big
    assert L.qlora_workspace_bytes(-1, 256, 256, 8) == 0
    # the dropout calls also hold dy W_hat in fp32
    assert L.qlora_dropout_workspace_bytes(2048, 4096, 4096, 16) >= big + 2048 * 4096 * 4
    assert L.qlora_dropout_workspace_bytes(-1, 256, 256, 8) == 0


def _w(n=256, k=256, codes=1, qs=1, st=1, mn=1):
    return qn._Weight(n, k, 16 * codes, 16 * qs, 16 * st, 16 * mn)


def test_bad_arguments_rejected_on_host(L):
    w = _w()
    p = ctypes.c_void_p(16)
    # null weight pointer / null input
    assert L.nf4_quantize(p, None, p, 1 << 20, None) == 1
    assert L.nf4_quantize(None, ctypes.byref(w), p, 1 << 20, None) == 1
    # k_in not a multiple of 64
    bad = _w(k=100)
    assert L.nf4_dequantize(ctypes.byref(bad), p, None) == 2
    # misaligned output
    assert L.nf4_dequantize(ctypes.byref(w), ctypes.c_void_p(18), None) == 3
    # workspace too small
    assert L.nf4_quantize(p, ctypes.byref(w), p, 16, None) == 4
    # rank not a multiple of 8, n_out not a multiple of 64
    assert L.qlora_linear_fwd(p, 16, ctypes.byref(w), p, p, 4, 8.0, p, None, p, 1 << 30, None) == 2
    bad_n = _w(n=100)
    assert L.qlora_linear_fwd(p, 16, ctypes.byref(bad_n), p, p, 8, 16.0, p, None, p, 1 << 30, None) == 2
    # LoRA rank given without A/B
    assert L.qlora_linear_fwd(p, 16, ctypes.byref(w), None, None, 8, 16.0, p, None, p, 1 << 30, None) == 1
    # GEMV path accepts at most 16 tokens; m = 0 is a no-op
    assert L.qlora_linear_fwd_gemv(p, 0, ctypes.byref(w), p, p, 8, 16.0, p, None, p, 1 << 30, None) == 0
    assert L.qlora_linear_bwd(None, p, 16, ctypes.byref(w), p, p, 8, 16.0, None, p, p, p, p, 1 << 30, None) == 1
    assert L.qlora_linear_bwd(p, p, 16, ctypes.byref(w), p, p, 8, 16.0, None, p, p, p, p, 64, None) == 4


def test_dropout_bad_arguments_rejected_on_host(L):
    w = _w()
    p = ctypes.c_void_p(16)
    u = ctypes.c_uint64
    # rate outside [0, 1), k not a multiple of 32, misaligned output
    for rate in (1.0, -0.5, float("nan")):
        assert L.lora_dropout(p, 16, 64, rate, u(1), u(0), p, p, None) == 1
    assert L.lora_dropout(p, 16, 48, 0.1, u(1), u(0), p, p, None) == 2
    assert L.lora_dropout(p, 16, 64, 0.1, u(1), u(0), ctypes.c_void_p(24), p, None) == 3
    assert L.lora_dropout(p, 0, 64, 0.1, u(1), u(0), None, None, None) == 0
    fwd = lambda r, rate, xd, ws_bytes: L.qlora_linear_fwd_dropout(
        p, 16, ctypes.byref(w), p, p, r, 16.0, rate, u(1), u(0), p, None, xd, p, p, ws_bytes, None)
    assert fwd(0, 0.1, p, 1 << 30) == 1          # dropout needs a LoRA path
    assert fwd(8, 1.0, p, 1 << 30) == 1
    assert fwd(8, 0.1, None, 1 << 30) == 1       # x_drop is an output the backward needs
    # the plain layer's workspace is too small for the dropout calls
    assert fwd(8, 0.1, p, L.qlora_workspace_bytes(16, 256, 256, 8)) == 4
    bwd = lambda keep, dx: L.qlora_linear_bwd_dropout(p, p, keep, 16, ctypes.byref(w), p, p, 8, 16.0, 0.1,
                                                      None, dx, p, p, p, 1 << 30, None)
    assert bwd(None, p) == 1                     # dx needs the mask
    assert bwd(ctypes.c_void_p(20), p) == 3


def test_adamw8_bad_arguments_rejected_on_host(L):
    p = ctypes.c_void_p(16)
    step = lambda n, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0, t=1, ptr=p: L.qlora_adamw8_step(
        ptr, p, n, p, p, p, p, None, lr, b1, b2, eps, wd, t, None)
    assert L.qlora_adamw8_blocks(0) == 0 and L.qlora_adamw8_blocks(1) == 1 and L.qlora_adamw8_blocks(513) == 3
    assert step(0) == 0                              # nothing to do
    assert step(-1) == 2
    for bad in (dict(b1=1.0), dict(b2=-0.5), dict(eps=0.0), dict(lr=float("inf")), dict(wd=-1.0), dict(t=0)):
        assert step(100, **bad) == 1
    assert step(100, ptr=None) == 1
    assert step(100, ptr=ctypes.c_void_p(20)) == 3


def test_no_gpu_reports_unsupported(L):
    """Well-formed calls on a machine without an sm_100 device are refused
    with a status, never run on the host."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    w = _w()
    p = ctypes.c_void_p(16)
    assert L.nf4_dequantize(ctypes.byref(w), p, None) == 7


def test_siblings_bad_groups_rejected_on_host(L):
    """Sibling calls check the groups before anything else: 1..4 groups, each
    a multiple of 256 rows, summing to the stacked weight's rows, and
    groups * r <= 128."""
    w = _w(n=768)
    p = ctypes.c_void_p(16)
    rows = lambda *v: (ctypes.c_int64 * len(v))(*v)
    fwd = lambda g, rw, r=8: L.qlora_siblings_fwd(p, 16, ctypes.byref(w), g, rw, p, p, r, 16.0, p, None, p,
                                                  1 << 30, None)
    assert fwd(3, rows(256, 256, 128)) == 2          # a group not a multiple of 256 rows
    assert fwd(2, rows(256, 256)) == 2               # rows do not add up to n_out
    assert fwd(0, rows(768)) == 2 and fwd(5, rows(256, 128, 128, 128, 128)) == 2
    assert fwd(3, rows(256, 256, 256), r=48) == 2    # 3 * 48 > 128
    assert fwd(3, None) == 1
    bwd = L.qlora_siblings_bwd(p, p, 16, ctypes.byref(w), 3, rows(256, 256, 128), p, p, 8, 16.0, None, p, p, p,
                               p, 1 << 30, None)
    assert bwd == 2
    assert L.qlora_siblings_workspace_bytes(16, 768, 256, 3, 8) >= L.qlora_workspace_bytes(16, 768, 256, 24)
