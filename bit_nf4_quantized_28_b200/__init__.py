"""Python binding of libqlora_nf4.so: the QLoRA NF4 frozen linear on B200.

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels of the library; PyTorch provides device memory and the current
stream.  There is no CPU fallback: if the library is missing or cannot be
loaded, importing the functions below raises.

    w = quantize(W)                      # bf16 [n_out, k_in] on cuda -> NF4Weight
    W_hat = dequantize(w)                # bf16 [n_out, k_in]
    y, u = linear_fwd(x, w, A, B, alpha) # y = x W_hat^T + (alpha/r) (x A^T) B^T
    dx, dA, dB = linear_bwd(dy, x, w, A, B, alpha, u)
    # with LoRA dropout (training): the backward reads x_drop and keep, not x
    y, u, x_drop, keep = linear_fwd_dropout(x, w, A, B, alpha, p, seed, offset)
    dx, dA, dB = linear_bwd_dropout(dy, x_drop, keep, w, A, B, alpha, p, u)
    # 8-bit AdamW on an adapter: fp32 master A32, bf16 copy A for the layer
    st = AdamW8State.zeros(A32.numel(), A32.device)
    adamw8_step(A32.view(-1), dA.view(-1), st, t, lr=2e-4, param_bf16=A.view(-1))

The C declarations, with argument meaning, layout and error behaviour, are
in include/qlora_nf4.h.
"""

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QN_STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "pointer not 16-byte aligned",
    4: "workspace missing or too small", 5: "CUDA error", 6: "device wait timed out",
    7: "device is not sm_100",
}


class QNError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {QN_STATUS.get(status, status)} (status {status})")


class _Weight(ctypes.Structure):
    _fields_ = [("n_out", ctypes.c_int64), ("k_in", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("qscale", ctypes.c_void_p),
                ("dq_step", ctypes.c_void_p), ("dq_mean", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded library (ctypes.CDLL); raises if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m bit_nf4_quantized_28_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, sz, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    u64 = ctypes.c_uint64
    wp = ctypes.POINTER(_Weight)
    sig = {
        "qn_abi_version": (i32, []),
        "qn_status_string": (ctypes.c_char_p, [i32]),
        "qn_last_error_string": (ctypes.c_char_p, []),
        "nf4_levels": (None, [ctypes.POINTER(ctypes.c_float)]),
        "qn_device_error": (i32, [ctypes.POINTER(ctypes.c_int)]),
        "qn_selftest_bounded_wait": (i32, [vp]),
        "nf4_quantize_workspace_bytes": (sz, [i64, i64]),
        "nf4_quantize": (i32, [vp, wp, vp, sz, vp]),
        "nf4_quantize_noalloc": (i32, [vp, wp, vp]),
        "nf4_dequantize": (i32, [wp, vp, vp]),
        "qlora_workspace_bytes": (sz, [i64, i64, i64, i32]),
        "qlora_linear_fwd": (i32, [vp, i64, wp, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "qlora_linear_fwd_gemm": (i32, [vp, i64, wp, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "qlora_linear_fwd_gemv": (i32, [vp, i64, wp, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "qlora_linear_bwd": (i32, [vp, vp, i64, wp, vp, vp, i32, f32, vp, vp, vp, vp, vp, sz, vp]),
        "qlora_merge": (i32, [wp, vp, vp, i32, f32, vp, vp]),
        "qlora_siblings_workspace_bytes": (sz, [i64, i64, i64, i32, i32]),
        "qlora_siblings_fwd": (i32, [vp, i64, wp, i32, vp, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "qlora_siblings_bwd": (i32, [vp, vp, i64, wp, i32, vp, vp, vp, i32, f32, vp, vp, vp, vp, vp, sz, vp]),
        "lora_dropout": (i32, [vp, i64, i64, f32, u64, u64, vp, vp, vp]),
        "qlora_adamw8_blocks": (sz, [i64]),
        "qlora_adamw8_step": (i32, [vp, vp, i64, vp, vp, vp, vp, vp, f32, f32, f32, f32, f32, i64, vp]),
        "qlora_dropout_workspace_bytes": (sz, [i64, i64, i64, i32]),
        "qlora_linear_fwd_dropout": (i32, [vp, i64, wp, vp, vp, i32, f32, f32, u64, u64, vp, vp, vp, vp,
                                           vp, sz, vp]),
        "qlora_linear_bwd_dropout": (i32, [vp, vp, vp, i64, wp, vp, vp, i32, f32, f32, vp, vp, vp, vp, vp,
                                           sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(status, what):
    if status != 0:
        if status == 5:
            what = f"{what} [{lib().qn_last_error_string().decode()}]"
        raise QNError(status, what)


def levels():
    """The 16 NF4 levels as the library computes them (fp32, host)."""
    out = (ctypes.c_float * 16)()
    lib().nf4_levels(out)
    return [out[i] for i in range(16)]


def device_error():
    """Reads and clears the device error word (synchronizes the device)."""
    v = ctypes.c_int(0)
    _check(lib().qn_device_error(ctypes.byref(v)), "qn_device_error")
    return v.value


@dataclass
class NF4Weight:
    """NF4 storage of a frozen weight [n_out, k_in] (device tensors)."""
    n_out: int
    k_in: int
    codes: torch.Tensor     # uint8 [n_out, k_in/2]
    qscale: torch.Tensor    # int8 [n_out*k_in/64]
    dq_step: torch.Tensor   # float32 [ceil(nblk/256)]
    dq_mean: torch.Tensor   # float32 [ceil(nblk/256)]

    def struct(self):
        return _Weight(self.n_out, self.k_in, self.codes.data_ptr(), self.qscale.data_ptr(),
                       self.dq_step.data_ptr(), self.dq_mean.data_ptr())

    @staticmethod
    def empty(n_out, k_in, device="cuda"):
        nblk = n_out * k_in // 64
        ng = (nblk + 255) // 256
        return NF4Weight(n_out, k_in,
                         torch.empty(n_out, k_in // 2, dtype=torch.uint8, device=device),
                         torch.empty(nblk, dtype=torch.int8, device=device),
                         torch.empty(ng, dtype=torch.float32, device=device),
                         torch.empty(ng, dtype=torch.float32, device=device))


def quantize(W, out=None, workspace=None):
    """bf16 W [n_out, k_in] (cuda, contiguous) -> NF4Weight (bit-exact format)."""
    assert W.dtype == torch.bfloat16 and W.is_cuda and W.is_contiguous()
    n_out, k_in = W.shape
    w = out if out is not None else NF4Weight.empty(n_out, k_in, W.device)
    need = lib().nf4_quantize_workspace_bytes(n_out, k_in)
    ws = workspace if workspace is not None else torch.empty(max(need, 256), dtype=torch.uint8, device=W.device)
    st = w.struct()
    _check(lib().nf4_quantize(_ptr(W), ctypes.byref(st), _ptr(ws), ws.numel(), _stream()), "nf4_quantize")
    return w


def quantize_noalloc(W, out=None):
    """quantize() through nf4_quantize_noalloc: no workspace is passed or
    allocated; the library's built-in scratch (up to 2^20 blocks of 64
    weights) is used.  Calls that overlap on the GPU race on that scratch."""
    assert W.dtype == torch.bfloat16 and W.is_cuda and W.is_contiguous()
    n_out, k_in = W.shape
    w = out if out is not None else NF4Weight.empty(n_out, k_in, W.device)
    st = w.struct()
    _check(lib().nf4_quantize_noalloc(_ptr(W), ctypes.byref(st), _stream()), "nf4_quantize_noalloc")
    return w


def dequantize(w, out=None):
    """NF4Weight -> bf16 W_hat [n_out, k_in]."""
    o = out if out is not None else torch.empty(w.n_out, w.k_in, dtype=torch.bfloat16, device=w.codes.device)
    st = w.struct()
    _check(lib().nf4_dequantize(ctypes.byref(st), _ptr(o), _stream()), "nf4_dequantize")
    return o


def merge(w, A=None, B=None, alpha=0.0, out=None, requantize=False):
    """W_hat + (alpha / r) B A as bf16 [n_out, k_in]; with requantize=True the
    merged weight quantized again to NF4 (an NF4Weight)."""
    r = 0 if A is None or B is None else int(A.shape[0])
    o = out if out is not None else torch.empty(w.n_out, w.k_in, dtype=torch.bfloat16, device=w.codes.device)
    st = w.struct()
    _check(lib().qlora_merge(ctypes.byref(st), _ptr(A) if r else None, _ptr(B) if r else None, r, float(alpha),
                             _ptr(o), _stream()), "qlora_merge")
    return quantize(o) if requantize else o


def workspace_bytes(m, n_out, k_in, r):
    return lib().qlora_workspace_bytes(m, n_out, k_in, r)


def make_workspace(m, n_out, k_in, r, device="cuda"):
    """Workspace of a layer call; zeroed once (its last 256 bytes hold the
    decode path's counters, which every call leaves zero)."""
    return torch.zeros(max(workspace_bytes(m, n_out, k_in, r), 256), dtype=torch.uint8, device=device)


def _fwd(fn_name, x, w, A, B, alpha, save_u, y, workspace):
    m = x.shape[0]
    r = 0 if A is None else A.shape[0]
    y = y if y is not None else torch.empty(m, w.n_out, dtype=torch.bfloat16, device=x.device)
    u = torch.empty(m, r, dtype=torch.bfloat16, device=x.device) if (save_u and r > 0) else None
    ws = workspace if workspace is not None else make_workspace(m, w.n_out, w.k_in, r, x.device)
    st = w.struct()
    _check(getattr(lib(), fn_name)(_ptr(x), m, ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha),
                                   _ptr(y), _ptr(u), _ptr(ws), ws.numel(), _stream()), fn_name)
    return y, u


def linear_fwd(x, w, A=None, B=None, alpha=0.0, save_u=True, y=None, workspace=None):
    """y = x W_hat^T + (alpha/r) (x A^T) B^T; returns (y, u = x A^T or None)."""
    return _fwd("qlora_linear_fwd", x, w, A, B, alpha, save_u, y, workspace)


def linear_fwd_gemm(x, w, A=None, B=None, alpha=0.0, save_u=True, y=None, workspace=None):
    return _fwd("qlora_linear_fwd_gemm", x, w, A, B, alpha, save_u, y, workspace)


def linear_fwd_gemv(x, w, A=None, B=None, alpha=0.0, save_u=True, y=None, workspace=None):
    return _fwd("qlora_linear_fwd_gemv", x, w, A, B, alpha, save_u, y, workspace)


def linear_bwd(dy, x, w, A=None, B=None, alpha=0.0, u=None, need_dx=True, out=None, workspace=None):
    """Returns (dx, dA, dB): dx bf16 [m, k_in] (None if not needed), dA fp32
    [r, k_in], dB fp32 [n_out, r] (None without LoRA)."""
    m = dy.shape[0]
    r = 0 if A is None else A.shape[0]
    dev = dy.device
    if out is not None:
        dx, dA, dB = out
    else:
        dx = torch.empty(m, w.k_in, dtype=torch.bfloat16, device=dev) if need_dx else None
        dA = torch.empty(r, w.k_in, dtype=torch.float32, device=dev) if r > 0 else None
        dB = torch.empty(w.n_out, r, dtype=torch.float32, device=dev) if r > 0 else None
    ws = workspace if workspace is not None else make_workspace(m, w.n_out, w.k_in, r, dev)
    st = w.struct()
    _check(lib().qlora_linear_bwd(_ptr(dy), _ptr(x), m, ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha),
                                  _ptr(u), _ptr(dx), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _stream()),
           "qlora_linear_bwd")
    return dx, dA, dB


# ------------------------------------------------------------------ LoRA dropout

def dropout_workspace_bytes(m, n_out, k_in, r):
    return lib().qlora_dropout_workspace_bytes(m, n_out, k_in, r)


def make_dropout_workspace(m, n_out, k_in, r, device="cuda"):
    return torch.zeros(max(dropout_workspace_bytes(m, n_out, k_in, r), 256), dtype=torch.uint8, device=device)


def _u64(v):
    return ctypes.c_uint64(int(v) & 0xFFFFFFFFFFFFFFFF)


def dropout(x, p, seed, offset=0, x_drop=None, keep=None):
    """(x_drop = x * keep, keep) for x bf16 [m, k]: keep is int32 [m, k/32]
    holding the uint32 mask words (bit j % 32 of word j / 32 of a row)."""
    m, k = x.shape
    x_drop = x_drop if x_drop is not None else torch.empty_like(x)
    keep = keep if keep is not None else torch.empty(m, k // 32, dtype=torch.int32, device=x.device)
    _check(lib().lora_dropout(_ptr(x), m, k, float(p), _u64(seed), _u64(offset), _ptr(x_drop), _ptr(keep),
                              _stream()), "lora_dropout")
    return x_drop, keep


def linear_fwd_dropout(x, w, A, B, alpha, p, seed, offset=0, save_u=True, y=None, x_drop=None, keep=None,
                       workspace=None):
    """Training forward with LoRA dropout of rate p: returns (y, u, x_drop, keep),
    y = x W_hat^T + (alpha/r)/(1-p) (x_drop A^T) B^T, u = x_drop A^T."""
    m = x.shape[0]
    r = A.shape[0]
    dev = x.device
    y = y if y is not None else torch.empty(m, w.n_out, dtype=torch.bfloat16, device=dev)
    u = torch.empty(m, r, dtype=torch.bfloat16, device=dev) if save_u else None
    x_drop = x_drop if x_drop is not None else torch.empty_like(x)
    keep = keep if keep is not None else torch.empty(m, w.k_in // 32, dtype=torch.int32, device=dev)
    ws = workspace if workspace is not None else make_dropout_workspace(m, w.n_out, w.k_in, r, dev)
    st = w.struct()
    _check(lib().qlora_linear_fwd_dropout(_ptr(x), m, ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha),
                                          float(p), _u64(seed), _u64(offset), _ptr(y), _ptr(u), _ptr(x_drop),
                                          _ptr(keep), _ptr(ws), ws.numel(), _stream()),
           "qlora_linear_fwd_dropout")
    return y, u, x_drop, keep


def linear_bwd_dropout(dy, x_drop, keep, w, A, B, alpha, p, u=None, need_dx=True, out=None, workspace=None):
    """Backward of linear_fwd_dropout: (dx, dA, dB) from its x_drop, keep and u."""
    m = dy.shape[0]
    r = A.shape[0]
    dev = dy.device
    if out is not None:
        dx, dA, dB = out
    else:
        dx = torch.empty(m, w.k_in, dtype=torch.bfloat16, device=dev) if need_dx else None
        dA = torch.empty(r, w.k_in, dtype=torch.float32, device=dev)
        dB = torch.empty(w.n_out, r, dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else make_dropout_workspace(m, w.n_out, w.k_in, r, dev)
    st = w.struct()
    _check(lib().qlora_linear_bwd_dropout(_ptr(dy), _ptr(x_drop), _ptr(keep), m, ctypes.byref(st), _ptr(A),
                                          _ptr(B), r, float(alpha), float(p), _ptr(u), _ptr(dx), _ptr(dA),
                                          _ptr(dB), _ptr(ws), ws.numel(), _stream()),
           "qlora_linear_bwd_dropout")
    return dx, dA, dB


# ------------------------------------------------------------------ 8-bit AdamW

@dataclass
class AdamW8State:
    """8-bit states of n parameters: E4M3 codes of m and v, one fp32 scale
    per block of 256 (all zero at the start)."""
    m_codes: torch.Tensor
    m_scale: torch.Tensor
    v_codes: torch.Tensor
    v_scale: torch.Tensor

    @staticmethod
    def zeros(n, device="cuda"):
        nb = lib().qlora_adamw8_blocks(n)
        return AdamW8State(torch.zeros(n, dtype=torch.uint8, device=device),
                           torch.zeros(max(nb, 1), dtype=torch.float32, device=device),
                           torch.zeros(n, dtype=torch.uint8, device=device),
                           torch.zeros(max(nb, 1), dtype=torch.float32, device=device))


def adamw8_step(param, grad, state, step, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0,
                param_bf16=None):
    """One AdamW step with 8-bit states on the fp32 tensor param (in place),
    writing bf16(param) into param_bf16 when given."""
    n = param.numel()
    _check(lib().qlora_adamw8_step(_ptr(param), _ptr(grad), n, _ptr(state.m_codes), _ptr(state.m_scale),
                                   _ptr(state.v_codes), _ptr(state.v_scale), _ptr(param_bf16), float(lr),
                                   float(beta1), float(beta2), float(eps), float(weight_decay), int(step),
                                   _stream()), "qlora_adamw8_step")


# ------------------------------------------------------------------ failure detection

WAIT_SELFTEST = 8     # device error bit of selftest_bounded_wait


def selftest_bounded_wait():
    """Enqueues a wait that nothing completes; it gives up after the
    library's limit and sets WAIT_SELFTEST in the device error word."""
    _check(lib().qn_selftest_bounded_wait(_stream()), "qn_selftest_bounded_wait")
