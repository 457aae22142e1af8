"""Runs a few launches of one hot-path case, for a profiler to capture.

    python -m bit_nf4_quantized_28_b200.profile_case CASE [--launches N]

Cases (seeded synthetic inputs, the shapes the benchmark times):
  gemm_fwd   fused NF4 GEMM forward, base path only: x [2048, 4096], W 4096 x 4096
  gemm_dx    fused NF4 GEMM backward dx, base path only, same sizes
  train      one full training step (forward + backward, rank 16, alpha 32)
  train_dropout  the same step with LoRA dropout p = 0.05
  gemv_t1    decode forward, W 11008 x 4096, 1 token, rank 64, alpha 16
  gemv_t16   decode forward, W 11008 x 4096, 16 tokens, rank 64, alpha 16
  quantize   NF4 quantization of a 4096 x 4096 weight
  dequantize NF4 -> bf16 W_hat of a 4096 x 4096 weight
  merge      LoRA merge W_hat + (alpha / r) B A, 4096 x 4096, rank 16, alpha 16
  adamw8     8-bit AdamW step over a 7B model's adapters (rank 16, all linears: 39,976,960 values)

Each launch is a plain library call (no CUDA graph), so a profiler sees the
kernels one by one; the process synchronizes once at the end.
"""

import argparse
import sys

import torch

import bit_nf4_quantized_28_b200 as qn
from bit_nf4_quantized_28_b200 import workloads as wl

CASES = ("gemm_fwd", "gemm_dx", "train", "train_dropout", "gemv_t1", "gemv_t16", "quantize", "dequantize",
         "merge", "adamw8")


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("case", choices=CASES)
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args(argv)
    dev = torch.device("cuda")
    qn.lib()
    if args.case in ("gemm_fwd", "gemm_dx", "train", "train_dropout"):
        t = wl.train()
        w = qn.quantize(t.W.to(dev))
        x, dy, A, B = t.x.to(dev), t.dy.to(dev), t.A.to(dev), t.B.to(dev)
        ws = (qn.make_dropout_workspace if args.case == "train_dropout" else qn.make_workspace)(
            t.m, t.n_out, t.k_in, t.r, dev)
        y = torch.empty(t.m, t.n_out, dtype=torch.bfloat16, device=dev)
        dx = torch.empty(t.m, t.k_in, dtype=torch.bfloat16, device=dev)
        dA = torch.empty(t.r, t.k_in, dtype=torch.float32, device=dev)
        dB = torch.empty(t.n_out, t.r, dtype=torch.float32, device=dev)
        for _ in range(args.launches):
            if args.case == "gemm_fwd":
                qn.linear_fwd_gemm(x, w, y=y, workspace=ws)
            elif args.case == "gemm_dx":
                qn.linear_bwd(dy, x, w, out=(dx, None, None), workspace=ws)
            elif args.case == "train_dropout":
                _, u, xd, keep = qn.linear_fwd_dropout(x, w, A, B, t.alpha, 0.05, 1234, y=y, workspace=ws)
                qn.linear_bwd_dropout(dy, xd, keep, w, A, B, t.alpha, 0.05, u, out=(dx, dA, dB), workspace=ws)
            else:
                _, u = qn.linear_fwd(x, w, A, B, t.alpha, y=y, workspace=ws)
                qn.linear_bwd(dy, x, w, A, B, t.alpha, u, out=(dx, dA, dB), workspace=ws)
    elif args.case in ("gemv_t1", "gemv_t16"):
        base = wl.decode(11008, 4096)
        T = 1 if args.case == "gemv_t1" else 16
        w = qn.quantize(base.W.to(dev))
        x, A, B = base.x[:T].to(dev), base.A.to(dev), base.B.to(dev)
        ws = qn.make_workspace(T, 11008, 4096, base.r, dev)
        y = torch.empty(T, 11008, dtype=torch.bfloat16, device=dev)
        for _ in range(args.launches):
            qn.linear_fwd(x, w, A, B, base.alpha, save_u=False, y=y, workspace=ws)
    elif args.case == "adamw8":
        n = 32 * (4 * 16 * (4096 + 4096) + 3 * 16 * (4096 + 11008))
        g_ = torch.Generator().manual_seed(5)
        p = (torch.randn(n, generator=g_) * 0.02).to(dev)
        grad = (torch.randn(n, generator=g_) * 1e-3).to(dev)
        st = qn.AdamW8State.zeros(n, dev)
        pb = torch.empty(n, dtype=torch.bfloat16, device=dev)
        for t in range(1, args.launches + 1):
            qn.adamw8_step(p, grad, st, t, lr=2e-4, weight_decay=0.01, param_bf16=pb)
    elif args.case in ("dequantize", "merge"):
        W = wl.quant_weight().to(dev)
        w = qn.quantize(W)
        out = torch.empty(w.n_out, w.k_in, dtype=torch.bfloat16, device=dev)
        g_ = torch.Generator().manual_seed(6)
        A = (torch.randn(16, w.k_in, generator=g_) / w.k_in ** 0.5).to(torch.bfloat16).to(dev)
        B = (torch.randn(w.n_out, 16, generator=g_) * 0.01).to(torch.bfloat16).to(dev)
        for _ in range(args.launches):
            if args.case == "dequantize":
                qn.dequantize(w, out=out)
            else:
                qn.merge(w, A, B, 16.0, out=out)
    else:
        W = wl.quant_weight().to(dev)
        for _ in range(args.launches):
            qn.quantize(W)
    torch.cuda.synchronize()
    print(f"{args.case}: {args.launches} launches ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
