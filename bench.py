"""Benchmark of the QLoRA NF4 frozen linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--quick]

One step = one training pass of the QLoRA linear at d_in = d_out = 4096,
2048 tokens (batch 4 x seq 512), rank 16, alpha 32: the forward (u = x A^T,
y = x W_hat^T + s u B^T with the NF4 dequantization fused into the GEMM) and
the backward (v = dy B, dx = dy W_hat + s v A, dA, dB).  Inputs are seeded
synthetic tensors already resident in HBM; a rotation of input sets larger
than the 126 MB L2 keeps every step reading HBM.  Steps are CUDA-graph
replays of the library's own launches, timed with CUDA events on the
launching stream; with N > 1 each rank runs an independent replica of the
step (no collective on the data path) and the time is the max over ranks.

The JSON line adds: the decode GEMV (4096 -> 11008 and 11008 -> 4096,
1/4/16 tokens, GB/s), NF4 quantize / dequantize of 4096 x 4096 (GB/s), the
7B block's seven linears at 8192 tokens (TFLOP/s), the training step with LoRA
dropout p = 0.05 and its mask kernel, the 8-bit AdamW step over a 7B model's
adapters, the LoRA merge, joined q/k/v decode, the roofline of the fused
GEMM, an end-to-end number through host buffers, the SM clocks seen during
the timed region, and the CPU oracle timed on a bounded sample.

--impl reference times the CPU oracle (the plain definition of the method)
on the same workload and metric, on a bounded sample of rows per step.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s and decode GEMV GB/s, % of B200 roofline"
M, D, R, ALPHA = 2048, 4096, 16, 32.0
WORKLOAD = ("QLoRA NF4 linear training step, d_in = d_out = 4096, x 2048 x 4096 bf16 "
            "(batch 4 x seq 512), rank 16, alpha 32, fwd + bwd (y, dx, dA, dB)")
L2_BYTES = 126 * 1024 * 1024


# Kernels of one training step: forward = rank-r (u) + fused GEMM; backward
# with u saved = rank-r (v) + rank-r (dA, dB) + fused GEMM (dx).
LAUNCHES_PER_STEP = 5


def train_flops(m, n, k, r):
    """fwd 2MNK + 2Mr(K+N); bwd 2MNK + 4Mr(N+K) (dx through W, v, dx LoRA, dA, dB)."""
    return 2 * m * n * k + 2 * m * r * (k + n) + 2 * m * n * k + 4 * m * r * (n + k)


# DRAM bytes of one launch of the fused GEMM at the training shape, read
# from an ncu capture (profiles/qlora_gemm_traffic.json) together with a
# hash of the kernel's sources at the time; a changed kernel reports null.
GEMM_SOURCES = ("bit_nf4_quantized_28_b200/csrc/gemm_tc.cuh", "bit_nf4_quantized_28_b200/csrc/common.cuh")


def sources_sha1(paths):
    import hashlib
    h = hashlib.sha1()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(path=None):
    """(bytes per launch, description) of the GEMM capture, or (None, why)."""
    path = path or os.path.join(ROOT, "profiles", "qlora_gemm_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None, "no capture recorded"
    if rec.get("sources_sha1") != sources_sha1(GEMM_SOURCES):
        return None, "kernel changed since the capture"
    return rec.get("dram_bytes_per_launch"), rec.get("note", "")


def dist_env():
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x, device, world):
    """The largest x over all ranks, returned on every rank (x itself alone)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, work_per_rank, ms):
    """Whole-job rate (work per second) when every rank did work_per_rank and
    the slowest took ms milliseconds (weak scaling: independent replicas)."""
    return world * work_per_rank / (ms * 1e-3)


# nominal B200 figures, reported beside the measured denominators
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- GPU arm

class TrainSet:
    """One independent copy of the training-step inputs, outputs and workspace."""

    def __init__(self, qn, t, dev):
        import torch
        self.W = t.W.to(dev)
        self.w = qn.quantize(self.W)
        del self.W
        self.x = t.x.to(dev)
        self.A = t.A.to(dev)
        self.B = t.B.to(dev)
        self.dy = t.dy.to(dev)
        self.y = torch.empty(t.m, t.n_out, dtype=torch.bfloat16, device=dev)
        self.dx = torch.empty(t.m, t.k_in, dtype=torch.bfloat16, device=dev)
        self.dA = torch.empty(t.r, t.k_in, dtype=torch.float32, device=dev)
        self.dB = torch.empty(t.n_out, t.r, dtype=torch.float32, device=dev)
        self.ws = qn.make_workspace(t.m, t.n_out, t.k_in, t.r, dev)
        self.alpha = t.alpha

    def bytes(self):
        b = sum(v.numel() * v.element_size() for v in (self.x, self.A, self.B, self.dy, self.y, self.dx,
                                                        self.dA, self.dB))
        w = self.w
        return b + sum(v.numel() * v.element_size() for v in (w.codes, w.qscale, w.dq_step, w.dq_mean))

    def step(self, qn):
        y, u = qn.linear_fwd(self.x, self.w, self.A, self.B, self.alpha, y=self.y, workspace=self.ws)
        qn.linear_bwd(self.dy, self.x, self.w, self.A, self.B, self.alpha, u,
                      out=(self.dx, self.dA, self.dB), workspace=self.ws)


def graph_of(fn, warm=2):
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(warm):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graphs(graphs, reps):
    """Average device time of one replay, cycling through `graphs`."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for i in range(reps):
        graphs[i % len(graphs)].replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def decode_bench(qn, wl, dev, reps=200):
    """GEMV GB/s per shape and token count; weight copies rotate past L2."""
    import torch
    out = {}
    hbm, _, _, _ = peaks()
    for (n, k) in wl.DECODE_SHAPES:
        base = wl.decode(n, k)
        w0 = qn.quantize(base.W.to(dev))
        wbytes = sum(v.numel() * v.element_size() for v in (w0.codes, w0.qscale, w0.dq_step, w0.dq_mean))
        copies = max(2, math.ceil(3 * L2_BYTES / wbytes))
        ws = [w0] + [qn.NF4Weight(n, k, w0.codes.clone(), w0.qscale.clone(), w0.dq_step.clone(),
                                  w0.dq_mean.clone()) for _ in range(copies - 1)]
        A, B = base.A.to(dev), base.B.to(dev)
        for T in wl.DECODE_TOKENS:
            x = base.x[:T].to(dev)
            y = torch.empty(T, n, dtype=torch.bfloat16, device=dev)
            wsp = qn.make_workspace(T, n, k, base.r, dev)
            # one graph runs the call once per weight copy (amortises replay overhead)
            g = graph_of(lambda: [qn.linear_fwd(x, w, A, B, base.alpha, save_u=False, y=y, workspace=wsp)
                                  for w in ws])
            ms = time_graphs([g], max(3, reps // len(ws))) / len(ws)
            graphs = [g]
            byts = wbytes + (A.numel() + B.numel() + x.numel() + y.numel()) * 2
            gbs = byts / (ms * 1e-3) / 1e9
            out[f"{n}x{k}_T{T}"] = {"us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                                    "frac_hbm": round(gbs / hbm, 3),
                                    "frac_hbm_nominal": round(gbs / NOMINAL_HBM_GBS, 3), "bytes": byts}
            del graphs
        del ws
        torch.cuda.empty_cache()
    return out


DROPOUT_P = 0.05


def dropout_bench(qn, sets, ms_plain, reps=20):
    """The training step with LoRA dropout p = 0.05 (the rate of the lesson's
    config) on the same rotating input sets: forward = mask + x_drop, u,
    fused GEMM; backward = base GEMM (fp32), v, dA / dB, masked LoRA dx.
    Also the mask kernel alone (GB/s: x read, x_drop and keep written)."""
    import torch
    extra = []
    for s in sets:
        d = {"xd": torch.empty_like(s.x),
             "keep": torch.empty(s.x.shape[0], s.x.shape[1] // 32, dtype=torch.int32, device=s.x.device),
             "ws": qn.make_dropout_workspace(s.x.shape[0], s.w.n_out, s.w.k_in, s.A.shape[0], s.x.device)}
        extra.append(d)

    def step(s, d):
        y, u, xd, keep = qn.linear_fwd_dropout(s.x, s.w, s.A, s.B, s.alpha, DROPOUT_P, 1234, 0, y=s.y,
                                               x_drop=d["xd"], keep=d["keep"], workspace=d["ws"])
        qn.linear_bwd_dropout(s.dy, xd, keep, s.w, s.A, s.B, s.alpha, DROPOUT_P, u, out=(s.dx, s.dA, s.dB),
                              workspace=d["ws"])

    graphs = [graph_of(lambda s=s, d=d: step(s, d)) for s, d in zip(sets, extra)]
    ms = time_graphs(graphs, max(3 * len(graphs), reps))
    mask_graphs = [graph_of(lambda s=s, d=d: qn.dropout(s.x, DROPOUT_P, 1234, 0, x_drop=d["xd"], keep=d["keep"]))
                   for s, d in zip(sets, extra)]
    ms_mask = time_graphs(mask_graphs, max(3 * len(mask_graphs), 5 * reps))
    x = sets[0].x
    mask_bytes = 2 * x.numel() * 2 + x.numel() // 8
    hbm, _, _, _ = peaks()
    gbs = mask_bytes / (ms_mask * 1e-3) / 1e9
    del graphs, mask_graphs
    return {"p": DROPOUT_P, "us": round(ms * 1e3, 1), "TFLOP/s": round(train_flops(M, D, D, R) / (ms * 1e-3) / 1e12, 1),
            "over_plain_step_us": round((ms - ms_plain) * 1e3, 1), "launches_per_step": 7,
            "mask_kernel": {"us": round(ms_mask * 1e3, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                            "bytes": mask_bytes}}


# adapters of a 7B decoder at rank 16 on all seven linears: q, k, v, o
# (4096 x 4096), gate, up (11008 x 4096), down (4096 x 11008), 32 layers
ADAPTERS_7B = 32 * (4 * 16 * (4096 + 4096) + 3 * 16 * (4096 + 11008))


def adamw8_bench(qn, dev, reps=20):
    """One 8-bit AdamW step over every adapter of the 7B model in one array
    (39,976,960 parameters; 720 MB of traffic, far past L2).  Bytes: p, g,
    both code arrays read; p, both code arrays, the bf16 copy written; the
    block scales read and written."""
    import torch
    n = ADAPTERS_7B
    g_ = torch.Generator(device="cpu").manual_seed(5)
    p = (torch.randn(n, generator=g_) * 0.02).to(dev)
    grad = (torch.randn(n, generator=g_) * 1e-3).to(dev)
    st = qn.AdamW8State.zeros(n, dev)
    pb = torch.empty(n, dtype=torch.bfloat16, device=dev)
    qn.adamw8_step(p, grad, st, 1, lr=2e-4, weight_decay=0.01, param_bf16=pb)
    g = graph_of(lambda: qn.adamw8_step(p, grad, st, 2, lr=2e-4, weight_decay=0.01, param_bf16=pb))
    ms = time_graphs([g], reps)
    nb = (n + 255) // 256
    byts = n * (4 + 4 + 1 + 1) + n * (4 + 1 + 1 + 2) + 4 * nb * 4
    hbm, _, _, _ = peaks()
    gbs = byts / (ms * 1e-3) / 1e9
    del g
    return {"params": n, "us": round(ms * 1e3, 1), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
            "bytes": byts}


def merge_bench(qn, wl, dev, reps=20):
    """LoRA merge W_hat + (alpha/r) B A -> bf16 of the 4096 x 4096 training
    weight, rank 16; weight copies rotate past L2.  Bytes: codes, scales,
    A and B read, the bf16 weight written."""
    import torch
    t = wl.train()
    w0 = qn.quantize(t.W.to(dev))
    A, B = t.A.to(dev), t.B.to(dev)
    wbytes = sum(v.numel() * v.element_size() for v in (w0.codes, w0.qscale, w0.dq_step, w0.dq_mean))
    obytes = t.n_out * t.k_in * 2
    copies = max(2, math.ceil(3 * L2_BYTES / (wbytes + obytes)))
    ws = [w0] + [qn.NF4Weight(t.n_out, t.k_in, w0.codes.clone(), w0.qscale.clone(), w0.dq_step.clone(),
                              w0.dq_mean.clone()) for _ in range(copies - 1)]
    outs = [torch.empty(t.n_out, t.k_in, dtype=torch.bfloat16, device=dev) for _ in range(copies)]
    g = graph_of(lambda: [qn.merge(w, A, B, t.alpha, out=o) for w, o in zip(ws, outs)])
    ms = time_graphs([g], max(3, reps)) / copies
    byts = wbytes + obytes + (A.numel() + B.numel()) * 2
    hbm, _, _, _ = peaks()
    gbs = byts / (ms * 1e-3) / 1e9
    return {"shape": [t.n_out, t.k_in], "rank": t.r, "us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
            "frac_hbm": round(gbs / hbm, 3), "bytes": byts}


def siblings_bench(qn, wl, dev, reps=20):
    """q, k, v of a 4096-wide attention block at decode (1 token, rank 16,
    alpha 32): three calls against one call of the joined layer; weight
    copies rotate past L2."""
    import torch
    from bit_nf4_quantized_28_b200 import siblings
    ts = [wl.make_linear(900 + i, 4096, 4096, 1, 16, 32.0, a_std=1.0 / 4096, with_dy=False) for i in range(3)]
    x = ts[0].x.to(dev)
    one = [qn.quantize(t.W.to(dev)) for t in ts]
    As, Bs = [t.A.to(dev) for t in ts], [t.B.to(dev) for t in ts]
    wbytes = sum(sum(v.numel() * v.element_size() for v in (w.codes, w.qscale, w.dq_step, w.dq_mean)) for w in one)
    sets = max(2, math.ceil(3 * L2_BYTES / wbytes))
    copies = [one] + [[qn.NF4Weight(w.n_out, w.k_in, w.codes.clone(), w.qscale.clone(), w.dq_step.clone(),
                                    w.dq_mean.clone()) for w in one] for _ in range(sets - 1)]
    joined = [siblings.join(c, As, Bs, 32.0) for c in copies]
    ys = [torch.empty(1, 4096, dtype=torch.bfloat16, device=dev) for _ in range(3)]
    yj = torch.empty(1, 3 * 4096, dtype=torch.bfloat16, device=dev)
    ws1 = qn.make_workspace(1, 4096, 4096, 16, dev)
    wsj = siblings.make_workspace(1, joined[0], dev)
    g_sep = graph_of(lambda: [qn.linear_fwd(x, w, As[i], Bs[i], 32.0, save_u=False, y=ys[i], workspace=ws1)
                              for c in copies for i, w in enumerate(c)])
    g_join = graph_of(lambda: [siblings.forward(x, j, save_u=False, y=yj, workspace=wsj) for j in joined])
    sep = time_graphs([g_sep], max(3, reps)) / sets
    jn = time_graphs([g_join], max(3, reps)) / sets
    return {"shape": "3 x 4096 x 4096, 1 token, rank 16", "separate_us": round(sep * 1e3, 2),
            "joined_us": round(jn * 1e3, 2), "speedup": round(sep / jn, 2)}


def quant_bench(qn, wl, dev, reps=20):
    import torch
    W = wl.quant_weight().to(dev)
    n, k = W.shape
    copies = 4
    Ws = [W] + [W.clone() for _ in range(copies - 1)]
    outs = [qn.NF4Weight.empty(n, k, dev) for _ in range(copies)]
    need = qn.lib().nf4_quantize_workspace_bytes(n, k)
    wsp = torch.empty(need, dtype=torch.uint8, device=dev)
    gq = graph_of(lambda: [qn.quantize(Ws[i], out=outs[i], workspace=wsp) for i in range(copies)])
    ms_q = time_graphs([gq], reps) / copies
    hats = [torch.empty(n, k, dtype=torch.bfloat16, device=dev) for _ in range(copies)]
    gd = graph_of(lambda: [qn.dequantize(outs[i], out=hats[i]) for i in range(copies)])
    ms_d = time_graphs([gd], reps) / copies
    wb = n * k * 2
    sb = n * k // 2 + n * k // 64 + 2 * 4 * math.ceil(n * k / 64 / 256)
    hbm, _, _, _ = peaks()
    q_gbs = (wb + sb) / (ms_q * 1e-3) / 1e9
    d_gbs = (wb + sb) / (ms_d * 1e-3) / 1e9
    # round-trip error of the NF4 weight (W_hat from the library's dequantize,
    # double-quantized scales) beside evenly spaced INT4 on the same blocks
    mse = float(((hats[0].float() - W.float()) ** 2).mean())
    mse_int4, mse_nf4_exact = block_round_trip_mse(W, torch.linspace(-1.0, 1.0, 16, device=dev)), \
        block_round_trip_mse(W, torch.tensor(qn.levels(), device=dev))
    return {"shape": [n, k], "quantize_us": round(ms_q * 1e3, 1), "quantize_GB/s": round(q_gbs, 1),
            "quantize_frac_hbm": round(q_gbs / hbm, 3), "dequantize_us": round(ms_d * 1e3, 1),
            "dequantize_GB/s": round(d_gbs, 1), "dequantize_frac_hbm": round(d_gbs / hbm, 3),
            "bits_per_param_scales": 8 / 64 + 64 / (64 * 256), "mse_nf4_round_trip": mse,
            "mse_nf4_exact_scales": mse_nf4_exact, "mse_int4_exact_scales": mse_int4,
            "nf4_over_int4": round(mse_nf4_exact / mse_int4, 4),
            "mse_note": "blocks of 64 along d_in, absmax scale; INT4 = 16 evenly spaced levels on [-1, 1], "
                        "nearest level; the exact-scale pair compares the two level sets alone, "
                        "mse_nf4_round_trip is the library's stored format (int8 double-quantized scales)"}


def block_round_trip_mse(W, levels):
    """Mean squared error of quantizing W [n, k] (bf16, cuda) in blocks of 64
    along k to `levels` times the block absmax (nearest level, first on a
    tie) and back, with fp32 torch operations: the comparison the NF4 snippet
    prints, evaluated on the benchmark's weight.  Not a path of the library."""
    import torch
    blocks = W.float().reshape(-1, 64)
    a = blocks.abs().amax(dim=1, keepdim=True)
    x = blocks / torch.where(a > 0, a, torch.ones_like(a))
    err = 0.0
    for i in range(0, x.shape[0], 1 << 16):       # chunks keep the [rows, 64, 16] distances small
        xc = x[i:i + (1 << 16)]
        idx = (xc.unsqueeze(-1) - levels).abs().argmin(dim=-1)
        err += float(((levels[idx] * a[i:i + (1 << 16)] - blocks[i:i + (1 << 16)]) ** 2).sum())
    return err / blocks.numel()


def block7b_bench(qn, wl, dev, reps=5):
    import torch
    sets = []
    flops = 0
    for name, n, k in wl.BLOCK7B:
        t = wl.block7b_layer(name)
        sets.append(TrainSet(qn, t, dev))
        flops += train_flops(t.m, n, k, t.r)
        del t
    g = graph_of(lambda: [s.step(qn) for s in sets])
    ms = time_graphs([g], reps)
    _, tc, tcs, _ = peaks()
    tf = flops / (ms * 1e-3) / 1e12
    out = {"ms": round(ms, 3), "TFLOP/s": round(tf, 1), "frac_tensor_burst": round(tf / tc, 3),
           "frac_tensor_sustained": round(tf / tcs, 3), "tflop": round(flops / 1e12, 3)}
    del sets, g
    torch.cuda.empty_cache()
    return out


def gemm_roofline(qn, sets, reps=20):
    """Average duration of the fused tensor-core GEMM kernel alone (forward
    y = x W_hat^T and dx = dy W_hat, the base product without the rank-r
    slice), timed by CUDA events around single-kernel calls."""
    import torch
    gf = [graph_of(lambda s=s: qn.linear_fwd_gemm(s.x, s.w, y=s.y, workspace=s.ws)) for s in sets]
    gb = [graph_of(lambda s=s: qn.linear_bwd(s.dy, s.x, s.w, out=(s.dx, None, None), workspace=s.ws))
          for s in sets]
    ms_f = time_graphs(gf, reps)
    ms_b = time_graphs(gb, reps)
    return ms_f, ms_b


# What the end-to-end steps read back: the step's result, the LoRA
# gradients (the trainable parameters' updates); y and dx stay on the device,
# where the neighbouring layers of a model consume them.
E2E_RESULTS = ("dA", "dB")


def e2e_bench(qn, t, dev, steps, results=E2E_RESULTS):
    """Same step through host buffers: every step copies its x and dy from
    pinned host memory to the device, runs the fwd + bwd calls and copies
    its result (`results`: dA and dB) back to pinned host memory.  As a
    training loop overlaps loading the next batch with the current one, the
    steps run on two device sets and three streams (host -> device, compute,
    device -> host), so that step i's input copies overlap step i - 1's
    compute and step i - 2's result copies; a set is reloaded only after its
    previous step has read it and recomputed only after its results were
    copied out."""
    import torch
    sets = [TrainSet(qn, t, dev) for _ in range(2)]
    hx = t.x.pin_memory()
    hdy = t.dy.pin_memory()
    outs = [{k: torch.empty(getattr(s, k).shape, dtype=getattr(s, k).dtype).pin_memory()
             for k in results} for s in sets]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        b = i % 2
        s, o = sets[b], outs[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_cmp[b])        # step i - 2 has read this set's inputs
            s.x.copy_(hx, non_blocking=True)
            s.dy.copy_(hdy, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            if i >= 2:
                s_cmp.wait_event(ev_out[b])       # step i - 2's results are on the host
            s.step(qn)
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            for k in results:
                o[k].copy_(getattr(s, k), non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(3, 3 + steps):
        one(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = (hx.numel() + hdy.numel()) * 2
    d2h = sum(v.numel() * v.element_size() for v in outs[0].values())
    return ms, h2d, d2h


# ---------------------------------------------------------------- CPU oracle

def oracle_step_sample(rows=256):
    """Builds a bounded sample of the training step for the CPU oracle: the
    full weight (dequantized on each pass, as the method does) and `rows`
    tokens of x and dy."""
    from bit_nf4_quantized_28_b200 import workloads as wl
    from oracle import nf4
    t = wl.train()
    q = nf4.quantize(wl.bits(t.W), t.n_out, t.k_in)
    return {"q": q, "x": wl.bits(t.x[:rows]), "dy": wl.bits(t.dy[:rows]), "A": wl.bits(t.A),
            "B": wl.bits(t.B), "rows": rows, "t": t}


def oracle_step(s):
    from oracle import linear, nf4
    q, t = s["q"], s["t"]
    w_hat = nf4.dequantize(q["codes"], q["qscale"], q["step"], q["mean"], t.n_out, t.k_in)
    linear.forward(s["x"], w_hat, s["A"], s["B"], t.alpha, t.r)
    w_hat = nf4.dequantize(q["codes"], q["qscale"], q["step"], q["mean"], t.n_out, t.k_in)
    linear.backward(s["dy"], s["x"], w_hat, s["A"], s["B"], t.alpha, t.r)


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(steps=3, rows=256):
    s = oracle_step_sample(rows)
    oracle_step(s)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_step(s)
    dt = (time.perf_counter() - t0) / steps
    tf = train_flops(rows, D, D, R) / dt / 1e12
    out = {"value": tf, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
           "sample": f"{rows} of 2048 tokens per step (fwd + bwd; W dequantized on both passes), "
                     f"{steps} steps, {dt:.2f} s per step"}
    # the same step on one host thread (one step of it)
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            oracle_step(s)
            dt1 = time.perf_counter() - t0
        out["single_thread"] = {"value": train_flops(rows, D, D, R) / dt1 / 1e12, "cores": 1,
                                "sample": f"one step of the same sample, {dt1:.2f} s"}
    except ImportError:
        pass
    return out


def run_reference(args):
    _, rank, _ = dist_env()
    if rank != 0:
        return
    rows = 128 if args.quick else 256
    s = oracle_step_sample(rows)
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_step(s)
    t0 = time.perf_counter()
    steps = max(1, args.steps)
    for _ in range(steps):
        oracle_step(s)
    dt = (time.perf_counter() - t0) / steps
    tf = train_flops(rows, D, D, R) / dt / 1e12
    cores = oracle_threads()
    line = {"impl": "reference", "metric": METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample_rows": rows},
            "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} of 2048 tokens per step, W dequantized on both passes"},
            "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--quick", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import torch.distributed as dist

    import bit_nf4_quantized_28_b200 as qn
    from bit_nf4_quantized_28_b200 import workloads as wl

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    qn.lib()
    warmup = max(3, args.warmup)

    def barrier():
        if world > 1:
            dist.barrier()

    # ------------------------------------------------------------ headline: training step
    t = wl.train()
    first = TrainSet(qn, t, dev)
    nsets = max(2, math.ceil(3 * L2_BYTES / first.bytes()))
    sets = [first] + [TrainSet(qn, t, dev) for _ in range(nsets - 1)]
    graphs = [graph_of(lambda s=s: s.step(qn)) for s in sets]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    # the warm-up steps run right before the timed ones (no idle gap between them)
    for i in range(warmup):
        graphs[i % nsets].replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        graphs[i % nsets].replay()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev, world)
    flops = train_flops(M, D, D, R)
    value = job_rate(world, flops, ms) / 1e12
    hbm, tc_burst, tc_sus, peak_src = peaks()

    # ------------------------------------------------------------ roofline of the fused GEMM
    ms_f, ms_b = gemm_roofline(qn, sets)
    gemm_flops = 2 * M * D * D
    ach = gemm_flops / (0.5 * (ms_f + ms_b) * 1e-3) / 1e12
    traffic, traffic_note = recorded_traffic()
    # the GEMM is timed alone in short replays at full clocks: the burst peak
    # is its denominator; the sustained one (a seconds-long loop under the
    # power cap) is reported beside it
    roofline = {"bound": "tensor", "kernel": "qlora_gemm_kernel (fused NF4 dequant + tcgen05 GEMM)",
                "achieved": round(ach, 1), "peak": tc_burst, "unit": "TFLOP/s",
                "frac": round(ach / tc_burst, 3), "traffic": traffic, "traffic_note": traffic_note,
                "peak_source": f"{peak_src} burst bf16", "fwd_us": round(ms_f * 1e3, 1),
                "dx_us": round(ms_b * 1e3, 1), "frac_of_sustained": round(ach / tc_sus, 3),
                "frac_of_nominal": round(ach / NOMINAL_BF16_TFLOPS, 3),
                "flops_per_launch": gemm_flops}
    del graphs
    torch.cuda.empty_cache()

    # ------------------------------------------------------------ secondary workloads
    secondary = {}
    if not args.quick:
        secondary["decode_gemv"] = decode_bench(qn, wl, dev)
        secondary["quantize_4096x4096"] = quant_bench(qn, wl, dev)
        secondary["merge_4096x4096_r16"] = merge_bench(qn, wl, dev)
        secondary["siblings_qkv_decode"] = siblings_bench(qn, wl, dev)
        secondary["train_step_lora_dropout"] = dropout_bench(qn, sets, ms)
        secondary["adamw8_7b_adapters"] = adamw8_bench(qn, dev)
        del sets
        torch.cuda.empty_cache()
        secondary["block7b_fwd_bwd"] = block7b_bench(qn, wl, dev)
    else:
        del sets
        torch.cuda.empty_cache()

    # ------------------------------------------------------------ end to end through host buffers
    e2e_ms, h2d, d2h = e2e_bench(qn, t, dev, steps=max(5, min(args.steps, 20)))
    e2e_val = job_rate(world, flops, max_over_ranks(e2e_ms, dev, world)) / 1e12

    err = qn.device_error()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "m": M, "d_in": D, "d_out": D, "rank": R, "alpha": ALPHA,
                       "l2": f"{nsets} rotating input sets of {first.bytes() / 2**20:.0f} MiB (> 126 MB L2)",
                       "timing": "CUDA-graph replays of the library's launches, CUDA events",
                       "parallelism": "replicas" if world > 1 else "single",
                       "frac_tensor_burst": round(value / world / tc_burst, 3),
                       "frac_tensor_sustained": round(value / world / tc_sus, 3)},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_val, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "h2d_tensors": ["x", "dy"], "d2h_tensors": list(E2E_RESULTS)},
            "gpu_launches": args.steps * LAUNCHES_PER_STEP,
            "clocks": clk,
            "device_error_word": err,
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
