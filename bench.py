#!/usr/bin/env python
"""Benchmark of the QLoRA hot path on B200 (one JSON line on rank 0).

Workload (default, "linear7b"): one LLaMA-7B layer's seven QLoRA linears
(q, k, v, o: 4096x4096; gate, up: 11008x4096; down: 4096x11008), 4096 tokens
(8 x 512) bf16 ~N(0, 1), r = 64, alpha = 16, NF4 + double-quantized frozen
weights ~N(0, 0.02) (synthetic, seeded).  One step = forward of the seven
linears (Y bf16, H saved) then their backward in reverse order (dX bf16, dA,
dB); with N > 1 processes every rank runs its own 4096 tokens and the adapter
gradients of the step are summed over ranks with one NCCL all-reduce (weak
scaling, data parallel).  value = total FLOP / time, FLOP per linear
4MNK + 6Mr(N+K).

The line also carries "codec": the NF4 + double-quantization round trip
(quantize then dequantize) over the 224 tensors of LLaMA-7B (6,476,005,376
bf16 weights ~N(0, 0.02)), algorithmic bytes 2.5159 per weight each way.

--impl reference times the oracle (float64 CPU implementation) on the same
metric, on a bounded sample per step.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s; NF4 (de)quant GB/s; fraction of roofline"
R, ALPHA, TOKENS = 64, 16.0, 4096
CODEC_BYTES_PER_WEIGHT = 2 + 0.5 + 1 / 64 + 4 / (64 * 256)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def linear_flops(M, N, K, r):
    return 4 * M * N * K + 6 * M * r * (N + K)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch from one
# ncu capture of the bench workloads, averaged over the launches of one step
# (the committed DRAM-traffic capture).  Each set describes the kernel sources
# whose SHA-256 it names and is reported only while they are unchanged.
_CSRC = os.path.join("bit_nf4_quantized_16_b200", "csrc")
MEASURED_TRAFFIC = {
    "linear": {
        "sources": ['gemm_pair.cuh', 'gemm.cuh', 'sm100.cuh', 'nf4_expand.cuh', 'linear.cu'],
        "sha256": "ceea941933843257c5ca362b56432e2fe88d59453937c6c75df7b0a5ad227317",
        "bytes": {"fwd_fused": 98.65e6, "bwd_fused": 111.93e6},
    },
    "codec": {
        "sources": ['codec.cu', 'nf4_expand.cuh', 'exact_mean.cuh'],
        "sha256": "9a7b14c79aad62eb21d1fa0581aa376d3ad0e7f64654f9402d7a4711c77a9406",
        "bytes": {"quantize": 58.64e6, "dequantize": 27.07e6},
    },
}


def measured_traffic(group, kernel):
    import hashlib
    t = MEASURED_TRAFFIC[group]
    h = hashlib.sha256()
    for f in t["sources"]:
        with open(os.path.join(ROOT, _CSRC, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != t["sha256"]:
        return None   # the kernels changed since the capture
    return t["bytes"].get(kernel)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---- clocks during the timed region -------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 9:
                    rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---- our arm ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bit_nf4_quantized_16_b200 as q
    from bit_nf4_quantized_16_b200 import dp
    import synthetic

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks, peak_src = load_peaks()

    # ---- set-up (untimed): quantize the seven frozen weights, allocate activations
    TOKENS = args.tokens
    if args.linears == "llama7b":
        shapes = synthetic.LLAMA7B_LINEARS
    else:
        n_, k_ = (int(v) for v in args.linears.lower().split("x"))
        shapes = [("single", n_, k_)]
    layers = []
    ws_bytes = 0
    qws_bytes = max(q.qlora_quantize_workspace_bytes(N, K) for _, N, K in shapes)
    qws = torch.empty(qws_bytes, dtype=torch.uint8, device=dev)
    grads = torch.empty(sum(R * K + N * R for _, N, K in shapes), dtype=torch.float32, device=dev)
    off = 0
    for i, (name, N, K) in enumerate(shapes):
        seed = 1000 * rank + 10 * i
        W = synthetic.normal((N, K), 0.02, seed, torch.bfloat16, dev)
        w = q.NF4Weight(N, K, device=dev)
        q.qlora_quantize_nf4_dq(W, w, qws)
        del W
        L = {
            "name": name, "N": N, "K": K, "w": w,
            "X": synthetic.normal((TOKENS, K), 1.0, seed + 1, torch.bfloat16, dev),
            "A": synthetic.normal((R, K), 1.0 / R, seed + 2, torch.bfloat16, dev),
            "B": synthetic.normal((N, R), 0.01, seed + 3, torch.bfloat16, dev),
            "dY": synthetic.normal((TOKENS, N), 1.0, seed + 4, torch.bfloat16, dev),
            "Y": torch.empty(TOKENS, N, dtype=torch.bfloat16, device=dev),
            "H": torch.empty(TOKENS, R, dtype=torch.float32, device=dev),
            "dX": torch.empty(TOKENS, K, dtype=torch.bfloat16, device=dev),
            "dA": grads[off: off + R * K].view(R, K),
            "dB": grads[off + R * K: off + R * K + N * R].view(N, R),
            "grad": grads[off: off + R * K + N * R],
        }
        off += R * K + N * R
        layers.append(L)
        ws_bytes = max(ws_bytes, q.qlora_linear_workspace_bytes(TOKENS, N, K, R))
    del qws
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    scale = ALPHA / R
    step_flops = sum(linear_flops(TOKENS, L["N"], L["K"], R) for L in layers)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2

    reducer = dp.OverlappedGradSum()

    # The seven linears are independent, so each linear's small adapter
    # products (H in the forward; G, then dA and dB, in the backward) run on a
    # low-priority side stream through the split-off adapter calls, beside
    # the previous linear's fused GEMM: they become runnable when that GEMM
    # does (an event recorded just before it), the GEMM's CTAs take the SMs
    # first, and the small kernels fill the SMs its partial last round of
    # tiles leaves idle.  Each linear then has its own workspace.
    mode = {"split": not args.no_adapter_split}
    gemm_s = torch.cuda.Stream(priority=-1)
    side_s = torch.cuda.Stream(priority=0)
    for L in layers:
        L["ws"] = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if mode["split"] else ws
        L["ev"] = [torch.cuda.Event() for _ in range(4)]   # fwd adapter done, fwd GEMM next, same for bwd

    def step():
        if not mode["split"]:
            for L in layers:
                q.qlora_linear_fwd(L["w"], L["X"], TOKENS, L["A"], L["B"], R, scale, L["Y"], L["H"], ws)
            for L in reversed(layers):
                q.qlora_linear_bwd(L["w"], L["X"], L["dY"], TOKENS, L["A"], L["B"], R, scale, L["H"], L["dX"],
                                   L["dA"], L["dB"], ws)
                reducer.ready(L["grad"])   # this linear's dA, dB: summed while the backward goes on
            reducer.wait()
            return
        cur = torch.cuda.current_stream()
        gemm_s.wait_stream(cur)
        side_s.wait_stream(cur)
        for phase, order in (("fwd", layers), ("bwd", list(reversed(layers)))):
            done, go = (0, 1) if phase == "fwd" else (2, 3)

            def adapter(L):
                with torch.cuda.stream(side_s):
                    if phase == "fwd":
                        q.qlora_linear_adapter_fwd(L["w"], L["X"], TOKENS, L["A"], L["B"], R, scale, L["H"],
                                                   L["ws"], stream=side_s)
                    else:
                        q.qlora_linear_adapter_bwd(L["w"], L["X"], L["dY"], TOKENS, L["A"], L["B"], R, scale,
                                                   L["H"], L["ws"], stream=side_s)
                    L["ev"][done].record(side_s)

            # host order matters: every event is recorded before a stream waits on it
            adapter(order[0])
            for i, L in enumerate(order):
                with torch.cuda.stream(gemm_s):
                    gemm_s.wait_event(L["ev"][done])
                    L["ev"][go].record(gemm_s)
                    if phase == "fwd":
                        q.qlora_linear_fwd(L["w"], L["X"], TOKENS, L["A"], L["B"], R, scale, L["Y"], L["H"],
                                           L["ws"], stream=gemm_s, adapter_ready=True)
                    else:
                        # the input gradient alone: dA and dB need G, not dX, and follow on the side stream
                        q.qlora_linear_bwd(L["w"], L["X"], L["dY"], TOKENS, L["A"], L["B"], R, scale, L["H"],
                                           L["dX"], None, None, L["ws"], stream=gemm_s, adapter_ready=True)
                if i + 1 < len(order):
                    # the next linear's adapter products become runnable with this GEMM
                    side_s.wait_event(L["ev"][go])
                    adapter(order[i + 1])
                if phase == "bwd":
                    with torch.cuda.stream(side_s):
                        q.qlora_linear_bwd(L["w"], L["X"], L["dY"], TOKENS, L["A"], L["B"], R, scale, L["H"],
                                           None, L["dA"], L["dB"], L["ws"], stream=side_s, adapter_ready=True)
                        reducer.ready(L["grad"])   # this linear's dA, dB: summed while the backward goes on
            if phase == "fwd":
                # the backward's adapter call rewrites the workspace the forward GEMM read
                side_s.wait_stream(gemm_s)
        with torch.cuda.stream(gemm_s):
            reducer.wait()
        cur.wait_stream(gemm_s)
        cur.wait_stream(side_s)

    def timed_steps(k, fn):
        """Device time of k steps, each after an L2 flush, CUDA events on the
        launching stream; a sleep kernel lets the host enqueue a whole step
        before the GPU reaches it."""
        total = 0.0
        for _ in range(k):
            flush.zero_()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            torch.cuda._sleep(20_000_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        return total

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    q.qlora_check_device_error()

    # ---- timed region (headline): no per-launch events, so that consecutive
    # kernels overlap set-up and tail as they do for a user
    launches0 = q.qlora_launch_count()
    with ClockSampler(local_rank) as clk:
        ms = timed_steps(args.steps, step)
    launches = q.qlora_launch_count() - launches0
    q.qlora_check_device_error()
    # ---- per-kernel device times: the same steps again with CUDA events around
    # every launch (on the launching stream), undivided calls on one stream so
    # that each launch's time is its own and not shared with a concurrent one
    split_headline = mode["split"]
    mode["split"] = False
    q.qlora_timing_reset()
    q.qlora_timing_enable(True)
    ms_events = timed_steps(args.steps, step)
    q.qlora_timing_enable(False)
    mode["split"] = split_headline
    kern = q.qlora_timing_read()
    q.qlora_check_device_error()
    clocks = clk.summary()
    ms = dp.max_over_ranks(ms, dev)
    value = step_flops * args.steps * world / (ms * 1e-3) / 1e12

    # ---- end to end through the same API with host buffers
    pin = {}
    for L in layers:
        pin[L["name"]] = {"X": L["X"].cpu().pin_memory(), "dY": L["dY"].cpu().pin_memory()}
    host_grads = torch.empty(grads.shape, dtype=torch.float32).pin_memory()
    h2d = sum(L["X"].numel() * 2 + L["dY"].numel() * 2 for L in layers)
    d2h = grads.numel() * 4

    copy_s = torch.cuda.Stream()

    def e2e_step():
        # host-to-device copies on a side stream, in the order the kernels
        # need them, so that they overlap the compute of the linears before
        main = torch.cuda.current_stream()
        copy_s.wait_stream(main)   # the previous step no longer reads these buffers
        ev_x, ev_dy = [], []
        with torch.cuda.stream(copy_s):
            for L in layers:
                L["X"].copy_(pin[L["name"]]["X"], non_blocking=True)
                ev_x.append(torch.cuda.Event())
                ev_x[-1].record(copy_s)
            for L in reversed(layers):
                L["dY"].copy_(pin[L["name"]]["dY"], non_blocking=True)
                ev_dy.append(torch.cuda.Event())
                ev_dy[-1].record(copy_s)
        for L, e in zip(layers, ev_x):
            main.wait_event(e)
            q.qlora_linear_fwd(L["w"], L["X"], TOKENS, L["A"], L["B"], R, scale, L["Y"], L["H"], ws)
        for L, e in zip(reversed(layers), ev_dy):
            main.wait_event(e)
            q.qlora_linear_bwd(L["w"], L["X"], L["dY"], TOKENS, L["A"], L["B"], R, scale, L["H"], L["dX"],
                               L["dA"], L["dB"], ws)
            reducer.ready(L["grad"])
        reducer.wait()
        host_grads.copy_(grads, non_blocking=True)

    e2e_step()
    e2e_ms = timed_steps(args.steps, e2e_step)
    e2e_ms = dp.max_over_ranks(e2e_ms, dev)
    e2e_value = step_flops * args.steps * world / (e2e_ms * 1e-3) / 1e12

    # ---- roofline of the dominant kernel (largest device time in the timed region)
    kflops = {
        "fwd_fused": sum(2 * TOKENS * L["N"] * L["K"] + 2 * TOKENS * L["N"] * R for L in layers) * args.steps,
        "bwd_fused": sum(2 * TOKENS * L["N"] * L["K"] + 2 * TOKENS * L["K"] * R for L in layers) * args.steps,
    }
    dom = max(("fwd_fused", "bwd_fused"), key=lambda k: kern[k][0])
    dom_ms, dom_n = kern[dom]
    achieved = kflops[dom] / (dom_ms * 1e-3) / 1e12
    # burst peak: the timed region lasts tens of milliseconds and the SM clock
    # stays at its maximum (the sustained figure is for seconds under the power cap)
    peak = peaks["bf16_tflops"]
    roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": measured_traffic("linear", dom),
                "peak_source": f"{peak_src} bf16_tflops (burst)",
                "launches": dom_n, "avg_launch_ms": round(dom_ms / max(dom_n, 1), 4),
                "timing": "CUDA events around every launch on its stream, in a second pass of the same steps "
                          "with undivided linear calls on one stream (no concurrent kernel)"}
    breakdown = {k: {"ms_per_step": round(v[0] / args.steps, 4), "launches_per_step": v[1] // args.steps}
                 for k, v in kern.items() if v[1]}

    variants = run_variants7b(args, q, torch, dev, layers, timed_steps, step_flops, TOKENS, scale, peaks, peak_src) \
        if (rank == 0 and not args.skip_variants and args.linears == "llama7b") else None
    codec = run_codec(args, q, torch, dev, peaks, peak_src) if (rank == 0 and not args.skip_codec) else None
    decode = run_decode65b(args, q, torch, dev, peaks, peak_src) if (rank == 0 and not args.skip_decode) else None
    adamw = run_adamw7b(args, q, torch, dev, peaks, peak_src) if (rank == 0 and not args.skip_optim) else None
    blockr = run_block7b(args, q, torch, dev, peaks, peak_src) if (rank == 0 and not args.skip_block) else None
    del layers, ws, grads, flush
    stack = run_stack65b(args, q, torch, dev, peaks, peak_src) if (rank == 0 and not args.skip_stack) else None

    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) weights quantized to NF4+DQ, N(0,1) activations and gradients)",
        "config": {"workload": ("linear7b: LLaMA-7B layer, 7 QLoRA linears fwd+bwd, 4096 tokens (8x512), "
                                "r=64, alpha=16, bf16 activations") if args.linears == "llama7b" else
                               f"single QLoRA linear {args.linears} fwd+bwd, {TOKENS} tokens, r=64, alpha=16",
                   "tokens_per_gpu": TOKENS, "rank": R, "alpha": ALPHA, "l2": "flushed (256 MB write) before each step",
                   "parallelism": f"dp{world}", "flop_per_step_per_gpu": step_flops,
                   "adapter_products": ("split off to a low-priority side stream, beside the previous linear's "
                                        "fused GEMM" if split_headline else "inside each linear call, one stream")},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "roofline": roofline,
        "kernels": breakdown,
        "clocks": clocks,
    }
    if variants is not None:
        line["variants7b"] = variants
    if codec is not None:
        line["codec"] = codec
    if decode is not None:
        line["decode65b"] = decode
    if adamw is not None:
        line["adamw7b"] = adamw
    if blockr is not None:
        line["block7b"] = blockr
    if stack is not None:
        line["stack65b"] = stack
    if world == 1 and not args.skip_cpu:
        line["cpu_baseline"] = cpu_baseline_linear(budget_s=args.cpu_seconds)
        line["cpu_baseline_tiny"] = cpu_baseline_tiny()
    return line


def run_variants7b(args, q, torch, dev, layers, timed_steps, step_flops, tokens, scale, peaks, peak_src):
    """The headline's LLaMA-7B layer step (7 linears fwd+bwd, 4096 tokens) under
    the variant knobs, timed the same way: the fp16 compute dtype (fp16
    activations, adapters and outputs, fp16 expansion of the 4-bit weight) and
    LoRA dropout (p = 0.05, keep mask drawn once, bf16)."""
    import synthetic
    out = {"workload": "linear7b step (7 LLaMA-7B QLoRA linears fwd+bwd, 4096 tokens, r=64) with the variant knobs",
           "unit": "TFLOP/s"}
    steps = max(args.steps // 2, 3)
    # fp16 compute dtype: same quantized weights, fp16 tensors
    f16 = []
    for L in layers:
        f16.append({k: L[k].to(torch.float16) for k in ("X", "A", "B", "dY")})
        f16[-1].update(Y=torch.empty_like(L["Y"], dtype=torch.float16), dX=torch.empty_like(L["dX"], dtype=torch.float16))
    ws = torch.empty(max(q.qlora_linear_workspace_bytes(tokens, L["N"], L["K"], R) for L in layers),
                     dtype=torch.uint8, device=dev)

    def step_f16():
        for L, F in zip(layers, f16):
            q.qlora_linear_fwd(L["w"], F["X"], tokens, F["A"], F["B"], R, scale, F["Y"], L["H"], ws)
        for L, F in zip(reversed(layers), reversed(f16)):
            q.qlora_linear_bwd(L["w"], F["X"], F["dY"], tokens, F["A"], F["B"], R, scale, L["H"], F["dX"],
                               L["dA"], L["dB"], ws)

    for _ in range(3):
        step_f16()
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    ms = timed_steps(steps, step_f16)
    out["fp16_compute"] = {"value": round(step_flops * steps / (ms * 1e-3) / 1e12, 2),
                           "ms_per_step": round(ms / steps, 4), "frac_of_bf16_peak": None}
    out["fp16_compute"]["frac_of_bf16_peak"] = round(out["fp16_compute"]["value"] / peaks["bf16_tflops"], 4)
    del f16
    # LoRA dropout: one mask per linear (M*K/8 bytes)
    masks = [synthetic.dropout_mask(tokens, L["K"], 0.05, 90_000 + i, dev)[1] for i, L in enumerate(layers)]
    wsd = torch.empty(max(q.qlora_linear_workspace_bytes(tokens, L["N"], L["K"], R, dropout=(masks[0], 0.05))
                          for L in layers), dtype=torch.uint8, device=dev)

    def step_drop():
        for L, m in zip(layers, masks):
            q.qlora_linear_fwd(L["w"], L["X"], tokens, L["A"], L["B"], R, scale, L["Y"], L["H"], wsd,
                               dropout=(m, 0.05))
        for L, m in zip(reversed(layers), reversed(masks)):
            q.qlora_linear_bwd(L["w"], L["X"], L["dY"], tokens, L["A"], L["B"], R, scale, L["H"], L["dX"],
                               L["dA"], L["dB"], wsd, dropout=(m, 0.05))

    for _ in range(3):
        step_drop()
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    ms = timed_steps(steps, step_drop)
    out["lora_dropout_0.05"] = {"value": round(step_flops * steps / (ms * 1e-3) / 1e12, 2),
                                "ms_per_step": round(ms / steps, 4),
                                "note": "FLOP counted as without dropout (the dropped-input pass and the separate "
                                        "adapter dX product are extra work)"}
    out["peak_source"] = f"{peak_src} bf16_tflops (burst); fp16 dense peak taken equal to bf16"
    return out


def run_codec(args, q, torch, dev, peaks, peak_src):
    """NF4+DQ quantize -> dequantize round trip over the LLaMA-7B tensors,
    replayed as one CUDA graph per step (four streams of independent tensors)."""
    import synthetic
    shapes = [(N, K) for _ in range(synthetic.LLAMA7B_LAYERS) for _, N, K in synthetic.LLAMA7B_LINEARS]
    if args.codec_tensors:
        shapes = shapes[:args.codec_tensors]
    tensors = []
    for i, (N, K) in enumerate(shapes):
        W = synthetic.normal((N, K), 0.02, 50_000 + i, torch.bfloat16, dev)
        tensors.append((W, q.NF4Weight(N, K, device=dev), torch.empty(N, K, dtype=torch.bfloat16, device=dev)))
    nweights = sum(N * K for N, K in shapes)
    # the tensors are independent: they are spread over a few streams (one
    # quantize workspace each) so that one tensor's launch and tail overlap
    # another's streaming
    n_streams = args.codec_streams
    qws_bytes = max(q.qlora_quantize_workspace_bytes(N, K) for N, K in shapes)
    qws = [torch.empty(qws_bytes, dtype=torch.uint8, device=dev) for _ in range(n_streams)]
    side = [torch.cuda.Stream() for _ in range(n_streams)]

    def round_trip():
        main = torch.cuda.current_stream()
        for st in side:
            st.wait_stream(main)
        for i, (W, w, out) in enumerate(tensors):
            with torch.cuda.stream(side[i % n_streams]):
                q.qlora_quantize_nf4_dq(W, w, qws[i % n_streams])
                q.qlora_dequantize_nf4_dq(w, out)
        for st in side:
            main.wait_stream(st)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):
            round_trip()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        round_trip()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    # the tensors (13 GB in, 13 GB out) are far larger than L2: no flush needed
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    bytes_rt = 2 * CODEC_BYTES_PER_WEIGHT * nweights
    gbs = bytes_rt / (ms * 1e-3) / 1e9
    # per-kernel device time: the same work on one stream, each kernel bracketed
    # by CUDA events (the breakdown: brackets separate the kernels)
    q.qlora_timing_reset()
    q.qlora_timing_enable(True)
    torch.cuda._sleep(100_000_000)
    for i, (W, w, out) in enumerate(tensors):
        q.qlora_quantize_nf4_dq(W, w, qws[0])
        q.qlora_dequantize_nf4_dq(w, out)
    q.qlora_timing_enable(False)
    kern = q.qlora_timing_read()
    # per-call device time: each API call bracketed by CUDA events, its own
    # kernels chained as a user sees them (quantize = workspace reset, the
    # first-level pass and the double quantization of its constants, whose
    # E4M3 codes and scales are part of the 2.5159 B per weight)
    marks = []
    torch.cuda._sleep(100_000_000)
    for W, w, out in tensors:
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record()
        q.qlora_quantize_nf4_dq(W, w, qws[0])
        ev[1].record()
        q.qlora_dequantize_nf4_dq(w, out)
        ev[2].record()
        marks.append(ev)
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    qms = sum(ev[0].elapsed_time(ev[1]) for ev in marks)
    dms = sum(ev[1].elapsed_time(ev[2]) for ev in marks)
    qgbs = CODEC_BYTES_PER_WEIGHT * nweights / (qms * 1e-3) / 1e9
    dgbs = CODEC_BYTES_PER_WEIGHT * nweights / (dms * 1e-3) / 1e9
    big = [i for i, (N, K) in enumerate(shapes) if N * K == max(a * b for a, b in shapes)]
    big_us = sorted(marks[i][0].elapsed_time(marks[i][1]) * 1e3 for i in big)
    big_n = shapes[big[0]][0] * shapes[big[0]][1]
    dom = "quantize" if qms >= dms else "dequantize"
    ach = qgbs if dom == "quantize" else dgbs
    peak = peaks["hbm_gbs"]
    del g
    # end to end on one layer's 7 tensors: each weight copied in from pinned host
    # memory, quantized, dequantized, and the bf16 result copied back, over the
    # same four streams
    layer = tensors[:len(synthetic.LLAMA7B_LINEARS)]
    pin_in = [W.cpu().pin_memory() for W, _, _ in layer]
    pin_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _, _, out in layer]
    lw = sum(W.numel() for W, _, _ in layer)

    def e2e_step():
        main = torch.cuda.current_stream()
        for st in side:
            st.wait_stream(main)
        for i, ((W, w, out), hi, ho) in enumerate(zip(layer, pin_in, pin_out)):
            with torch.cuda.stream(side[i % n_streams]):
                W.copy_(hi, non_blocking=True)
                q.qlora_quantize_nf4_dq(W, w, qws[i % n_streams])
                q.qlora_dequantize_nf4_dq(w, out)
                ho.copy_(out, non_blocking=True)
        for st in side:
            main.wait_stream(st)

    e2e_step()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(args.steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    e2e = {"value": round(2 * CODEC_BYTES_PER_WEIGHT * lw / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
           "ms_per_layer": round(e2e_ms, 4), "h2d_bytes_per_step": 2 * lw, "d2h_bytes_per_step": 2 * lw,
           "workload": "one layer's 7 tensors: pinned host bf16 in, quantize, dequantize, pinned host bf16 out"}
    cpu = None if args.skip_cpu else cpu_baseline_codec(q, torch, tensors)
    return {
        "workload": "codec7b: NF4+DQ quantize->dequantize round trip, 224 LLaMA-7B tensors, "
                    f"{nweights} bf16 weights ~N(0,0.02), one CUDA graph per step",
        "value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 4),
        "weights_per_s": nweights / (ms * 1e-3),
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(ach / peak, 4), "traffic": measured_traffic("codec", dom),
                     "peak_source": f"{peak_src} hbm_gbs"},
        "kernels": {"quantize_gbs": round(qgbs, 1), "dequantize_gbs": round(dgbs, 1),
                    "quantize_ms": round(qms, 4), "dequantize_ms": round(dms, 4),
                    "quantize_largest_tensor": {"shape": list(shapes[big[0]]), "us_median": round(big_us[len(big_us) // 2], 2),
                                                "gbs": round(CODEC_BYTES_PER_WEIGHT * big_n / (big_us[len(big_us) // 2] * 1e-6) / 1e9, 1)},
                    "per_kernel_ms_bracketed": {"quantize_blocks": round(kern["quantize"][0], 4),
                                                "dq_encode": round(kern["dq_encode"][0], 4),
                                                "dequantize": round(kern["dequantize"][0], 4)},
                    "note": "quantize_ms / dequantize_ms: each API call bracketed by CUDA events on one stream "
                            "(quantize = workspace reset + first-level pass + double quantization); "
                            "per_kernel_ms_bracketed: every kernel bracketed separately (no overlap)"},
        "e2e": e2e,
        "cpu_baseline": cpu,
    }


def weight_bytes(N, K):
    """Bytes of one quantized weight: packed codes, E4M3 block codes, group scales."""
    nblocks = N * K // 64
    return N * K // 2 + nblocks + 4 * (-(-nblocks // 256))


def run_decode65b(args, q, torch, dev, peaks, peak_src):
    """Decode-shaped forward of the seven LLaMA-65B linears at 1, 4 and 16
    tokens: every call streams its packed weight from HBM once.  One step is
    the seven linears; the 437 MB of weights per step exceed L2, so nothing
    needs flushing."""
    import synthetic
    shapes = synthetic.LLAMA65B_LINEARS
    qws = torch.empty(max(q.qlora_quantize_workspace_bytes(N, K) for _, N, K in shapes), dtype=torch.uint8,
                      device=dev)
    layers = []
    for i, (name, N, K) in enumerate(shapes):
        W = synthetic.normal((N, K), 0.02, 70_000 + i, torch.bfloat16, dev)
        w = q.NF4Weight(N, K, device=dev)
        q.qlora_quantize_nf4_dq(W, w, qws)
        del W
        layers.append({"N": N, "K": K, "w": w,
                       "A": synthetic.normal((R, K), 1.0 / R, 70_100 + i, torch.bfloat16, dev),
                       "B": synthetic.normal((N, R), 0.01, 70_200 + i, torch.bfloat16, dev)})
    del qws
    scale = ALPHA / R
    out = {"workload": "decode65b: forward of the 7 LLaMA-65B linears (8192x8192 x4, 22016x8192 x2, 8192x22016), "
                       "r=64, bf16 activations, tokens 1/4/16", "unit": "GB/s", "tokens": {}}
    if not args.skip_cpu:
        L0 = layers[0]
        X1 = synthetic.normal((1, L0["K"]), 1.0, 70_301, torch.bfloat16, dev)
        out["cpu_baseline"] = cpu_baseline_decode(q, torch, L0["w"], X1, L0["A"], L0["B"], 1)
    for M in (1, 4, 16):
        ws = torch.empty(max(q.qlora_linear_workspace_bytes(M, L["N"], L["K"], R) for L in layers),
                         dtype=torch.uint8, device=dev)
        for L in layers:
            L["X"] = synthetic.normal((M, L["K"]), 1.0, 70_300 + M, torch.bfloat16, dev)
            L["Y"] = torch.empty(M, L["N"], dtype=torch.bfloat16, device=dev)

        def step():
            for L in layers:
                q.qlora_linear_fwd(L["w"], L["X"], M, L["A"], L["B"], R, scale, L["Y"], None, ws)

        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize()
        q.qlora_check_device_error()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(args.steps, 10)
        torch.cuda._sleep(20_000_000)
        e0.record()
        for _ in range(reps):
            step()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        # algorithmic bytes: quantized weights, adapters, activations in and out
        nbytes = sum(weight_bytes(L["N"], L["K"]) + 2 * R * (L["N"] + L["K"]) + 2 * M * (L["N"] + L["K"])
                     for L in layers)
        q.qlora_timing_reset()
        q.qlora_timing_enable(True)
        torch.cuda._sleep(20_000_000)
        for _ in range(reps):
            step()
        q.qlora_timing_enable(False)
        kern = q.qlora_timing_read()
        q.qlora_check_device_error()
        gemv_ms = kern["fwd_fused"][0] / reps
        gemv_bytes = sum(weight_bytes(L["N"], L["K"]) + 2 * R * L["K"] + 2 * M * L["K"] + 4 * M * L["N"]
                         for L in layers)
        gbs = nbytes / (ms * 1e-3) / 1e9
        ach = gemv_bytes / (gemv_ms * 1e-3) / 1e9
        # end to end: every linear's X from pinned host memory, Y back to pinned host memory
        pin_x = [L["X"].cpu().pin_memory() for L in layers]
        pin_y = [torch.empty(L["Y"].shape, dtype=L["Y"].dtype).pin_memory() for L in layers]

        def e2e_step():
            for L, hx, hy in zip(layers, pin_x, pin_y):
                L["X"].copy_(hx, non_blocking=True)
                q.qlora_linear_fwd(L["w"], L["X"], M, L["A"], L["B"], R, scale, L["Y"], None, ws)
                hy.copy_(L["Y"], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        torch.cuda._sleep(20_000_000)
        e0.record()
        for _ in range(reps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / reps
        out["tokens"][str(M)] = {
            "value": round(gbs, 1), "us_per_layer": round(ms * 1e3, 2), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "e2e": {"value": round(nbytes / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s", "us_per_layer": round(e2e_ms * 1e3, 2),
                    "h2d_bytes_per_step": sum(2 * M * L["K"] for L in layers),
                    "d2h_bytes_per_step": sum(2 * M * L["N"] for L in layers)},
            "roofline": {"kernel": "decode_gemv", "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": None,
                         "peak_source": f"{peak_src} hbm_gbs"},
            "kernels_us": {k: round(v[0] / reps * 1e3, 2) for k, v in kern.items() if v[1]},
        }
    return out


def run_stack65b(args, q, torch, dev, peaks, peak_src, layers_n=None, tokens=2048):
    """Forward then backward through a stack of 80 LLaMA-65B layers of 7 QLoRA
    linears each (no attention) at 2048 tokens.  Every linear has its own
    quantized weight buffers (about 33 GB in all), adapters and gradients;
    the seven quantized weights of one layer are generated and copied into
    the other layers' buffers (same values, distinct memory), and the
    activation buffers are shared per shape."""
    import synthetic
    shapes = synthetic.LLAMA65B_LINEARS
    n_layers = layers_n or synthetic.LLAMA65B_LAYERS
    qws = torch.empty(max(q.qlora_quantize_workspace_bytes(N, K) for _, N, K in shapes), dtype=torch.uint8,
                      device=dev)
    proto = []
    for i, (name, N, K) in enumerate(shapes):
        W = synthetic.normal((N, K), 0.02, 80_000 + i, torch.bfloat16, dev)
        w = q.NF4Weight(N, K, device=dev)
        q.qlora_quantize_nf4_dq(W, w, qws)
        del W
        proto.append(w)
    del qws
    act = {}
    for _, N, K in shapes:
        act.setdefault(("X", K), synthetic.normal((tokens, K), 1.0, 80_100 + K, torch.bfloat16, dev))
        act.setdefault(("dY", N), synthetic.normal((tokens, N), 1.0, 80_200 + N, torch.bfloat16, dev))
        act.setdefault(("Y", N), torch.empty(tokens, N, dtype=torch.bfloat16, device=dev))
        act.setdefault(("dX", K), torch.empty(tokens, K, dtype=torch.bfloat16, device=dev))
    lin = []
    for layer in range(n_layers):
        for i, (name, N, K) in enumerate(shapes):
            w = q.NF4Weight(N, K, codebook=proto[i].codebook, device=dev)
            for dst, src in ((w.packed, proto[i].packed), (w.code2, proto[i].code2), (w.c2, proto[i].c2),
                             (w.mean, proto[i].mean)):
                dst.copy_(src)
            lin.append({"N": N, "K": K, "w": w,
                        "A": synthetic.normal((R, K), 1.0 / R, 80_300 + i, torch.bfloat16, dev),
                        "B": synthetic.normal((N, R), 0.01, 80_400 + i, torch.bfloat16, dev),
                        "H": torch.empty(tokens, R, dtype=torch.float32, device=dev),
                        "dA": torch.empty(R, K, dtype=torch.float32, device=dev),
                        "dB": torch.empty(N, R, dtype=torch.float32, device=dev)})
    del proto
    wbytes = sum(L["w"].nbytes for L in lin)
    ws = torch.empty(max(q.qlora_linear_workspace_bytes(tokens, N, K, R) for _, N, K in shapes), dtype=torch.uint8,
                     device=dev)
    scale = ALPHA / R

    def step():
        for L in lin:
            q.qlora_linear_fwd(L["w"], act[("X", L["K"])], tokens, L["A"], L["B"], R, scale, act[("Y", L["N"])],
                               L["H"], ws)
        for L in reversed(lin):
            q.qlora_linear_bwd(L["w"], act[("X", L["K"])], act[("dY", L["N"])], tokens, L["A"], L["B"], R, scale,
                               L["H"], act[("dX", L["K"])], L["dA"], L["dB"], ws)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    steps = max(1, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = q.qlora_launch_count()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    launches = q.qlora_launch_count() - launches0
    q.qlora_check_device_error()
    ms = e0.elapsed_time(e1) / steps
    flops = sum(linear_flops(tokens, L["N"], L["K"], R) for L in lin)
    value = flops / (ms * 1e-3) / 1e12
    # end to end: the stack's input activation and output gradient come from
    # pinned host memory each step, and the gradients of the first linear (the
    # last ones the backward writes) go back to pinned host memory
    x0, dy0 = act[("X", lin[0]["K"])], act[("dY", lin[-1]["N"])]
    hx, hdy = x0.cpu().pin_memory(), dy0.cpu().pin_memory()
    hda = torch.empty(lin[0]["dA"].shape, dtype=torch.float32).pin_memory()
    hdb = torch.empty(lin[0]["dB"].shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        x0.copy_(hx, non_blocking=True)
        dy0.copy_(hdy, non_blocking=True)
        step()
        hda.copy_(lin[0]["dA"], non_blocking=True)
        hdb.copy_(lin[0]["dB"], non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / steps
    e2e = {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 3),
           "h2d_bytes_per_step": 2 * (x0.numel() + dy0.numel()),
           "d2h_bytes_per_step": 4 * (lin[0]["dA"].numel() + lin[0]["dB"].numel())}
    return {
        "workload": f"stack65b: {n_layers} LLaMA-65B layers x 7 QLoRA linears fwd+bwd, {tokens} tokens, r=64, "
                    "alpha=16, no attention",
        "value": round(value, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 3), "steps": steps,
        "flop_per_step": flops, "nf4_weight_gb": round(wbytes / 1e9, 2),
        # a step lasts about half a second at the power limit: the sustained peak applies
        "roofline": {"bound": "tensor", "achieved": round(value, 1), "peak": peaks["bf16_tflops_sustained"],
                     "unit": "TFLOP/s", "frac": round(value / peaks["bf16_tflops_sustained"], 4),
                     "frac_of_burst_peak": round(value / peaks["bf16_tflops"], 4), "traffic": None,
                     "peak_source": f"{peak_src} bf16_tflops_sustained"},
        "gpu_launches_per_step": launches // steps,
        "clocks": clk.summary(),
        "e2e": e2e,
        "cpu_baseline": None if args.skip_cpu else cpu_baseline_stack(),
    }


def run_adamw7b(args, q, torch, dev, peaks, peak_src):
    """Paged AdamW over every LoRA adapter of a 32-layer LLaMA-7B (r = 64: the
    A and B of the seven linears of each layer, flattened), with the moments m
    and v in unified memory.  Timed twice: with the state resident on the GPU
    (the roofline: 30 bytes per parameter), and after evicting the state to
    host memory, so that the update pages it back on demand."""
    import synthetic
    n = synthetic.LLAMA7B_LAYERS * sum(R * (N + K) for _, N, K in synthetic.LLAMA7B_LINEARS)
    p = synthetic.normal((n,), 0.02, 90_001, torch.float32, dev)
    p16 = torch.empty(n, dtype=torch.bfloat16, device=dev)
    g = synthetic.normal((n,), 1e-3, 90_002, torch.float32, dev)
    m, v = q.PagedBuffer(n), q.PagedBuffer(n)
    hp = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0)
    step_no = [0]

    def step():
        step_no[0] += 1
        q.qlora_adamw_step(p, p16, g, m.tensor, v.tensor, hp["lr"], hp["beta1"], hp["beta2"], hp["eps"],
                           hp["weight_decay"], step_no[0])

    for b in (m, v):
        q.qlora_paged_prefetch(b, to_device=True)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    reps = max(args.steps, 10)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms_res = e0.elapsed_time(e1) / reps
    bytes_per_step = 30 * n
    gbs = bytes_per_step / (ms_res * 1e-3) / 1e9
    # evicted state: every step first pushes m and v out to the host, then the
    # update faults them back (timed: the update alone, and prefetch + update)
    paged_ms, prefetch_ms = [], []
    for mode in ("demand", "prefetch"):
        for _ in range(3):
            for b in (m, v):
                q.qlora_paged_prefetch(b, to_device=False)
            torch.cuda.synchronize()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            if mode == "prefetch":
                for b in (m, v):
                    q.qlora_paged_prefetch(b, to_device=True)
            step()
            a1.record()
            torch.cuda.synchronize()
            (paged_ms if mode == "demand" else prefetch_ms).append(a0.elapsed_time(a1))
    q.qlora_check_device_error()
    state_bytes = m.nbytes + v.nbytes
    m.free()
    v.free()
    return {
        "workload": f"adamw7b: AdamW over the LoRA adapters of 32 LLaMA-7B layers (r=64), {n} parameters, "
                    "m and v in unified (paged) memory",
        "value": round(gbs, 1), "unit": "GB/s", "ms_per_step_resident": round(ms_res, 4),
        "params": n, "bytes_per_param": 30, "paged_state_bytes": state_bytes,
        "ms_per_step_after_eviction": {"demand_paging": round(sorted(paged_ms)[1], 3),
                                       "prefetch_then_update": round(sorted(prefetch_ms)[1], 3)},
        "roofline": {"kernel": "adamw", "bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None,
                     "peak_source": f"{peak_src} hbm_gbs"},
    }


def run_block7b(args, q, torch, dev, peaks, peak_src, batch=8, seq=512):
    """One LLaMA-7B transformer block (hidden 4096, 32 heads of 128, inter
    11008) with QLoRA adapters (r = 64, alpha = 16) on all seven linears, at
    4096 tokens (8 x 512): the forward pass (checkpointed: only the output is
    kept) and the backward pass (recompute, then gradients of x and of the 14
    adapter matrices).  FLOP are counted as the model's: every linear's
    4MNK + 6Mr(N+K) and the attention products 12 B H S^2 D (dense count);
    the recomputed forward is extra work the count leaves out."""
    import synthetic
    hidden, heads, inter = 4096, 32, 11008
    case = synthetic.block_case(batch, seq, hidden, heads, inter, R, ALPHA, seed=95_000, device=dev)
    weights = []
    qws = torch.empty(q.qlora_quantize_workspace_bytes(inter, hidden), dtype=torch.uint8, device=dev)
    for W in case["W"]:
        w = q.NF4Weight(*W.shape, device=dev)
        q.qlora_quantize_nf4_dq(W, w, qws)
        weights.append(w)
    del qws, case["W"]
    blk = q.Block(batch, seq, hidden, heads, inter, R, ALPHA / R, weights, case["A"], case["B"],
                  case["norm1"], case["norm2"])
    ws = torch.empty(q.qlora_block_workspace_bytes(blk), dtype=torch.uint8, device=dev)
    T = batch * seq
    x, dy = case["x"], case["dy"]
    y = torch.empty(T, hidden, dtype=torch.bfloat16, device=dev)
    dx = torch.empty_like(y)
    dA = [torch.empty(R, w.cols, dtype=torch.float32, device=dev) for w in weights]
    dB = [torch.empty(w.rows, R, dtype=torch.float32, device=dev) for w in weights]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        q.qlora_block_fwd(blk, x, y, ws)
        q.qlora_block_bwd(blk, x, dy, dx, dA, dB, ws)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    steps = max(1, min(args.steps, 10))
    total = 0.0
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(steps):
            flush.zero_()
            torch.cuda.synchronize()
            torch.cuda._sleep(20_000_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            step()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
    q.qlora_check_device_error()
    ms = total / steps
    lin = sum(linear_flops(T, w.rows, w.cols, R) for w in weights)
    att = 12 * batch * heads * seq * seq * (hidden // heads)
    recompute = sum(2 * T * w.rows * w.cols + 2 * T * R * (w.rows + w.cols) for w in weights[:6]) + att // 3
    model = lin + att
    value = model / (ms * 1e-3) / 1e12
    # per-kind device time of one step, every launch bracketed by events
    q.qlora_timing_reset()
    q.qlora_timing_enable(True)
    step()
    q.qlora_timing_enable(False)
    kern = q.qlora_timing_read()
    return {
        "workload": f"block7b: one LLaMA-7B block (QLoRA on q,k,v,o,gate,up,down; RMSNorm, RoPE, causal attention, "
                    f"SwiGLU), checkpointed forward + backward, {T} tokens ({batch}x{seq}), r=64, alpha=16",
        "value": round(value, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
        "model_flop_per_step": model, "hardware_flop_per_step": model + recompute,
        "hardware_tflops": round((model + recompute) / (ms * 1e-3) / 1e12, 2),
        "roofline": {"bound": "tensor", "achieved": round(value, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(value / peaks["bf16_tflops"], 4), "traffic": None,
                     "peak_source": f"{peak_src} bf16_tflops (burst); achieved counts model FLOP"},
        "kernels_ms_bracketed": {k: round(v[0], 4) for k, v in kern.items() if v[1]},
        "clocks": clk.summary(),
    }


# ---- CPU baselines (the oracle, as it stands) ---------------------------------------

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline_linear(budget_s=15.0):
    """Oracle fwd+bwd of one 4096x4096 QLoRA linear on a token sample sized
    to about `budget_s` seconds of host time."""
    import numpy as np

    import synthetic
    from oracle import linear as olin
    N = K = 4096
    case = synthetic.linear_case(64, N, K, R, ALPHA, seed=7)
    Wd = case["W"].float().numpy().astype(np.float64)   # raw N(0, 0.02) weight: the same arithmetic as a dequantized one
    A = case["A"].float().numpy()
    B = case["B"].float().numpy()
    rng = np.random.default_rng(0)
    M = 64
    spent, flops = 0.0, 0.0
    while spent < budget_s:
        X = rng.standard_normal((M, K))
        dY = rng.standard_normal((M, N))
        t0 = time.perf_counter()
        olin.forward(X, Wd, A, B, ALPHA / R)
        olin.backward(X, Wd, A, B, ALPHA / R, dY)
        dt = time.perf_counter() - t0
        spent += dt
        flops += linear_flops(M, N, K, R)
        if dt < budget_s / 8 and M < 8192:
            M *= 2
    return {"value": round(flops / spent / 1e12, 5), "unit": "TFLOP/s", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"oracle float64 fwd+bwd of one 4096x4096 linear (r=64; the raw N(0,0.02) weight stands "
                      f"for the dequantized one), token batches up to {M}, {spent:.1f} s of host time"}


def _omp_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline_codec(q, torch, tensors, budget_s=10.0):
    """Oracle codec (C loops, OpenMP) on the host: quantize + dequantize of
    one tensor of each LLaMA-7B shape in the round trip, inputs copied from
    the device, outputs compared bit for bit with the device's."""
    import numpy as np

    from oracle import codebook as ocb
    from oracle import codec as occ
    Q = ocb.nf4_codebook()
    seen, spent, nweights, exact = set(), 0.0, 0, True
    for W, w, out in tensors:
        shape = tuple(W.shape)
        if shape in seen or spent > budget_s:
            continue
        seen.add(shape)
        Wh = W.float().cpu().numpy()
        t0 = time.perf_counter()
        ref = occ.quantize(Wh, Q)
        deq = occ.dequantize(ref["packed"], ref["e"], ref["c2"], ref["mean"], Q)
        spent += time.perf_counter() - t0
        nweights += Wh.size
        exact &= bool(np.array_equal(w.packed.cpu().numpy(), ref["packed"]))
        exact &= bool(np.array_equal(w.code2.cpu().numpy(), ref["e"]))
        exact &= bool(np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16).ravel(), deq))
    return {"value": round(2 * CODEC_BYTES_PER_WEIGHT * nweights / spent / 1e9, 3), "unit": "GB/s",
            "cores": _omp_threads(), "kind": "oracle", "bit_exact_vs_device": exact,
            "sample": f"oracle quantize + dequantize of one tensor of each shape {sorted(seen)} "
                      f"({nweights} weights, {spent:.1f} s of host time)"}


def cpu_baseline_decode(q, torch, w, X, A, B, M):
    """Oracle decode forward of one LLaMA-65B 8192x8192 linear at M tokens:
    dequantize (C loops) then the float64 layer (numpy)."""
    import numpy as np

    from oracle import codec as occ
    from oracle import linear as olin
    Q = np.asarray(w.codebook, np.float32)
    packed, e, c2 = w.packed.cpu().numpy(), w.code2.cpu().numpy(), w.c2.cpu().numpy()
    mean = np.float32(w.mean[0].item())
    Xh, Ah, Bh = (t.float().cpu().numpy().astype(np.float64) for t in (X, A, B))
    t0 = time.perf_counter()
    Wd = occ.bf16_bits_to_f32(occ.dequantize(packed, e, c2, mean, Q)).reshape(w.rows, w.cols).astype(np.float64)
    olin.forward(Xh, Wd, Ah, Bh, ALPHA / R)
    dt = time.perf_counter() - t0
    nbytes = weight_bytes(w.rows, w.cols) + 2 * R * (w.rows + w.cols) + 2 * M * (w.rows + w.cols)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"oracle dequantize + float64 forward of one 8192x8192 linear at {M} token(s), "
                      f"{dt:.2f} s of host time"}


def cpu_baseline_stack(budget_s=10.0):
    """Oracle fwd+bwd of one LLaMA-65B 8192x8192 linear (r = 64) on a token
    sample of the stack's 2048 tokens; TFLOP/s, the rate one stack layer
    would run at."""
    import numpy as np

    import synthetic
    from oracle import linear as olin
    N = K = 8192
    case = synthetic.linear_case(16, N, K, R, ALPHA, seed=8)
    Wd = case["W"].float().numpy().astype(np.float64)   # raw N(0, 0.02) weight: the same arithmetic as a dequantized one
    A, B = case["A"].float().numpy(), case["B"].float().numpy()
    rng = np.random.default_rng(1)
    M, spent, flops = 32, 0.0, 0.0
    while spent < budget_s:
        X, dY = rng.standard_normal((M, K)), rng.standard_normal((M, N))
        t0 = time.perf_counter()
        olin.forward(X, Wd, A, B, ALPHA / R)
        olin.backward(X, Wd, A, B, ALPHA / R, dY)
        dt = time.perf_counter() - t0
        spent += dt
        flops += linear_flops(M, N, K, R)
        if dt < budget_s / 8 and M < 2048:
            M *= 2
    return {"value": round(flops / spent / 1e12, 5), "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"oracle float64 fwd+bwd of one 8192x8192 linear (r=64), token batches up to {M} of 2048, "
                      f"{spent:.1f} s of host time"}


def cpu_baseline_tiny():
    """Oracle on the tiny configuration (W 256x256, 16 tokens, r = 8): codec
    and linear fwd+bwd, timed on one core and on all cores."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import synthetic
    from oracle import codebook as ocb
    from oracle import codec as occ
    from oracle import linear as olin
    c = synthetic.tiny_linear(seed=0)
    Q = ocb.nf4_codebook()
    W = c["W"].numpy()
    X, A, B, dY = (c[k].float().numpy().astype(np.float64) for k in ("X", "A", "B", "dY"))

    def once():
        ref = occ.quantize(W, Q)
        Wd = occ.bf16_bits_to_f32(occ.dequantize(ref["packed"], ref["e"], ref["c2"], ref["mean"], Q))
        Wd = Wd.reshape(W.shape).astype(np.float64)
        olin.forward(X, Wd, A, B, c["scale"])
        olin.backward(X, Wd, A, B, c["scale"], dY)

    out = {}
    for label, n in (("1_core", 1), ("all_cores", _blas_threads())):
        with threadpool_limits(limits=n):
            os.environ["OMP_NUM_THREADS"] = str(n)
            once()
            reps, t0 = 0, time.perf_counter()
            while time.perf_counter() - t0 < 1.0:
                once()
                reps += 1
            out[label] = {"ms_per_call": round((time.perf_counter() - t0) / reps * 1e3, 3), "cores": n}
    os.environ.pop("OMP_NUM_THREADS", None)
    return {"kind": "oracle", "unit": "ms per quantize + dequantize + linear fwd+bwd", **out,
            "sample": "the whole tiny configuration, repeated for 1 s"}


def run_reference(args, rank, world):
    """The reference arm: the oracle, timed on the host cores, same metric."""
    if rank != 0:
        return None
    import numpy as np

    import synthetic
    from oracle import linear as olin
    Ms = args.tokens   # the full workload: every token of each linear, every step (about 3 s per step)
    rng = np.random.default_rng(0)
    mats = []
    for i, (name, N, K) in enumerate(synthetic.LLAMA7B_LINEARS):
        Wd = rng.standard_normal((N, K)) * 0.02
        mats.append((N, K, Wd, rng.standard_normal((R, K)) / R, rng.standard_normal((N, R)) * 0.01))
    X = {K: rng.standard_normal((Ms, K)) for K in (4096, 11008)}
    dY = {N: rng.standard_normal((Ms, N)) for N in (4096, 11008)}

    def step():
        for N, K, Wd, A, B in mats:
            olin.forward(X[K], Wd, A, B, ALPHA / R)
            olin.backward(X[K], Wd, A, B, ALPHA / R, dY[N])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    flops = sum(linear_flops(Ms, N, K, R) for N, K, *_ in mats) * args.steps
    value = flops / dt / 1e12
    cores = _blas_threads()
    sample = f"oracle float64 fwd+bwd of the 7 LLaMA-7B linears on all {Ms} tokens per step (the full workload)"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": "linear7b: LLaMA-7B layer, 7 QLoRA linears fwd+bwd, "
                                                    "4096 tokens (8x512), r=64, alpha=16, bf16 activations"
                                        if Ms == 4096 else f"7 LLaMA-7B QLoRA linears fwd+bwd, {Ms} tokens, r=64, alpha=16",
                                        "tokens_per_gpu": Ms, "rank": R, "alpha": ALPHA, "parallelism": f"dp{world}"},
        "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_codec_shape(args, q, torch, dev):
    """Quantize and dequantize one N(0, 0.02) bf16 tensor of the shape given by
    --codec-shape NxK: `warmup` untimed calls, then `steps` calls of each, every
    call after an L2 flush and bracketed by CUDA events (a per-shape view of the
    codec, small enough for a full ncu capture)."""
    import synthetic
    N, K = (int(v) for v in args.codec_shape.lower().split("x"))
    W = synthetic.normal((N, K), 0.02, 77, torch.bfloat16, dev)
    w = q.NF4Weight(N, K, device=dev)
    ws = torch.empty(q.qlora_quantize_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
    out = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2
    for _ in range(args.warmup):
        q.qlora_quantize_nf4_dq(W, w, ws)
        q.qlora_dequantize_nf4_dq(w, out)
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    times = {"quantize": [], "dequantize": []}
    for _ in range(args.steps):
        for kind in ("quantize", "dequantize"):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            if kind == "quantize":
                q.qlora_quantize_nf4_dq(W, w, ws)
            else:
                q.qlora_dequantize_nf4_dq(w, out)
            e1.record()
            torch.cuda.synchronize()
            times[kind].append(e0.elapsed_time(e1) * 1e3)
    q.qlora_check_device_error()
    res = {"workload": f"codec shape {N}x{K}: one bf16 tensor ~N(0,0.02), L2 flushed before each call",
           "unit": "GB/s", "bytes_per_weight": CODEC_BYTES_PER_WEIGHT}
    for kind, ts in times.items():
        us = sorted(ts)[len(ts) // 2]
        res[kind] = {"us_median": round(us, 2), "value": round(CODEC_BYTES_PER_WEIGHT * N * K / (us * 1e-6) / 1e9, 1)}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-codec", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--no-adapter-split", action="store_true",
                    help="linear7b step: undivided linear calls on one stream (no side stream for H and G)")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-stack", action="store_true")
    ap.add_argument("--skip-optim", action="store_true")
    ap.add_argument("--skip-block", action="store_true")
    ap.add_argument("--skip-variants", action="store_true")
    ap.add_argument("--block-only", action="store_true", help="run only the transformer-block object (profiling runs)")
    ap.add_argument("--optim-only", action="store_true", help="run only the paged AdamW object (profiling runs)")
    ap.add_argument("--decode-only", action="store_true", help="run only the decode-shaped forward (profiling runs)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--linears", default="llama7b",
                    help="llama7b (the seven linears of one layer) or NxK for one linear (profiling runs)")
    ap.add_argument("--tokens", type=int, default=TOKENS)
    ap.add_argument("--codec-tensors", type=int, default=0,
                    help="limit the codec round trip to the first N LLaMA-7B tensors (profiling runs)")
    ap.add_argument("--codec-only", action="store_true", help="run only the codec round trip (profiling runs)")
    ap.add_argument("--codec-streams", type=int, default=4, help="streams the independent codec tensors spread over")
    ap.add_argument("--codec-shape", default=None,
                    help="NxK: time quantize and dequantize of one tensor of this shape only (profiling runs)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.codec_shape:
            import bit_nf4_quantized_16_b200 as q
            torch.cuda.set_device(local_rank)
            line = {"impl": "ours", "codec_shape": run_codec_shape(args, q, torch, torch.device("cuda", local_rank))}
        elif args.block_only:
            import bit_nf4_quantized_16_b200 as q
            torch.cuda.set_device(local_rank)
            peaks, src = load_peaks()
            line = {"impl": "ours", "block7b": run_block7b(args, q, torch, torch.device("cuda", local_rank), peaks, src)}
        elif args.decode_only:
            import bit_nf4_quantized_16_b200 as q
            torch.cuda.set_device(local_rank)
            peaks, src = load_peaks()
            line = {"impl": "ours",
                    "decode65b": run_decode65b(args, q, torch, torch.device("cuda", local_rank), peaks, src)}
        elif args.optim_only:
            import bit_nf4_quantized_16_b200 as q
            torch.cuda.set_device(local_rank)
            peaks, src = load_peaks()
            line = {"impl": "ours", "adamw7b": run_adamw7b(args, q, torch, torch.device("cuda", local_rank), peaks, src)}
        elif args.codec_only:
            import bit_nf4_quantized_16_b200 as q
            torch.cuda.set_device(local_rank)
            peaks, src = load_peaks()
            line = {"impl": "ours", "codec": run_codec(args, q, torch, torch.device("cuda", local_rank), peaks, src)}
        else:
            line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
