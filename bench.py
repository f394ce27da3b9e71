"""Benchmark of the BitLinear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|hbitlinear|tiny]
                    [--impl ours|reference]

One step = one BitLinear forward over one batch: the activation quantiser
(RMSNorm + absmax int8, or RMSNorm + Hadamard + int4) and the ternary product
with its dequantisation.  Weights are quantised offline, outside the timed
region.  The default workload is the decode GEMV: X bf16 [16, 2560],
W ternary [6912, 2560].  Rank 0 prints one JSON line.

Device timing: the K timed steps are captured in one CUDA graph and replayed
between CUDA events on the launching stream, with a barrier and a device
synchronise on both sides; each step reads the next of a ring of weight copies
whose total size exceeds twice the 126 MB L2.  The dominant kernel is timed the
same way on its own for the roofline.  e2e: the same steps through the Python
API with pinned host input/output buffers, the host<->device copies inside the
timed region.  The CPU oracle is timed on a bounded sample on the host.

Under torchrun (N > 1) each rank runs its own batches (independent tokens:
weak scaling, no data-path collective); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bitlinear_bitnet_quant_b200 import workloads as wl  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "BitLinear tokens/sec and GB/s|TOPS vs HBM/int8 roofline, 1xB200"


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

WORKLOADS = {
    "decode": lambda: wl.decode(16, with_weights=False),
    "decode_m4": lambda: wl.decode(4, with_weights=False),
    "decode_m1": lambda: wl.decode(1, with_weights=False),
    "prefill": lambda: wl.prefill(with_weights=False),
    "hbitlinear": lambda: wl.hbitlinear(with_weights=False),
    "tiny": lambda: wl.tiny(),
}
CHAIN_WORKLOADS = {"chain_decode": 32, "chain_prefill": 512}    # tokens per step
CHAIN_LAYERS = 24


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bitlinear_bitnet_quant_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(kernel_tag: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("kernel_source_hash") != kernel_source_hash():
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=2)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=1)
        sm, mx, reasons = [], 0.0, set()
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------

def max_over_ranks(ms: float, world: int, dev) -> float:
    """The slowest rank's time (every rank takes this collective step)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed_replay(g, stream, world, dev) -> float:
    """One warm replay, then a timed replay between CUDA events on the
    launching stream, with a barrier and a device synchronise on both sides."""
    import torch
    import torch.distributed as dist
    g.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1), world, dev)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from bitlinear_bitnet_quant_b200 import api, build_lib

    build_lib.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    c = WORKLOADS[args.workload]()
    M, K, N, bits = c["M"], c["K"], c["N"], c["act_bits"]
    eps = 1e-6
    out_dtype = torch.bfloat16 if args.workload == "prefill" else torch.float32
    out_bytes = 2 if out_dtype == torch.bfloat16 else 4

    # ---- weights: quantised offline, a ring of copies larger than 2x L2 ----
    packed_bytes = N * K // 4
    copies = max(2, min(64, math.ceil(2.2 * L2_BYTES / packed_bytes)))
    rng = np.random.default_rng(1234 + rank)
    base_w = torch.from_numpy(wl.weights(N, K, seed=rank)).to(dev)
    ring = []
    for i in range(copies):
        w = base_w if i == 0 else base_w[torch.from_numpy(rng.permutation(N)).to(dev)]
        pk, s_w = api.bitnet_quantize_weights(w.contiguous())
        ring.append((pk, s_w))
    del base_w
    torch.cuda.synchronize()

    x_host = c["x"]
    if c["x_dtype"] == "bf16":
        x = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        x = torch.from_numpy(x_host).to(dev)
    # preallocated outputs (the graph reuses them)
    if bits == 8:
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    else:
        xq = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    s_x = torch.empty((M,), dtype=torch.float32, device=dev)
    Y = torch.empty((M, N), dtype=out_dtype, device=dev)

    def quant():
        if bits == 8:
            api.bitnet_quant_act(x, None, eps, Xq=xq, s_x=s_x, stream=stream)
        else:
            api.bitnet_hadamard_quant_act(x, None, eps, c.get("had_block", 0), Xq4=xq, s_x=s_x, stream=stream)

    def linear(i):
        pk, s_w = ring[i % copies]
        api.bitnet_linear(xq, bits, s_x, pk, s_w, Y=Y, stream=stream)

    # the step is the quantiser and the linear kernel (the single-kernel path
    # of bitnet_bitlinear is slower on B200; the decode sweep reports it)
    def step(i):
        quant()
        linear(i)

    warmup = max(3, args.warmup)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()

    def graph_of(fn, count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(count):
                fn(i)
        return g

    def timed(g):
        return timed_replay(g, stream, world, dev)

    steps = args.steps
    g_step = graph_of(step, steps)
    g_lin = graph_of(linear, steps)
    g_q = graph_of(lambda i: quant(), steps)

    visible = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    clocks = ClockSampler(visible[local_rank] if local_rank < len(visible) else str(local_rank))
    clocks.start()
    t_step = timed(g_step)
    t_lin = timed(g_lin)
    t_q = timed(g_q)
    clk = clocks.stop()

    # ---- e2e through the public API with pinned host buffers ----
    x_pin = torch.empty_like(x, device="cpu").pin_memory()
    x_pin.copy_(x.cpu())
    y_pin = torch.empty((M, N), dtype=out_dtype).pin_memory()
    h2d = x_pin.numel() * x_pin.element_size()
    d2h = y_pin.numel() * y_pin.element_size()

    def e2e_step(i):
        x.copy_(x_pin, non_blocking=True)
        pk, s_w = ring[i % copies]
        Yo = api.bitlinear_forward(x, pk, s_w, act_bits=bits, eps=eps, had_block=c.get("had_block", 0),
                                   out_dtype=out_dtype, Y=Y, Xq=xq, s_x=s_x, stream=stream)
        y_pin.copy_(Yo, non_blocking=True)

    for i in range(warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev)

    # the offline weight path (absmean ternarisation + packing) on fp32 weights of this layer's
    # shape, timed on its own: it is not part of a forward step
    wq = None
    if args.workload in ("decode", "prefill", "hbitlinear"):
        w32 = torch.from_numpy(wl.weights(N, K, seed=rank + 7)).to(dev)
        pk_o = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
        sw_o = torch.empty((1,), dtype=torch.float32, device=dev)
        ws_o = torch.empty((api.bitnet_quantize_weights_workspace_size(N, K),), dtype=torch.uint8, device=dev)
        for _ in range(3):
            api.bitnet_quantize_weights(w32, pkW=pk_o, s_w=sw_o, workspace=ws_o, stream=stream)
        reps = 10
        t_wq = timed(graph_of(lambda i: api.bitnet_quantize_weights(w32, pkW=pk_o, s_w=sw_o, workspace=ws_o,
                                                                    stream=stream), reps)) / reps / 1e3
        wbytes = N * K * 4 * 2 + N * K // 4 + 4          # fp32 weights read twice (mean, codes), packed written
        wq = {"us": t_wq * 1e6, "achieved_GBs": wbytes / t_wq / 1e9, "frac": wbytes / t_wq / 1e9 /
              load_peaks()[0]["hbm_gbs"], "algorithmic_bytes": wbytes, "weights": N * K, "input": "fp32"}
        del w32

    # decode: the same weight ring at the other decode batch sizes (linear launches only)
    sweep = []
    if args.workload == "decode":
        # the same weights five per byte (1.6 bits per weight), repacked on the GPU
        ring5 = [api.bitnet_repack_trit5(pk, stream=stream) for pk, _ in ring]
        torch.cuda.synchronize()
        r5_bytes = N * api.bitnet_trit5_row_bytes(K)
        for Ms in (1, 4, 16):
            cs = wl.decode(Ms, with_weights=False)
            xs = torch.from_numpy(cs["x"].view(np.int16)).view(torch.bfloat16).to(dev)
            xqs = torch.empty((Ms, K), dtype=torch.int8, device=dev)
            sxs = torch.empty((Ms,), dtype=torch.float32, device=dev)
            Ys = torch.empty((Ms, N), dtype=out_dtype, device=dev)
            api.bitnet_quant_act(xs, None, eps, Xq=xqs, s_x=sxs, stream=stream)

            def lin_s(i, xqs=xqs, sxs=sxs, Ys=Ys):
                pk, s_w = ring[i % copies]
                api.bitnet_linear(xqs, 8, sxs, pk, s_w, Y=Ys, stream=stream)

            def fused_s(i, xs=xs, xqs=xqs, sxs=sxs, Ys=Ys):
                pk, s_w = ring[i % copies]
                api.bitnet_bitlinear(xs, pk, s_w, None, eps, Y=Ys, Xq=xqs, s_x=sxs, stream=stream)

            def lin5_s(i, xqs=xqs, sxs=sxs, Ys=Ys):
                api.bitnet_linear_trit5(xqs, 8, sxs, ring5[i % copies], ring[i % copies][1], K, Y=Ys, stream=stream)

            def step_s(i, xs=xs, xqs=xqs, sxs=sxs, Ys=Ys):
                api.bitnet_quant_act(xs, None, eps, Xq=xqs, s_x=sxs, stream=stream)
                lin_s(i)

            api.bitnet_set_linear_path(4)
            for i in range(warmup):
                fused_s(i)
            t_f = timed(graph_of(fused_s, steps)) / steps / 1e3
            api.bitnet_set_linear_path(0)
            for i in range(warmup):
                lin_s(i)
                step_s(i)
            t_s = timed(graph_of(lin_s, steps)) / steps / 1e3
            t_st = timed(graph_of(step_s, steps)) / steps / 1e3
            for i in range(warmup):
                lin5_s(i)
            t_5 = timed(graph_of(lin5_s, steps)) / steps / 1e3
            hbm = load_peaks()[0]["hbm_gbs"]
            b = packed_bytes + Ms * K + 4 * Ms + 4 + Ms * N * out_bytes
            bf = packed_bytes + 2 * Ms * K + Ms * K + 4 * Ms + 4 + Ms * N * out_bytes
            b5 = r5_bytes + Ms * K + 4 * Ms + 4 + Ms * N * out_bytes
            sweep.append({"M": Ms, "linear_us": t_s * 1e6, "linear_GBs": b / t_s / 1e9,
                          "trit5_linear_us": t_5 * 1e6, "trit5_linear_GBs": b5 / t_5 / 1e9,
                          "trit5_linear_frac": b5 / t_5 / 1e9 / hbm,
                          "linear_frac": b / t_s / 1e9 / hbm, "step_us": t_st * 1e6, "tokens_per_s": Ms / t_st,
                          "fused_kernel_us": t_f * 1e6, "fused_kernel_frac": bf / t_f / 1e9 / hbm})

    if rank != 0:
        return None

    tokens_per_step = M * world
    value = tokens_per_step * steps / (t_step / 1e3)
    ms_per_step = t_step / steps
    peaks, peak_src = load_peaks()
    lin_s = t_lin / steps / 1e3
    q_s = t_q / steps / 1e3
    x_in_bytes = M * K * (2 if c["x_dtype"] == "bf16" else 4)
    xq_bytes = M * K if bits == 8 else M * K // 2
    if args.workload.startswith("decode") or args.workload == "tiny":
        alg_bytes = packed_bytes + xq_bytes + 4 * M + 4 + M * N * out_bytes
        roof = {"bound": "hbm", "achieved": alg_bytes / lin_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "kernel": "bitnet_linear (warp-MMA decode)" if M <= 32 and K % 512 == 0 else "bitnet_linear (tcgen05)",
                "algorithmic_bytes_per_launch": alg_bytes}
        tag = f"linear_{args.workload}"
    else:
        ops = 2.0 * M * N * K
        int8_peak = 2.0 * peaks["bf16_tflops"]          # nominal int8 : bf16 = 4.5 : 2.25
        roof = {"bound": "tensor", "achieved": ops / lin_s / 1e12, "peak": int8_peak, "unit": "TOPS",
                "kernel": "bitnet_linear (tcgen05 kind::i8)", "algorithmic_ops_per_launch": ops,
                "peak_note": "2 x measured bf16 burst (nominal int8/bf16 ratio)"}
        tag = f"linear_{args.workload}"
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(tag)
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    quant_bytes = x_in_bytes + xq_bytes + 4 * M
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8xternary->int32" if bits == 8 else "int4xternary->int32",
        "data": "synthetic",
        "config": {"workload": c["name"], "M_tokens": M, "K": K, "N": N, "act_bits": bits,
                   "x_dtype": c["x_dtype"], "out_dtype": "bf16" if out_bytes == 2 else "f32",
                   "l2": f"ring of {copies} packed-weight copies ({copies * packed_bytes / 1e6:.0f} MB > 2x L2)",
                   "timing": "CUDA graph of the K steps, CUDA events on the launching stream",
                   "parallelism": f"dp{world} (independent batches per rank)"},
        "roofline": roof,
        "kernels_us": {"quant": q_s * 1e6, "linear": lin_s * 1e6},
        "quant_roofline": {"bound": "hbm", "achieved": quant_bytes / q_s / 1e9, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": quant_bytes / q_s / 1e9 / peaks["hbm_gbs"]},
        "e2e": {"value": tokens_per_step * steps / (t_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * steps,
        "clocks": clk,
    }
    if sweep:
        line["decode_sweep"] = sweep
    if wq is not None:
        line["weights_quant"] = wq
    return line


def run_chain(args, rank, world, local_rank):
    """24 stacked layers (hidden 2048, FFN 5632) on M tokens per step."""
    import torch
    import torch.distributed as dist

    from bitlinear_bitnet_quant_b200 import api, build_lib, chain

    build_lib.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    M = CHAIN_WORKLOADS[args.workload]
    H, F = wl.CHAIN_HIDDEN, wl.CHAIN_FFN
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + rank)
    layers = []
    for _ in range(CHAIN_LAYERS):          # N(0, 0.02) weights drawn on the device, quantised offline
        w = {name: torch.randn((n, k), generator=g, device=dev) * 0.02 for name, n, k, _ in wl.CHAIN_PROJ}
        layers.append(chain.quantize_layer(w))
        del w
    torch.cuda.synchronize()
    ch = chain.BitLinearChain(layers, M, H, F, dev)
    x = torch.from_numpy(wl.chain_input(M)).to(dev)

    warmup = max(3, args.warmup)
    for _ in range(warmup):
        ch.forward(x, stream)
    torch.cuda.synchronize()

    def graph_of(fn):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for _ in range(args.steps):
                fn()
        return gr

    def lin_only():                          # the chain's linear layers alone, same operands
        for w in layers:
            for name, Xq, sx, Y, bits in (("q", ch.xq, ch.sx, ch.q, 8), ("k", ch.xq, ch.sx, ch.k, 8),
                                          ("v", ch.xq, ch.sx, ch.v, 8), ("o", ch.v4, ch.sv, ch.o, 4),
                                          ("up", ch.hq, ch.sh, ch.up, 8), ("gate", ch.hq, ch.sh, ch.gate, 8),
                                          ("down", ch.a4, ch.sa, ch.d, 4)):
                api.bitnet_linear(Xq, bits, sx, *w[name], Y=Y, stream=stream)

    g_step = graph_of(lambda: ch.forward(x, stream))
    g_lin = graph_of(lin_only)
    visible = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    clocks = ClockSampler(visible[local_rank] if local_rank < len(visible) else str(local_rank))
    clocks.start()
    t_step = timed_replay(g_step, stream, world, dev)
    t_lin = timed_replay(g_lin, stream, world, dev)
    clk = clocks.stop()

    # e2e: host input in, host output back, through the Python API
    x_pin = torch.empty((M, H), dtype=torch.float32).pin_memory()
    x_pin.copy_(x.cpu())
    y_pin = torch.empty((M, H), dtype=torch.float32).pin_memory()
    for _ in range(warmup):
        x.copy_(x_pin, non_blocking=True)
        y_pin.copy_(ch.forward(x, stream), non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        x.copy_(x_pin, non_blocking=True)
        y_pin.copy_(ch.forward(x, stream), non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    steps = args.steps
    step_s = t_step / steps / 1e3
    lin_s = t_lin / steps / 1e3                       # all 7 x 24 linear launches of one step
    packed = ch.packed_bytes()
    ops = 2.0 * M * sum(n * k for _, n, k, _ in wl.CHAIN_PROJ) * CHAIN_LAYERS
    act_bytes = CHAIN_LAYERS * M * (4 * (5 * H + 3 * F) + 2 * H + H // 2 + F // 2 + 7 * 4)
    if M <= 64:
        roof = {"bound": "hbm", "achieved": (packed + act_bytes) / lin_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "kernel": "bitnet_linear, all 168 launches of a step",
                "algorithmic_bytes_per_step": packed + act_bytes}
    else:
        roof = {"bound": "tensor", "achieved": ops / lin_s / 1e12, "peak": 2.0 * peaks["bf16_tflops"],
                "unit": "TOPS", "kernel": "bitnet_linear, all 168 launches of a step",
                "algorithmic_ops_per_step": ops, "peak_note": "2 x measured bf16 burst (nominal int8/bf16 ratio)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(f"linear_{args.workload}")
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    tokens = M * world
    return {
        "metric": METRIC, "value": tokens * steps / (t_step / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": t_step / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8/int4 x ternary -> int32, fp32 glue",
        "data": "synthetic",
        "config": {"workload": f"bitlinear_chain_{CHAIN_LAYERS}layers_m{M}_hidden{H}_ffn{F}", "M_tokens": M,
                   "layers": CHAIN_LAYERS, "l2": f"{packed / 1e6:.0f} MB of packed weights per step (> 2x L2)",
                   "timing": "CUDA graph of the K steps, CUDA events on the launching stream",
                   "parallelism": f"dp{world} (independent batches per rank)"},
        "roofline": roof,
        "kernels_us": {"linear_all_per_step": lin_s * 1e6, "step": step_s * 1e6},
        "e2e": {"value": tokens * steps / (t_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": M * H * 4, "d2h_bytes_per_step": M * H * 4},
        "gpu_launches": ch.launches * steps,
        "clocks": clk,
    }


def chain_cpu_baseline(M, budget_s=10.0):
    """Oracle tokens/s through the chain: two layers, scaled to 24."""
    from oracle import bitnet_oracle as O
    layers = []
    for l in range(2):
        lw = {}
        for name, w in wl.chain_weights(l).items():
            _, s_w, q = O.quantize_weights(w)
            lw[name] = (q, s_w)
        layers.append(lw)
    x = wl.chain_input(min(M, 4))
    t0 = time.perf_counter()
    n = 0
    while True:
        y = x
        for lw in layers:
            y = O.chain_layer(y, lw)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = (time.perf_counter() - t0) * CHAIN_LAYERS / 2
    return {"value": n * len(x) / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} passes of {len(x)} tokens through 2 oracle layers, time scaled to {CHAIN_LAYERS} layers"}


# ----------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline leg)
# ----------------------------------------------------------------------------

def oracle_step_fn(c):
    from oracle import bitnet_oracle as O
    w = wl.weights(c["N"], c["K"], seed=0)
    _, s_w, qw = O.quantize_weights(w)
    x = O.bf16_bits_to_f32(c["x"]) if c["x_dtype"] == "bf16" else c["x"]

    def step(rows):
        xs = x[rows]
        if c["act_bits"] == 8:
            q, s = O.quant_act(xs, None, 1e-6)
        else:
            _, s, q, _ = O.hadamard_quant_act(xs, None, 1e-6, c.get("had_block", 0))
        O.linear(q, s, qw, s_w)
        return len(xs)
    return step


def sample_rows(c):
    """Rows of one sampled step: the whole batch when small, else 8 tokens."""
    return np.arange(c["M"]) if c["M"] <= 16 else np.arange(8)


def cpu_baseline(c, budget_s=10.0):
    step = oracle_step_fn(c)
    rows = sample_rows(c)
    step(rows[:1])                                   # warm-up (allocations)
    t0 = time.perf_counter()
    tokens, n = 0, 0
    while True:
        tokens += step(rows)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} oracle steps of {len(rows)} tokens of {c['name']} (numpy, single thread)"}


def cpu_baseline_omp(c, budget_s=5.0):
    """The same oracle step through the plain C++ oracle, its loops over tokens and
    output rows on all host cores (bit-identical results to the numpy oracle)."""
    from oracle import c_oracle as C
    w = wl.weights(c["N"], c["K"], seed=0)
    _, s_w, qw = C.quantize_weights(w)
    x = (c["x"].astype(np.uint32) << 16).view(np.float32) if c["x_dtype"] == "bf16" else c["x"]
    rows = np.arange(c["M"]) if c["M"] <= 16 else np.arange(128)

    def step():
        xs = x[rows]
        if c["act_bits"] == 8:
            q, s = C.quant_act(xs, None, 1e-6)
        else:
            _, s, q, _ = C.hadamard_quant_act(xs, None, 1e-6, c.get("had_block", 0))
        C.linear(q, s, qw, s_w)
        return len(rows)

    step()                                           # warm-up
    t0 = time.perf_counter()
    tokens, n = 0, 0
    while True:
        tokens += step()
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": C.threads(), "kind": "oracle (C++, OpenMP)",
            "sample": f"{n} oracle steps of {len(rows)} tokens of {c['name']} (C++ oracle, OpenMP over tokens "
                      f"and output rows)"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    c = WORKLOADS[args.workload]()
    step = oracle_step_fn(c)
    rows = sample_rows(c)
    for _ in range(max(3, args.warmup)):
        step(rows)
    t0 = time.perf_counter()
    tokens = 0
    for _ in range(args.steps):
        tokens += step(rows)
    dt = time.perf_counter() - t0
    value = tokens / dt
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8xternary->int64" if c["act_bits"] == 8 else "int4xternary->int64",
            "data": "synthetic",
            "config": {"workload": c["name"], "M_tokens": c["M"], "K": c["K"], "N": c["N"],
                       "act_bits": c["act_bits"], "parallelism": "rank 0 only (CPU oracle)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step: {len(rows)} tokens of {c['name']} through the numpy oracle"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(CHAIN_WORKLOADS), default="decode")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        world = max(world, 1)

    if args.impl == "reference":
        line = run_reference(args, rank, world) if args.workload in WORKLOADS else None
        if args.workload in CHAIN_WORKLOADS and rank == 0:
            cb = chain_cpu_baseline(CHAIN_WORKLOADS[args.workload], budget_s=2.0 * max(1, args.steps))
            line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
                    "n_gpus": world, "steps": args.steps, "warmup": 0, "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None, "data": "synthetic",
                    "config": {"workload": args.workload, "parallelism": "rank 0 only (CPU oracle)"},
                    "cpu_baseline": cb, "e2e": {"value": cb["value"], "unit": "tokens/s",
                                                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    pg = False
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        pg = True
    try:
        if args.workload in CHAIN_WORKLOADS:
            line = run_chain(args, rank, world, local_rank)
            if line is not None and world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = chain_cpu_baseline(CHAIN_WORKLOADS[args.workload])
        else:
            line = run_ours(args, rank, world, local_rank)
            if line is not None and world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(WORKLOADS[args.workload]())
                try:
                    line["cpu_baseline_all_cores"] = cpu_baseline_omp(WORKLOADS[args.workload]())
                except Exception as e:                   # e.g. no C++ compiler on the host
                    line["cpu_baseline_all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
