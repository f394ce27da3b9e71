"""Benchmark of the BitLinear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|<name>]
                    [--impl ours|reference] [--min-time S] [--no-cpu-baseline]

With no --workload every configuration runs in one invocation, and rank 0
prints one JSON line.  Its top-level keys describe the headline: the largest
configuration, 24 stacked BitLinear layers (hidden 2048, FFN 5632) on a
512-token prefill batch.  The key "configs" holds one object per other
configuration (tiny BitLinear, decode GEMV at 1, 4 and 16 tokens, batched
prefill GEMM, the H-BitLinear a4 layer, the chain at 32 decode tokens), each
with its own throughput, roofline, cpu_baseline and e2e.

A step is one pass of the whole path over one batch: for a single layer the
activation quantiser (RMSNorm + absmax int8, or RMSNorm + Hadamard + int4) and
the ternary product with its dequantisation; for the chain every quantiser,
product and element-wise step of all 24 layers.  Weights are quantised
offline, outside the timed region.

Device timing: the K steps are captured in one CUDA graph.  The timed region
is R back-to-back replays of that graph (R chosen so the region lasts at
least --min-time seconds), between a barrier and a device synchronise on both
sides; each replay is bracketed by CUDA events on the launching stream.  The
step time is the median replay time / K (max over ranks), with the spread
over replays reported.  Every single-layer step reads the next of a ring of
weight (and, where the activations are large, activation) copies whose total
exceeds twice the 126 MB L2; the chain's 308 MB of packed weights exceed it
by themselves.  The dominant kernel is timed the same way in a graph of its
own launches for the roofline.  e2e: the same steps through the public Python
API with pinned host buffers, host<->device copies inside the timed region.
Clocks are sampled with nvidia-smi during every timed region.  The CPU oracle
is timed on a bounded sample on the host.

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
NOMINAL_INT8_TOPS = 4500.0
METRIC = "BitLinear tokens/sec and GB/s|TOPS vs HBM/int8 roofline, 1xB200"
EPS = 1e-6

# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

WORKLOADS = {
    "tiny": lambda: wl.tiny(),
    "decode_m1": lambda: wl.decode(1, with_weights=False),
    "decode_m4": lambda: wl.decode(4, with_weights=False),
    "decode_m16": lambda: wl.decode(16, with_weights=False),
    "prefill": lambda: wl.prefill(with_weights=False),
    "hbitlinear": lambda: wl.hbitlinear(with_weights=False),
}
CHAIN_WORKLOADS = {"chain_decode": 32, "chain_prefill": 512,          # tokens per step
                   "chain_decode_attn": 32, "chain_prefill_attn": 512}
# with the attention core: (sequences, tokens per sequence, first position, cache rows)
CHAIN_ATTENTION = {"chain_prefill_attn": (1, 512, 0, 512), "chain_decode_attn": (32, 1, 512, 513)}
CHAIN_LAYERS = 24
ORDER = ["tiny", "decode_m1", "decode_m4", "decode_m16", "prefill", "hbitlinear", "chain_decode", "chain_decode_attn",
         "chain_prefill_attn", "chain_prefill"]
HEADLINE = "chain_prefill"
# roofline fractions the decode GEMV and the batched prefill GEMM are held to
TARGET_FRAC = {"decode_m1": 0.70, "decode_m4": 0.70, "decode_m16": 0.70, "prefill": 0.50}


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


def int8_peak_from_bf16(peaks) -> float:
    """Dense int8 TOPS derived from the measured bf16 burst x the nominal int8 : bf16 ratio (4.5 : 2.25)."""
    return 2.0 * float(peaks["bf16_tflops"])


def measure_int8_peak(api, stream, sms: int) -> dict:
    """Dense int8 tensor-core throughput measured here: back-to-back tcgen05 kind::i8
    MMAs (128 x 128 x 32, the GEMM's instruction form) on every SM, between CUDA
    events; the SM clock over the run comes from the kernel's own cycle and
    nanosecond counters."""
    import torch
    n_mma = 65536
    best = None
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cyc, ns = api.bitnet_measure_i8_mma(n_mma, 128, sms, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        tops = 2.0 * 128 * 128 * 32 * n_mma * sms / (ms * 1e-3) / 1e12
        mhz = float((cyc.double() / ns.double()).median().item() * 1e3)
        if best is None or tops > best["tops"]:
            best = {"tops": tops, "sm_mhz": mhz, "ms": ms}
    return {"value": best["tops"], "unit": "TOPS", "sm_mhz_during": best["sm_mhz"],
            "method": f"bitnet_measure_i8_mma: {n_mma} back-to-back 128x128x32 kind::i8 MMAs per SM on {sms} SMs, "
                      "CUDA events (best of 3)"}


def tensor_peak(ctx) -> tuple:
    """(peak TOPS, source) for the int8 tensor-core rooflines: this run's measurement."""
    m = ctx.get("int8_peak")
    if m is not None:
        return m["value"], "measured in this run (bitnet_measure_i8_mma)"
    return int8_peak_from_bf16(ctx["peaks"][0]), "2 x bf16 burst (nominal int8 : bf16 ratio)"


def profiled_traffic(kernel_tag: str):
    """DRAM bytes per launch (per step for the stacked-layer workloads, whose
    roofline covers every linear launch of a step) from the committed ncu
    summary, if it was taken on the current kernel sources (else None)."""
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
        return float(kv["dram_bytes_per_launch"] if "dram_bytes_per_launch" in kv else kv["dram_bytes_per_step"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled in the background; each
    sample carries the host time it arrived, so a window can be summarised."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: str, period_ms: int = 100):
        self.gpu = gpu_index
        self.period_ms = period_ms
        self.proc = None
        self.samples = []            # (host time, sm MHz, max MHz, reasons)
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.strip().split(",")]
            if len(f) < 9:
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            reasons = {n for n, v in zip(self.REASONS, f[5:9]) if v.lower().startswith("active")}
            self.samples.append((time.monotonic(), sm, mx, reasons))

    def summary(self, t0=None, t1=None):
        sel = [s for s in self.samples if (t0 is None or s[0] >= t0) and (t1 is None or s[0] <= t1)]
        if not sel:
            return None
        reasons = set()
        for s in sel:
            reasons |= s[3]
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": max(s[2] for s in sel),
                "reasons": sorted(reasons), "samples": len(sel)}

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
        return self.summary()


# ----------------------------------------------------------------------------
# device timing
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


class Timer:
    """Times CUDA graphs of K steps: R replays (at least min_time seconds in
    all) between a barrier and a device synchronise on both sides, CUDA events
    around each replay on the launching stream."""

    def __init__(self, stream, world, dev, steps, min_time_s, clocks):
        self.stream, self.world, self.dev = stream, world, dev
        self.steps, self.min_time_s, self.clocks = steps, min_time_s, clocks
        self.windows = []

    def graph(self, fn, count=None):
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for i in range(self.steps if count is None else count):
                fn(i)
        return g

    def time(self, g, count=None):
        """Returns dict(ms per step: median / min / max over replays, replays)."""
        import torch
        import torch.distributed as dist
        count = self.steps if count is None else count
        g.replay()
        torch.cuda.synchronize()
        if self.world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_host0 = time.monotonic()
        events = []
        batch = 1
        while True:
            for _ in range(batch):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(self.stream)
                g.replay()
                e1.record(self.stream)
                events.append((e0, e1))
            torch.cuda.synchronize()
            if time.monotonic() - t_host0 >= self.min_time_s or len(events) >= 100000:
                break
            batch = min(2 * batch, 4096)
        t_host1 = time.monotonic()
        if self.world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        per = sorted(e0.elapsed_time(e1) / count for e0, e1 in events)
        med = max_over_ranks(statistics.median(per), self.world, self.dev)
        self.windows.append((t_host0, t_host1))
        return {"ms": med, "min_ms": per[0], "max_ms": per[-1], "replays": len(per), "steps_per_replay": count,
                "window": (t_host0, t_host1)}


def spread(t):
    return {"replays": t["replays"], "steps_per_replay": t["steps_per_replay"], "median_ms_per_step": t["ms"],
            "min_ms_per_step": t["min_ms"], "max_ms_per_step": t["max_ms"]}


def e2e_time(step_fn, stream, world, dev, steps, min_time_s):
    """Seconds per step of step_fn run eagerly (host copies included), at least
    `steps` steps and min_time_s seconds, between CUDA events."""
    import torch
    import torch.distributed as dist
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.monotonic()
    n = 0
    e0.record(stream)
    while n < steps or time.monotonic() - t0 < min_time_s:
        step_fn(n)
        n += 1
        if n % 64 == 0:
            stream.synchronize()
    e1.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1) / n, world, dev) / 1e3


def to_device_x(c, dev):
    import torch
    if c["x_dtype"] == "bf16":
        return torch.from_numpy(c["x"].view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(c["x"]).to(dev)


# ----------------------------------------------------------------------------
# our implementation: one BitLinear layer
# ----------------------------------------------------------------------------

def run_layer(name, args, ctx):
    import torch

    api, rank, world, dev, stream, timer = ctx["api"], ctx["rank"], ctx["world"], ctx["dev"], ctx["stream"], \
        ctx["timer"]
    c = WORKLOADS[name]()
    M, K, N, bits = c["M"], c["K"], c["N"], c["act_bits"]
    had_block = c.get("had_block", 0)
    out_dtype = torch.bfloat16 if name == "prefill" else torch.float32
    out_bytes = 2 if out_dtype == torch.bfloat16 else 4

    # weights, quantised offline: a ring of copies larger than 2x L2
    packed_bytes = N * K // 4
    copies = max(2, min(64, math.ceil(2.2 * L2_BYTES / packed_bytes)))
    rng = np.random.default_rng(1234 + rank)
    base_w = torch.from_numpy(wl.weights(N, K, seed=rank)).to(dev)
    ring = []
    for i in range(copies):
        w = base_w if i == 0 else base_w[torch.from_numpy(rng.permutation(N)).to(dev)]
        ring.append(api.bitnet_quantize_weights(w.contiguous(), stream=stream))
    del base_w
    # activations: a ring too when one input is a sizeable part of the L2
    x0 = to_device_x(c, dev)
    x_bytes = x0.numel() * x0.element_size()
    xcopies = 1 if x_bytes * 8 < L2_BYTES else max(2, math.ceil(2.2 * L2_BYTES / x_bytes))
    xring = [x0] + [x0[torch.from_numpy(rng.permutation(M)).to(dev)].contiguous() for _ in range(xcopies - 1)]
    torch.cuda.synchronize()

    xq = torch.empty((M, K) if bits == 8 else (M, K // 2), dtype=torch.int8 if bits == 8 else torch.uint8,
                     device=dev)
    s_x = torch.empty((M,), dtype=torch.float32, device=dev)
    Y = torch.empty((M, N), dtype=out_dtype, device=dev)

    def quant(i):
        x = xring[i % xcopies]
        if bits == 8:
            api.bitnet_quant_act(x, None, EPS, Xq=xq, s_x=s_x, stream=stream)
        else:
            api.bitnet_hadamard_quant_act(x, None, EPS, had_block, Xq4=xq, s_x=s_x, stream=stream)

    def linear(i):
        pk, s_w = ring[i % copies]
        api.bitnet_linear(xq, bits, s_x, pk, s_w, Y=Y, stream=stream)

    def step(i):
        quant(i)
        linear(i)

    warmup = max(3, args.warmup)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    t_step = timer.time(timer.graph(step))
    t_lin = timer.time(timer.graph(linear))
    t_q = timer.time(timer.graph(quant))

    # e2e through the public API: pinned host input in, host output back
    x_pin = torch.empty_like(x0, device="cpu").pin_memory()
    x_pin.copy_(x0.cpu())
    x_dev = torch.empty_like(x0)
    y_pin = torch.empty((M, N), dtype=out_dtype).pin_memory()

    def e2e_step(i):
        x_dev.copy_(x_pin, non_blocking=True)
        pk, s_w = ring[i % copies]
        Yo = api.bitlinear_forward(x_dev, pk, s_w, act_bits=bits, eps=EPS, had_block=had_block,
                                   out_dtype=out_dtype, Y=Y, Xq=xq, s_x=s_x, stream=stream)
        y_pin.copy_(Yo, non_blocking=True)

    for i in range(warmup):
        e2e_step(i)
    t_e2e = e2e_time(e2e_step, stream, world, dev, args.steps, args.min_time / 2)

    sub = {"workload": c["name"], "M_tokens": M, "K": K, "N": N, "act_bits": bits, "x_dtype": c["x_dtype"],
           "out_dtype": "bf16" if out_bytes == 2 else "f32",
           "l2": (f"ring of {copies} packed-weight copies ({copies * packed_bytes / 1e6:.0f} MB)"
                  + (f" and {xcopies} activation copies ({xcopies * x_bytes / 1e6:.0f} MB)" if xcopies > 1 else "")
                  + ": > 2x L2")}
    lin_s = t_lin["ms"] / 1e3
    q_s = t_q["ms"] / 1e3
    step_s = t_step["ms"] / 1e3
    peaks, peak_src = ctx["peaks"]
    x_in_bytes = M * K * (2 if c["x_dtype"] == "bf16" else 4)
    xq_bytes = M * K if bits == 8 else M * K // 2
    if M <= 32:
        alg_bytes = packed_bytes + xq_bytes + 4 * M + 4 + M * N * out_bytes
        roof = {"bound": "hbm", "achieved": alg_bytes / lin_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "kernel": "bitnet_linear (warp-MMA decode)" if K % 512 == 0 else "bitnet_linear (tcgen05)",
                "algorithmic_bytes_per_launch": alg_bytes}
    else:
        ops = 2.0 * M * N * K
        tp, tsrc = tensor_peak(ctx)
        roof = {"bound": "tensor", "achieved": ops / lin_s / 1e12, "peak": tp, "unit": "TOPS",
                "kernel": "bitnet_linear (tcgen05 kind::i8)", "algorithmic_ops_per_launch": ops,
                "peak_note": tsrc,
                "frac_of_bf16_derived_peak": ops / lin_s / 1e12 / int8_peak_from_bf16(peaks),
                "frac_of_nominal_4500_tops": ops / lin_s / 1e12 / NOMINAL_INT8_TOPS}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(f"linear_{name}")
    if roof["bound"] == "hbm":
        roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    # the targets stated for this build: decode GEMV >= 70 % of HBM, prefill GEMM >= 50 % of int8
    target = TARGET_FRAC.get(name)
    if target is not None:
        roof["target_frac"] = target
        roof["target_met"] = bool(roof["frac"] >= target)
    quant_bytes = x_in_bytes + xq_bytes + 4 * M
    sub.update({
        "value": M * world / step_s, "unit": "tokens/s", "ms_per_step": t_step["ms"],
        "timing": spread(t_step),
        "roofline": roof,
        "kernels_us": {"quant": q_s * 1e6, "linear": lin_s * 1e6, "step": step_s * 1e6},
        "quant_roofline": {"bound": "hbm", "achieved": quant_bytes / q_s / 1e9, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": quant_bytes / q_s / 1e9 / peaks["hbm_gbs"],
                           "algorithmic_bytes_per_launch": quant_bytes},
        "e2e": {"value": M * world / t_e2e, "unit": "tokens/s",
                "h2d_bytes_per_step": x_pin.numel() * x_pin.element_size(),
                "d2h_bytes_per_step": y_pin.numel() * y_pin.element_size()},
        "gpu_launches_per_step": 2,
        "clocks": ctx["clocks"].summary(t_step["window"][0], t_q["window"][1]),
    })

    if name.startswith("decode"):
        sub["decode_variants"] = decode_variants(ctx, c, ring, copies, xq, s_x, Y, x0, packed_bytes, out_bytes)
    if name in ("decode_m16", "prefill", "hbitlinear"):
        sub["weights_quant"] = weights_quant(ctx, N, K)
    del ring, xring
    return sub


def decode_variants(ctx, c, ring, copies, xq, s_x, Y, x0, packed_bytes, out_bytes):
    """The same decode shape through the single fused kernel and with the
    weights five per byte (linear launches only), for comparison."""
    import torch
    api, stream, timer = ctx["api"], ctx["stream"], ctx["timer"]
    M, K, N = c["M"], c["K"], c["N"]
    hbm = ctx["peaks"][0]["hbm_gbs"]
    ring5 = [api.bitnet_repack_trit5(pk, stream=stream) for pk, _ in ring]
    torch.cuda.synchronize()
    r5_bytes = N * api.bitnet_trit5_row_bytes(K)
    Xq2 = torch.empty_like(xq)
    s_x2 = torch.empty_like(s_x)

    def fused(i):
        pk, s_w = ring[i % copies]
        api.bitnet_bitlinear(x0, pk, s_w, None, EPS, Y=Y, Xq=Xq2, s_x=s_x2, stream=stream, kernel=4)

    def lin5(i):
        api.bitnet_linear_trit5(xq, 8, s_x, ring5[i % copies], ring[i % copies][1], K, Y=Y, stream=stream)

    for i in range(3):
        fused(i)
        lin5(i)
    t_f = timer.time(timer.graph(fused))["ms"] / 1e3
    t_5 = timer.time(timer.graph(lin5))["ms"] / 1e3
    bf = packed_bytes + 2 * M * K + M * K + 4 * M + 4 + M * N * out_bytes
    b5 = r5_bytes + M * K + 4 * M + 4 + M * N * out_bytes
    del ring5
    return {"fused_kernel_us": t_f * 1e6, "fused_kernel_frac": bf / t_f / 1e9 / hbm,
            "trit5_linear_us": t_5 * 1e6, "trit5_linear_frac": b5 / t_5 / 1e9 / hbm,
            "trit5_algorithmic_bytes": b5}


def weights_quant(ctx, N, K):
    """The offline weight path (absmean ternarisation + packing) on fp32 weights
    of this layer's shape, timed on its own: it is not part of a step."""
    import torch
    api, stream, timer, dev = ctx["api"], ctx["stream"], ctx["timer"], ctx["dev"]
    w32 = torch.from_numpy(wl.weights(N, K, seed=ctx["rank"] + 7)).to(dev)
    pk_o = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
    sw_o = torch.empty((1,), dtype=torch.float32, device=dev)
    ws_o = torch.empty((api.bitnet_quantize_weights_workspace_size(N, K),), dtype=torch.uint8, device=dev)

    def wq(i):
        api.bitnet_quantize_weights(w32, pkW=pk_o, s_w=sw_o, workspace=ws_o, stream=stream)

    for i in range(3):
        wq(i)
    t = timer.time(timer.graph(wq, 4), 4)["ms"] / 1e3
    # algorithmic bytes: the fp32 weights read once, the packed codes written once (the
    # second pass over the weights, for the codes, is counted only where it cannot hit L2)
    reads = 2 if N * K * 4 > L2_BYTES else 1
    wbytes = N * K * 4 * reads + N * K // 4 + 4
    hbm = ctx["peaks"][0]["hbm_gbs"]
    return {"us": t * 1e6, "achieved_GBs": wbytes / t / 1e9, "frac": wbytes / t / 1e9 / hbm,
            "algorithmic_bytes": wbytes, "weights": N * K, "input": "fp32",
            "note": f"fp32 weights counted {'twice (larger than L2)' if reads == 2 else 'once (they fit in L2)'}"}


# ----------------------------------------------------------------------------
# our implementation: the stacked chain
# ----------------------------------------------------------------------------

def run_chain(name, args, ctx):
    import torch

    from bitlinear_bitnet_quant_b200 import chain

    api, rank, world, dev, stream, timer = ctx["api"], ctx["rank"], ctx["world"], ctx["dev"], ctx["stream"], \
        ctx["timer"]
    M = CHAIN_WORKLOADS[name]
    H, F = wl.CHAIN_HIDDEN, wl.CHAIN_FFN
    layers = ctx.get("chain_layers")
    if layers is None:
        g = torch.Generator(device=dev)
        g.manual_seed(1000 + rank)
        layers = []
        for _ in range(CHAIN_LAYERS):      # N(0, 0.02) weights drawn on the device, quantised offline
            w = {pn: torch.randn((n, k), generator=g, device=dev) * 0.02 for pn, n, k, _ in wl.CHAIN_PROJ}
            layers.append(chain.quantize_layer(w, stream=stream))
            del w
        torch.cuda.synchronize()
        ctx["chain_layers"] = layers
    att = CHAIN_ATTENTION.get(name)
    t0 = 0
    if att is None:
        ch = chain.BitLinearChain(layers, M, H, F, dev)
    else:
        B, L, t0, T_cap = att
        ch = chain.BitLinearChain(layers, M, H, F, dev, attention=dict(B=B, L=L, T_cap=T_cap, heads=wl.CHAIN_HEADS))
        if t0 > 0:
            # the decode step continues B sequences whose first t0 tokens went through a prefill
            pre = chain.BitLinearChain(layers, B * t0, H, F, dev,
                                       attention=dict(B=B, L=t0, T_cap=T_cap, heads=wl.CHAIN_HEADS))
            pre.kc, pre.vc = ch.kc, ch.vc
            pre.forward(torch.from_numpy(wl.chain_input(B * t0, seed=9)).to(dev), stream, t0=0)
            torch.cuda.synchronize()
            del pre
            torch.cuda.empty_cache()
    x = torch.from_numpy(wl.chain_input(M)).to(dev)

    warmup = max(3, args.warmup)
    for _ in range(warmup):
        ch.forward(x, stream, t0=t0)
    torch.cuda.synchronize()

    def lin_only(i):                       # the chain's linear launches alone, same operands
        for w in layers:
            api.bitnet_linear_group(ch.xq, 8, ch.sx, [w["q"], w["k"], w["v"]], Ys=[ch.q, ch.k, ch.v], stream=stream)
            api.bitnet_linear(ch.v4, 4, ch.sv, *w["o"], Y=ch.o, stream=stream)
            api.bitnet_linear_group(ch.hq, 8, ch.sh, [w["up"], w["gate"]], Ys=[ch.up, ch.gate], stream=stream)
            api.bitnet_linear(ch.a4, 4, ch.sa, *w["down"], Y=ch.d, stream=stream)

    t_step = timer.time(timer.graph(lambda i: ch.forward(x, stream, t0=t0)))
    t_lin = timer.time(timer.graph(lin_only))
    t_att = None
    if att is not None:
        def att_only(i):                   # rotary embedding, cache append and attention of every layer
            for li in range(CHAIN_LAYERS):
                api.bitnet_rope_append(ch.q, ch.k, ch.v, ch.kc[li], ch.vc[li], B, L, t0, ch.heads, stream=stream)
                api.bitnet_attention(ch.q, ch.kc[li], ch.vc[li], B, L, t0, ch.heads, A=ch.att, stream=stream)
        t_att = timer.time(timer.graph(att_only))

    # e2e: host input in, host output back, through the Python API
    x_pin = torch.empty((M, H), dtype=torch.float32).pin_memory()
    x_pin.copy_(x.cpu())
    y_pin = torch.empty((M, H), dtype=torch.float32).pin_memory()

    def e2e_step(i):
        x.copy_(x_pin, non_blocking=True)
        y_pin.copy_(ch.forward(x, stream, t0=t0), non_blocking=True)

    for i in range(warmup):
        e2e_step(i)
    t_e2e = e2e_time(e2e_step, stream, world, dev, args.steps, args.min_time / 2)

    peaks, peak_src = ctx["peaks"]
    step_s = t_step["ms"] / 1e3
    lin_s = t_lin["ms"] / 1e3                       # all 7 x 24 linear launches of one step
    packed = ch.packed_bytes()
    ops = 2.0 * M * sum(n * k for _, n, k, _ in wl.CHAIN_PROJ) * CHAIN_LAYERS
    act_bytes = CHAIN_LAYERS * M * (4 * (5 * H + 3 * F) + 2 * H + H // 2 + F // 2 + 7 * 4)
    if M <= 64:
        roof = {"bound": "hbm", "achieved": (packed + act_bytes) / lin_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "kernel": f"bitnet_linear(_group), all {4 * CHAIN_LAYERS} launches of a step",
                "algorithmic_bytes_per_step": packed + act_bytes}
    else:
        tp, tsrc = tensor_peak(ctx)
        roof = {"bound": "tensor", "achieved": ops / lin_s / 1e12, "peak": tp,
                "unit": "TOPS", "kernel": f"bitnet_linear(_group), all {4 * CHAIN_LAYERS} launches of a step",
                "algorithmic_ops_per_step": ops, "peak_note": tsrc,
                "frac_of_bf16_derived_peak": ops / lin_s / 1e12 / int8_peak_from_bf16(peaks),
                "frac_of_nominal_4500_tops": ops / lin_s / 1e12 / NOMINAL_INT8_TOPS}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(f"linear_{name}")
    if roof["bound"] == "hbm":
        roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    # whole-step view: the slower of the weight stream and the integer work, against the step time
    ideal = max((packed + act_bytes) / (peaks["hbm_gbs"] * 1e9), ops / (tensor_peak(ctx)[0] * 1e12))
    extra = {}
    if att is not None:
        att_s = t_att["ms"] / 1e3
        n_ctx = t0 + L
        # per layer: the caches' keys and values each sequence's queries read (fp32), and the
        # score and weighted-sum multiply-adds (causal: a query at position p reads p + 1 keys)
        pairs = B * sum(t0 + l + 1 for l in range(L))
        kv_bytes = CHAIN_LAYERS * B * n_ctx * H * 4 * 2
        flops = CHAIN_LAYERS * 2 * 2 * pairs * H
        extra["attention"] = {
            "us_per_step": att_s * 1e6, "sequences": B, "tokens_per_sequence": L, "first_position": t0,
            "cache_bytes_read_per_step": kv_bytes, "fp32_flops_per_step": flops,
            "achieved_GBs": kv_bytes / att_s / 1e9, "achieved_TFLOPs": flops / att_s / 1e12,
            "note": "rotary embedding + cache append + causal softmax attention of all 24 layers (fp32 CUDA cores)"}
    return {
        "workload": (f"bitlinear_chain_{CHAIN_LAYERS}layers_m{M}_hidden{H}_ffn{F}" +
                     ("" if att is None else f"_attention_{B}seq_ctx{t0 + L}")), "M_tokens": M,
        "layers": CHAIN_LAYERS, "hidden": H, "ffn": F,
        "l2": f"{packed / 1e6:.0f} MB of packed weights per step (> 2x L2)",
        "value": M * world / step_s, "unit": "tokens/s", "ms_per_step": t_step["ms"],
        "timing": spread(t_step),
        "roofline": roof,
        "step_roofline": {"ideal_us": ideal * 1e6, "achieved_us": step_s * 1e6, "frac": ideal / step_s,
                          "note": "max(bytes / HBM peak, int ops / int8 peak) over the step time"},
        "kernels_us": {"linear_all_per_step": lin_s * 1e6, "step": step_s * 1e6},
        "e2e": {"value": M * world / t_e2e, "unit": "tokens/s",
                "h2d_bytes_per_step": M * H * 4, "d2h_bytes_per_step": M * H * 4},
        "gpu_launches_per_step": ch.launches,
        "clocks": ctx["clocks"].summary(t_step["window"][0], (t_att or t_lin)["window"][1]),
        **extra,
    }


# ----------------------------------------------------------------------------
# CPU oracle (the cpu_baseline legs and the reference arm)
# ----------------------------------------------------------------------------

_ORACLE_WEIGHTS = {}


def _oracle_weights(N, K, which):
    """Quantised weights of the (N, K) workload layer by one of the two oracles,
    computed once per process (the decode batch sizes share their layer)."""
    key = (N, K, which)
    if key not in _ORACLE_WEIGHTS:
        if which == "numpy":
            from oracle import bitnet_oracle as O
            _, s_w, qw = O.quantize_weights(wl.weights(N, K, seed=0))
        else:
            from oracle import c_oracle as C
            _, s_w, qw = C.quantize_weights(wl.weights(N, K, seed=0))
        _ORACLE_WEIGHTS[key] = (s_w, qw)
    return _ORACLE_WEIGHTS[key]


def oracle_step_fn(c):
    from oracle import bitnet_oracle as O
    s_w, qw = _oracle_weights(c["N"], c["K"], "numpy")
    x = O.bf16_bits_to_f32(c["x"]) if c["x_dtype"] == "bf16" else c["x"]

    def step(rows):
        xs = x[rows]
        if c["act_bits"] == 8:
            q, s = O.quant_act(xs, None, EPS)
        else:
            _, s, q, _ = O.hadamard_quant_act(xs, None, EPS, c.get("had_block", 0))
        O.linear(q, s, qw, s_w)
        return len(xs)
    return step


def sample_rows(c):
    """Rows of one sampled step: the whole batch when small, else 8 tokens."""
    return np.arange(c["M"]) if c["M"] <= 16 else np.arange(8)


def _timed_loop(step, budget_s):
    t0 = time.perf_counter()
    tokens, n = 0, 0
    while True:
        tokens += step()
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return tokens, n, time.perf_counter() - t0


def cpu_baseline(c, budget_s=2.0):
    step = oracle_step_fn(c)
    rows = sample_rows(c)
    step(rows[:1])                                   # warm-up (allocations)
    tokens, n, dt = _timed_loop(lambda: step(rows), budget_s)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} oracle steps of {len(rows)} tokens of {c['name']} (numpy, single thread)"}


def cpu_baseline_omp(c, budget_s=1.5):
    """The same oracle step through the plain C++ oracle, its loops over tokens and
    output rows on all host cores (bit-identical results to the numpy oracle)."""
    from oracle import c_oracle as C
    s_w, qw = _oracle_weights(c["N"], c["K"], "c")
    x = (c["x"].astype(np.uint32) << 16).view(np.float32) if c["x_dtype"] == "bf16" else c["x"]
    rows = np.arange(c["M"]) if c["M"] <= 16 else np.arange(128)

    def step():
        xs = x[rows]
        if c["act_bits"] == 8:
            q, s = C.quant_act(xs, None, EPS)
        else:
            _, s, q, _ = C.hadamard_quant_act(xs, None, EPS, c.get("had_block", 0))
        C.linear(q, s, qw, s_w)
        return len(rows)

    step()                                           # warm-up
    tokens, n, dt = _timed_loop(step, budget_s)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": C.threads(), "kind": "oracle (C++, OpenMP)",
            "sample": f"{n} oracle steps of {len(rows)} tokens of {c['name']} (C++ oracle, OpenMP over tokens "
                      f"and output rows)"}


class ChainOracle:
    """The numpy oracle's stacked layer over all 24 layers.  Two layers' weights
    are quantised and alternated (a token's work does not depend on the weight
    values), which keeps the set-up to seconds."""

    def __init__(self):
        from oracle import bitnet_oracle as O
        self.O = O
        self.layers = []
        for l in range(2):
            lw = {}
            for pn, w in wl.chain_weights(l).items():
                _, s_w, q = O.quantize_weights(w)
                lw[pn] = (q, s_w)
            self.layers.append(lw)

    def step(self, x, context: int = 0):
        """x [1, hidden] through all layers; with context > 0 the token sits at position
        context - 1 and attends over a cache of that many keys (seeded values)."""
        y = x
        for l in range(CHAIN_LAYERS):
            if context:
                rng = np.random.default_rng(l)
                kc = rng.standard_normal((1, context, wl.CHAIN_HIDDEN)) * 0.6
                vc = rng.standard_normal((1, context, wl.CHAIN_HIDDEN)) * 0.6
                y = self.O.chain_layer_attention(y, self.layers[l % 2], kc, vc, context - 1, wl.CHAIN_HEADS)
            else:
                y = self.O.chain_layer(y, self.layers[l % 2])
        return len(x)


def chain_cpu_baseline(budget_s=4.0, oracle=None, context: int = 0):
    o = oracle or ChainOracle()
    x = wl.chain_input(1)
    tokens, n, dt = _timed_loop(lambda: o.step(x, context), budget_s)
    what = f"at position {context - 1} over a {context}-key cache " if context else ""
    return {"value": tokens / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} passes of 1 token {what}through all {CHAIN_LAYERS} layers of the numpy oracle "
                      f"(numpy, single thread)"}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on the headline workload
    (or --workload), rank 0 only; each step is a bounded sample of it."""
    if rank != 0:
        return None
    name = HEADLINE if args.workload == "all" else args.workload
    warmup = max(3, args.warmup)
    if name in CHAIN_WORKLOADS:
        o = ChainOracle()
        x = wl.chain_input(1)
        for _ in range(warmup):
            o.step(x)
        t0 = time.perf_counter()
        tokens = sum(o.step(x) for _ in range(args.steps))
        dt = time.perf_counter() - t0
        sample = f"each step: 1 token through all {CHAIN_LAYERS} layers of the numpy oracle"
        config = {"workload": f"bitlinear_chain_{CHAIN_LAYERS}layers_m{CHAIN_WORKLOADS[name]}_hidden"
                              f"{wl.CHAIN_HIDDEN}_ffn{wl.CHAIN_FFN}", "M_tokens": CHAIN_WORKLOADS[name],
                  "layers": CHAIN_LAYERS}
        dtype = "int8/int4 x ternary -> int64, fp32 glue"
    else:
        c = WORKLOADS[name]()
        step = oracle_step_fn(c)
        rows = sample_rows(c)
        for _ in range(warmup):
            step(rows)
        t0 = time.perf_counter()
        tokens = sum(step(rows) for _ in range(args.steps))
        dt = time.perf_counter() - t0
        sample = f"each step: {len(rows)} tokens of {c['name']} through the numpy oracle"
        config = {"workload": c["name"], "M_tokens": c["M"], "K": c["K"], "N": c["N"], "act_bits": c["act_bits"]}
        dtype = "int8xternary->int64" if c["act_bits"] == 8 else "int4xternary->int64"
    value = tokens / dt
    config["parallelism"] = "rank 0 only (CPU oracle)"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def add_cpu_baselines(subs):
    """cpu_baseline (numpy oracle, one core) and cpu_baseline_all_cores (C++
    oracle, OpenMP) for every configuration that ran."""
    chain_oracle = None
    for name, sub in subs.items():
        if name in CHAIN_WORKLOADS:
            chain_oracle = chain_oracle or ChainOracle()
            att = CHAIN_ATTENTION.get(name)
            sub["cpu_baseline"] = chain_cpu_baseline(oracle=chain_oracle,
                                                     context=0 if att is None else att[2] + att[1])
            continue
        c = WORKLOADS[name]()
        sub["cpu_baseline"] = cpu_baseline(c)
        try:
            sub["cpu_baseline_all_cores"] = cpu_baseline_omp(c)
        except Exception as e:                       # e.g. no C++ compiler on the host
            sub["cpu_baseline_all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}


# ----------------------------------------------------------------------------
# driver
# ----------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch

    from bitlinear_bitnet_quant_b200 import api, build_lib

    build_lib.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    visible = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    clocks = ClockSampler(visible[local_rank] if local_rank < len(visible) else str(local_rank)).start()
    timer = Timer(stream, world, dev, args.steps, args.min_time, clocks)
    ctx = {"api": api, "rank": rank, "world": world, "dev": dev, "stream": stream, "timer": timer,
           "clocks": clocks, "peaks": load_peaks()}
    ctx["int8_peak"] = measure_int8_peak(api, stream, torch.cuda.get_device_properties(dev).multi_processor_count)
    names = ORDER if args.workload == "all" else [args.workload]
    subs = {}
    try:
        for name in names:
            subs[name] = (run_chain if name in CHAIN_WORKLOADS else run_layer)(name, args, ctx)
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        if api.bitnet_device_error() != 0:
            raise RuntimeError("a kernel reported a device-side wait timeout")
    finally:
        overall = clocks.stop()
    if rank != 0:
        return None
    if world == 1 and not args.no_cpu_baseline:
        add_cpu_baselines(subs)

    head_name = HEADLINE if HEADLINE in subs else names[-1]
    head = subs[head_name]
    steps = args.steps
    launches = head["gpu_launches_per_step"] * head["timing"]["steps_per_replay"] * head["timing"]["replays"]
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": max(3, args.warmup), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("int8/int4 x ternary -> int32, fp32 glue" if head_name in CHAIN_WORKLOADS else
                  "int8xternary->int32" if head["act_bits"] == 8 else "int4xternary->int32"),
        "data": "synthetic",
        "config": {k: head[k] for k in ("workload", "M_tokens", "layers", "hidden", "ffn", "K", "N", "act_bits",
                                        "l2") if k in head},
        "roofline": head["roofline"],
        "timing": head["timing"],
        "e2e": head["e2e"],
        "gpu_launches": launches,
        "clocks": head["clocks"] or overall,
        "kernels_us": head["kernels_us"],
    }
    line["config"]["timing"] = ("R replays of a CUDA graph of K steps between a barrier and a device synchronise "
                                "on both sides; CUDA events around each replay on the launching stream; median")
    line["config"]["parallelism"] = f"dp{world} (independent batches per rank)"
    for k in ("step_roofline", "cpu_baseline", "cpu_baseline_all_cores", "attention", "quant_roofline",
              "decode_variants", "weights_quant"):
        if k in head:
            line[k] = head[k]
    line["configs"] = {n: s for n, s in subs.items() if n != head_name}
    line["int8_peak_measured"] = ctx["int8_peak"]
    line["clocks_whole_run"] = overall
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", choices=["all"] + ORDER, default="all")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--min-time", type=float, default=0.5, help="seconds of graph replays per timed region")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    world = max(world, 1)

    if args.impl == "reference":
        line = run_reference(args, rank, world)
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
        line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
