#!/usr/bin/env python
"""Benchmark of the hybrid MoE feed-forward block (Gemma-4-26B-A4B shape) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill]

A step is one moe_block_forward (router -> permute -> experts + dense MLP -> combine,
post norms, residual) over one batch of synthetic tokens.  The default workload is the
decode layer: T=8 tokens, H=2816, E=128, top-8, expert intermediate 704, dense
intermediate 2112, bf16 weights N(0, 0.02), activations N(0, 1), gains U(0.5, 1.5).
Steps rotate over distinct layer copies (and distinct inputs) so that no step finds
its weights in L2.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (numpy, fp64) on the same workload instead, on a
bounded sample per step; it is the baseline arm, not a GPU path.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = ("MoE-FFN tokens/s (1 B200) at T=8..16K; % HBM roofline (decode) / "
          "% TC peak (prefill)")
UNIT = "tokens/s"

WORKLOADS = {
    "decode": dict(shape=synth.DECODE, layers=8, steps=3000, warmup=100,
                   name="Gemma-4-26B-A4B-shaped MoE-FFN layer, decode T=8 (bf16 experts)"),
    "decode_T1": dict(shape=synth.Shape(T=1, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                      steps=3000, warmup=100,
                      name="Gemma-4-26B-A4B-shaped MoE-FFN layer, decode T=1 (bf16 experts)"),
    "decode_T64": dict(shape=synth.Shape(T=64, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                       steps=2000, warmup=100,
                       name="Gemma-4-26B-A4B-shaped MoE-FFN layer, T=64 (bf16 experts)"),
    "prefill": dict(shape=synth.PREFILL, layers=4, zipf=True, steps=300, warmup=10,
                    name="Gemma-4-26B-A4B-shaped MoE-FFN layer, prefill T=2048, Zipf-skewed router"),
    "int8_T1": dict(shape=synth.Shape(T=1, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                    int8=True, steps=3000, warmup=100,
                    name="same layer with per-channel int8 experts, T=1"),
    "int8_T64": dict(shape=synth.Shape(T=64, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                     int8=True, steps=2000, warmup=100,
                     name="same layer with per-channel int8 experts, T=64"),
    "int8_T1024": dict(shape=synth.Shape(T=1024, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                       int8=True, steps=500, warmup=20,
                       name="same layer with per-channel int8 experts, T=1024"),
    "fp8_T8": dict(shape=synth.DECODE, layers=8, fp8=True, steps=3000, warmup=100,
                   name="same layer with E4M3 experts and per-token E4M3 activations, T=8"),
    "fp8_T64": dict(shape=synth.Shape(T=64, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                    fp8=True, steps=2000, warmup=100,
                    name="same layer with E4M3 experts and per-token E4M3 activations, T=64"),
    "fp8_T1024": dict(shape=synth.Shape(T=1024, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                      fp8=True, steps=500, warmup=20,
                      name="same layer with E4M3 experts and per-token E4M3 activations, T=1024"),
    "nvfp4_T1": dict(shape=synth.Shape(T=1, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                     nvfp4=True, steps=3000, warmup=100,
                     name="same layer with NVFP4 experts (weight-only), T=1"),
    "nvfp4_T64": dict(shape=synth.Shape(T=64, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                      nvfp4=True, steps=2000, warmup=100,
                      name="same layer with NVFP4 experts (weight-only), T=64"),
    "nvfp4_T1024": dict(shape=synth.Shape(T=1024, H=2816, E=128, k=8, I=704, D=2112), layers=8,
                        nvfp4=True, steps=500, warmup=20,
                        name="same layer with NVFP4 experts (weight-only), T=1024"),
    "stack": dict(shape=synth.Shape(T=synth.STACK_T, H=2816, E=128, k=8, I=704, D=2112),
                  layers=synth.STACK_LAYERS, chain=True, steps=3, warmup=1,
                  name="stack of 30 distinct MoE-FFN layers, residual-chained, T=16384 (one 16K chunk)"),
}
ZIPF_ALPHA_FILE = os.path.join(ROOT, "tests", "golden", "zipf_alpha.json")

# The default run measures the headline workload (decode, T=8) with the requested
# --steps/--warmup, then, on one GPU, every other workload with these step counts (each
# a few seconds of GPU time; the stack's steps are 30 chained layers each), so that one
# run of a few minutes carries every configuration.
SWEEP = {"decode_T1": (2000, 50), "decode_T64": (1000, 50), "prefill": (200, 10),
         "int8_T1": (2000, 50), "int8_T64": (1000, 50), "int8_T1024": (200, 10),
         "fp8_T8": (1000, 50), "fp8_T64": (1000, 50), "fp8_T1024": (200, 10),
         "nvfp4_T1": (2000, 50), "nvfp4_T64": (1000, 50), "nvfp4_T1024": (200, 10),
         "stack": (3, 2)}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------------------- ncu traffic

PROFILES = os.path.join(ROOT, "profiles")
GEMM_SOURCES = [os.path.join(ROOT, "mixture_experts_ffn_05_b200", "csrc", f)
                for f in ("grouped_gemm.cu", "common.cuh")]


def strip_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines (string and character literals,
    such as inline PTX, are kept as they are)."""
    out = []
    i, n = 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln.strip())


def kernel_sha() -> str:
    """Hash of the GEMM kernel's code: its sources without comments, so that the ncu
    counters recorded for a kernel stay attached to it across comment edits and are
    dropped as soon as any code changes."""
    import hashlib
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(f) as fh:
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()


def ncu_traffic(summary: str):
    """DRAM bytes per launch from a committed ncu summary, or None when the kernel's
    source has changed since the counters were taken."""
    try:
        vals = {}
        with open(os.path.join(PROFILES, summary)) as f:
            for line in f:
                if ":" in line:
                    k, v = line.strip().split(":", 1)
                    vals[k.strip()] = v.strip()
        if vals.get("source_sha256") != kernel_sha():
            return None
        return int(vals["traffic_bytes_per_launch"])
    except Exception:
        return None


def max_over_ranks(t_ms: float, world: int, device) -> float:
    """The slowest rank's time (every rank takes part)."""
    if world <= 1:
        return t_ms
    tt = torch.tensor([t_ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
    return float(tt.item())


# ---------------------------------------------------------------------------- clocks

class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            return None
        return parse_clock_samples(out)


def parse_clock_samples(text: str):
    """Clock record of nvidia-smi samples (`Clocks.FIELDS`, csv, no header, no units):
    median SM clock, the largest max clock, and every throttle reason seen Active in any
    sample; None without a usable sample."""
    rows = []
    for line in text.splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) != 8:
            continue
        try:
            rows.append((float(parts[0]), float(parts[1]), parts[4:]))
        except ValueError:
            continue
    if not rows:
        return None
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
    return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
            "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------- work model

def algorithmic(shape, used_experts: int, int8: bool = False, nvfp4: bool = False):
    """Bytes that must move and FLOPs that must run for one block call.

    Bytes: the weights of the experts that received a token (int8 or E4M3 codes plus
    fp32 row scales for 8-bit experts: `int8` means any 1-byte weight here; NVFP4: half a
    byte per weight, one E4M3 block scale per 16 weights, an fp32 scale per matrix), the
    dense MLP, the router and the norm vectors, plus x in and out.  Intermediates are
    implementation traffic.
    """
    H, E, k, I, D, T = shape.H, shape.E, shape.k, shape.I, shape.D, shape.T
    if nvfp4:
        wb = 0.5 + 1.0 / 16
        sc_gu, sc_all = 4, 8
    else:
        wb = 1 if int8 else 2
        sc_gu, sc_all = (2 * I * 4, (2 * I + H) * 4) if int8 else (0, 0)
    b_experts = used_experts * (3 * I * H * wb + sc_all)
    b_dense = 3 * D * H * 2
    b = b_experts + b_dense + E * H * 2 + 6 * H * 2 + E * 2 + 2 * T * H * 2
    flops = T * (2 * k * 3 * I * H + 2 * 3 * D * H + 2 * E * H)
    # the gate_up launch alone: its weights, its token rows in, h out
    b_gate_up = (used_experts * (2 * I * H * wb + sc_gu) + 2 * D * H * 2
                 + (T * k + T) * H * 2 + (T * k * I + T * D) * 2)
    f_gate_up = T * (2 * k * 2 * I * H + 2 * 2 * D * H)
    return {"bytes": b, "flops": flops, "gate_up_bytes": b_gate_up, "gate_up_flops": f_gate_up}


# ---------------------------------------------------------------------------- our arm

def workload_config(wl, world, nl, alpha):
    """The `config` object of a workload's JSON line (both arms print the same one)."""
    shape = wl["shape"]
    int8, fp8, nvfp4 = bool(wl.get("int8")), bool(wl.get("fp8")), bool(wl.get("nvfp4"))
    wbytes = 0.5 + 1.0 / 16 if nvfp4 else (1 if int8 or fp8 else 2)
    return {"workload": wl["name"], "T": shape.T, "H": shape.H, "E": shape.E, "top_k": shape.k,
            "expert_inter": shape.I, "dense_inter": shape.D,
            "expert_weights": ("int8 per-channel" if int8 else
                               "E4M3 per-channel, E4M3 per-token activations" if fp8 else
                               "NVFP4 (E2M1, E4M3 per 16, fp32 per matrix), weight-only" if nvfp4
                               else "bf16"),
            "router_bias": ("zipf s=1.1, alpha=%.5f" % alpha) if wl.get("zipf") else "none",
            "layers": nl, "chained": bool(wl.get("chain")),
            "l2": ("steps rotate over %d distinct layers (%.1f GB of weights) and distinct "
                   "inputs; no step's weights are L2-resident" %
                   (nl, nl * 3 * shape.E * shape.I * shape.H * wbytes / 1e9)),
            "parallelism": f"dp{world} (replicas, no collective)"}


def zipf_alpha(wl):
    if not wl.get("zipf"):
        return None
    with open(ZIPF_ALPHA_FILE) as f:
        return float(json.load(f)["alpha"])


def _make_layers(mf, cfg, shape, wl, n, seed, device):
    layers, alpha = [], None
    for l in range(n):
        t = synth.torch_layer(shape, seed, l, device)
        if wl.get("zipf"):
            with open(ZIPF_ALPHA_FILE) as f:
                alpha = float(json.load(f)["alpha"])
            t["logit_bias"] = torch.from_numpy(synth.zipf_bias(seed, shape.E, alpha)).to(device)
        if wl.get("nvfp4"):
            for name, bname, sname in (("w_gate_up", "b_gate_up", "s_gate_up"),
                                       ("w_down", "b_down", "s_down")):
                w = t.pop(name)
                E_, rows, cols = w.shape
                q = torch.empty(E_, rows, cols // 2, dtype=torch.uint8, device=device)
                bs = torch.empty(E_, rows, cols // 16, dtype=torch.uint8, device=device)
                ts = torch.empty(E_, dtype=torch.float32, device=device)
                mf.moe_quantize_nvfp4(w, q, bs, ts)
                t[name], t[bname], t[sname] = q, bs, ts
                del w
        elif wl.get("int8") or wl.get("fp8"):
            for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down")):
                w = t.pop(name)
                cols = w.shape[-1]
                fp8 = bool(wl.get("fp8"))
                q = torch.empty(w.shape, dtype=torch.uint8 if fp8 else torch.int8, device=device)
                sc = torch.empty(w.shape[:-1], dtype=torch.float32, device=device)
                quant = mf.moe_quantize_fp8 if fp8 else mf.moe_quantize_int8
                quant(w.view(-1, cols), q.view(-1, cols), sc.view(-1))
                t[name], t[sname] = q, sc
                del w
        layers.append(t)
    torch.cuda.synchronize(device)
    return layers, alpha


def run_ours(args, wl, rank, world, device, K=None, W=None, headline=True):
    """One workload: K timed steps after W warm-up steps.  The headline adds the
    end-to-end run, the launch count and the CPU baseline."""
    import mixture_experts_ffn_05_b200 as mf
    mf.lib()  # fails loudly without the built CUDA library
    shape = wl["shape"]
    T = shape.T
    int8 = bool(wl.get("int8"))
    fp8 = bool(wl.get("fp8"))
    nvfp4 = bool(wl.get("nvfp4"))
    chain = bool(wl.get("chain"))
    cfg = mf.Config(shape.H, shape.E, shape.k, shape.I, shape.D, shape.eps, int8, fp8, nvfp4)
    seed = 1234 + 7919 * rank
    nl = args.layers or wl["layers"]
    layers, alpha = _make_layers(mf, cfg, shape, wl, nl, seed, device)
    bws = [mf.BlockWeights(cfg, t) for t in layers]
    W = args.warmup if W is None else W
    K = args.steps if K is None else K
    xs = [synth.torch_x(shape, seed, i, device) for i in range(W + K)]
    out = torch.empty(T, shape.H, dtype=torch.bfloat16, device=device)
    bufs = [torch.empty_like(out), torch.empty_like(out)]
    ws = mf.workspace(cfg, T, device)
    stream = torch.cuda.current_stream(device)

    def calls(i, x=None, final=None):
        """(layer, input, output) of step i: one layer, or every layer chained."""
        x = xs[i] if x is None else x
        if not chain:
            return [(i % nl, x, out if final is None else final)]
        res, cur = [], x
        for l in range(nl):
            dst = (out if final is None else final) if l == nl - 1 else bufs[l % 2]
            res.append((l, cur, dst))
            cur = dst
        return res

    def step(i, evs=None, x=None, final=None):
        for c, (l, xin, dst) in enumerate(calls(i, x, final)):
            mf.moe_block_forward(cfg, xin, bws[l], dst, ws, stream=stream,
                                 stage_events=None if evs is None else evs[c])

    # experts that receive tokens in each timed call (outside the timed region)
    used = []
    ti = torch.empty(T, shape.k, dtype=torch.int32, device=device)
    tw = torch.empty(T, shape.k, dtype=torch.float32, device=device)
    xa = torch.empty(T, shape.H, dtype=torch.bfloat16, device=device)
    xb = torch.empty_like(xa)
    for i in range(K):
        for (l, xin, dst) in calls(W + i):
            L = layers[l]
            mf.moe_router(cfg, xin, L["router_scale"], L["w_router"], L.get("logit_bias"),
                          L["per_expert_scale"], L["g_pre_moe"], L["g_pre_dense"], ti, tw, xa, xb, ws)
            used.append(int(torch.unique(ti).numel()))
            if chain:
                mf.moe_block_forward(cfg, xin, bws[l], dst, ws, stream=stream)

    for i in range(W):
        step(i)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    ncalls = len(calls(0))
    stage_ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(mf.MOE_BLOCK_EVENTS)]
                 for _ in range(ncalls)] for _ in range(K)]
    for evs in stage_ev:  # create the CUDA events before the timed region
        for ev in evs:
            for e in ev:
                e.record(stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    clocks = Clocks(device)
    time.sleep(0.15)
    torch.cuda.synchronize(device)
    # timed region 1: the steps alone (events inside a step would order its kernels and
    # hide the overlap of consecutive launches)
    e0.record(stream)
    for i in range(K):
        step(W + i)
    e1.record(stream)
    torch.cuda.synchronize(device)
    # timed region 2: the same steps with events at every stage boundary, for the
    # duration of each kernel (the roofline of the dominant one)
    for i in range(K):
        step(W + i, stage_ev[i])
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    st = mf.moe_check_device_status(ws)
    if st != mf.MOE_OK:
        raise RuntimeError(f"device status after the timed region: {mf.status_string(st)}")
    t_ms = e0.elapsed_time(e1)
    stages = {n: [] for n in ("router", "permute", "gather", "gate_up", "down", "combine")}
    for evs in stage_ev:
        for ev in evs:
            for j, n in enumerate(stages):
                stages[n].append(ev[j].elapsed_time(ev[j + 1]))
    t_max = max_over_ranks(t_ms, world, device)
    te = None
    if headline:
        te = _e2e(mf, shape, xs, step, W, K, world, device, ws, stream)
    res = _report(mf, wl, shape, cfg, used, stages, t_max, K, W, world, nl, alpha, chain, int8,
                  fp8, nvfp4, clk, calls, te, headline)
    if headline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(shape, layers[0], xs[W], wl, alpha, nl if chain else 1)
    return res


def _e2e(mf, shape, xs, step, W, K, world, device, ws, stream):
    """The same steps end to end through the public API: pinned host input copied in and
    the output copied out inside the timed region.  Returns the slowest rank's ms."""
    T = shape.T
    x_host = torch.empty(W + K, T, shape.H, dtype=torch.bfloat16, pin_memory=True)
    for i in range(W + K):
        x_host[i].copy_(xs[i])
    out_host = torch.empty(K, T, shape.H, dtype=torch.bfloat16, pin_memory=True)
    x_dev = torch.empty(T, shape.H, dtype=torch.bfloat16, device=device)
    y_dev = torch.empty_like(x_dev)

    def e2e_step(i, j):
        x_dev.copy_(x_host[i], non_blocking=True)
        step(i, x=x_dev, final=y_dev)
        out_host[j].copy_(y_dev, non_blocking=True)

    for i in range(min(W, 10)):
        e2e_step(i, 0)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(K):
        e2e_step(W + i, i)
    f1.record(stream)
    torch.cuda.synchronize(device)
    te = max_over_ranks(f0.elapsed_time(f1), world, device)
    if mf.moe_check_device_status(ws) != mf.MOE_OK:
        raise RuntimeError("device status after the end-to-end region")
    return te


def _report(mf, wl, shape, cfg, used, stages, t_max, K, W, world, nl, alpha, chain, int8, fp8,
            nvfp4, clk, calls, te, headline):
    T = shape.T
    # ---- roofline of the dominant kernel (the gate_up grouped GEMM) and of the block
    pk = peaks()
    long_step = t_max / K > 10.0  # ms: a kernel inside a long step meets the sustained peak
    tc_peak = pk["bf16_tflops_sustained"] if long_step else pk["bf16_tflops"]
    # an E4M3 contraction's peak: the measured bf16 peak times the nominal fp8:bf16 ratio
    # (4.5 : 2.25 PFLOP/s dense); only the routed experts' matmuls run in fp8, so the
    # gate_up launch's peak is the FLOP-weighted mix
    alg = [algorithmic(shape, u, int8 or fp8, nvfp4) for u in used]
    gu_ms = sum(stages["gate_up"])
    gu_bytes = sum(a["gate_up_bytes"] for a in alg)
    gu_flops = sum(a["gate_up_flops"] for a in alg)
    gu_gbs = gu_bytes / (gu_ms * 1e-3) / 1e9
    gu_tf = gu_flops / (gu_ms * 1e-3) / 1e12
    blk_bytes = sum(a["bytes"] for a in alg) / K
    blk_flops = sum(a["flops"] for a in alg) / K
    ms_step = t_max / K
    gu_t_hbm = gu_bytes / (pk["hbm_gbs"] * 1e9)
    gu_t_tc = gu_flops / (tc_peak * 1e12)
    streaming = nvfp4 or (int8 and T <= 256)  # the library's choice of GEMM kernel
    kern = ("stream_gemm_kernel (gate_up launch, " + ("NVFP4" if nvfp4 else "int8") +
            " weights widened in registers)" if streaming else
            "grouped_gemm_kernel (gate_up launch" + (", int8 converter variant)" if int8 else
                                                      ", E4M3 experts)" if fp8 else ")"))
    if fp8:
        f_exp = 2 * shape.k * 2 * shape.I * shape.H
        f_den = 2 * 2 * shape.D * shape.H
        tc_peak = round(tc_peak * (f_exp + f_den) / (f_exp / 2.0 + f_den), 1)
    if gu_t_tc > gu_t_hbm:
        roof = {"bound": "tensor", "achieved": round(gu_tf, 2), "peak": tc_peak,
                "unit": "TFLOP/s", "frac": round(gu_tf / tc_peak, 4), "traffic": None,
                "kernel": kern,
                "peak_source": ("bf16_tflops_sustained" if long_step else "bf16_tflops")
                               + f" of {pk['source']} peaks"}
    else:
        summary = {(8, False): "grouped_gemm_gate_up_decode_T8.md"}.get((T, int8 or fp8))
        roof = {"bound": "hbm", "achieved": round(gu_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(gu_gbs / pk["hbm_gbs"], 4),
                "traffic": ncu_traffic(summary) if summary else None,
                "kernel": kern, "peak_source": f"hbm_gbs of {pk['source']} peaks"}
    t_hbm = blk_bytes / (pk["hbm_gbs"] * 1e9)
    t_tc = blk_flops / (tc_peak * 1e12)
    block_roof = {"bytes_per_step": int(blk_bytes), "flops_per_step": int(blk_flops),
                  "hbm_frac": round(t_hbm / (ms_step * 1e-3), 4),
                  "tc_frac": round(t_tc / (ms_step * 1e-3), 4),
                  "binding_frac": round(max(t_hbm, t_tc) / (ms_step * 1e-3), 4),
                  "mean_used_experts": round(sum(used) / len(used), 2)}
    launches_per_call = mf.moe_block_launch_count(cfg, T)  # the library's own count
    ncalls = len(calls(0))
    if not headline:
        return {"workload": wl["name"], "steps": K, "warmup": W, "ms_per_step": round(ms_step, 5),
                "value": round(world * T * K / (t_max * 1e-3), 1), "unit": UNIT,
                "dtype": "e4m3 x e4m3 (experts), bf16 (dense)" if fp8 else
                         ("int8 weights, fp16 activations (experts), bf16 (dense)" if int8 else
                          "nvfp4 weights, fp16 activations (experts), bf16 (dense)" if nvfp4 else
                          "bf16"),
                "config": workload_config(wl, world, nl, alpha),
                "roofline": roof, "block_roofline": block_roof,
                "stages_ms": {n: round(statistics.mean(v), 5) for n, v in stages.items()},
                "gpu_launches_per_step": launches_per_call * ncalls, "clocks": clk}
    res = {
        "metric": METRIC, "value": round(world * T * K / (t_max * 1e-3), 1), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 x e4m3 (experts), bf16 (dense)" if fp8 else "bf16",
        "data": "synthetic (seeded; random-init weights of the layer's shape)",
        "config": workload_config(wl, world, nl, alpha),
        "roofline": roof,
        "block_roofline": block_roof,
        "stages_ms": {n: round(statistics.mean(v), 5) for n, v in stages.items()},
        "e2e": {"value": round(world * T * K / (te * 1e-3), 1), "unit": UNIT,
                "h2d_bytes_per_step": T * shape.H * 2, "d2h_bytes_per_step": T * shape.H * 2},
        "gpu_launches": launches_per_call * ncalls * K,
        "clocks": clk,
    }
    return res


# ---------------------------------------------------------------------------- the oracle

def _host_layer(layer):
    out = {}
    for n, t in layer.items():
        if t.dtype == torch.bfloat16:
            out[n] = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        else:
            out[n] = t.cpu().numpy()
    return out


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


REF_BUDGET_S = 120.0  # the reference arm's timed region, about


def _oracle_rows(shape):
    return shape.T if shape.T <= 64 else 64


def _oracle_experts(p):
    import oracle
    if "s_gate_up" in p:
        return oracle.Experts(q_gate_up=p["w_gate_up"], s_gate_up=p["s_gate_up"],
                              q_down=p["w_down"], s_down=p["s_down"])
    return oracle.Experts(w_gate_up=p["w_gate_up"], w_down=p["w_down"])


def cpu_baseline(shape, layer, x, wl, alpha, layers_per_step=1, budget_s=15.0):
    """The oracle, as it stands, on the host cores: tokens/s over a bounded sample.
    For the chained stack one layer is timed and the rate divided by the layer count."""
    import oracle
    p = _host_layer(layer)
    bias = p.pop("logit_bias", None)
    ex = _oracle_experts(p)
    rows = _oracle_rows(shape)
    xh = x[:rows].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.block_forward(xh, p, ex, shape.k, shape.eps, bias)
        n += 1
        el = time.perf_counter() - t0
        if el > budget_s or n >= 200:
            break
    extra = (f"; one layer timed, rate divided by {layers_per_step} layers"
             if layers_per_step > 1 else "")
    return {"value": round(n * rows / el / layers_per_step, 3), "unit": UNIT,
            "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{n} oracle block calls of {rows} tokens of the {wl['name']} workload "
                      f"(layer 0), {el:.1f} s{extra}"}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return None
    import oracle
    shape = wl["shape"]
    layer = synth.torch_layer(shape, 1234, 0, "cpu")
    alpha = zipf_alpha(wl)
    p = _host_layer(layer)
    bias = synth.zipf_bias(1234, shape.E, alpha) if wl.get("zipf") else None
    if wl.get("int8"):
        qg, sg = oracle.quantize_int8_per_channel(p["w_gate_up"])
        qd, sd = oracle.quantize_int8_per_channel(p["w_down"])
        ex = oracle.Experts(q_gate_up=qg, s_gate_up=sg, q_down=qd, s_down=sd)
    elif wl.get("fp8"):
        qg, sg = oracle.quantize_fp8_per_channel(p["w_gate_up"])
        qd, sd = oracle.quantize_fp8_per_channel(p["w_down"])
        ex = oracle.Experts(q_gate_up=qg, s_gate_up=sg, q_down=qd, s_down=sd, fp8=True)
    elif wl.get("nvfp4"):
        ex = oracle.Experts(nvfp4={
            part: [oracle.quantize_nvfp4(p[name][e]) for e in range(shape.E)]
            for part, name in (("gate_up", "w_gate_up"), ("down", "w_down"))})
    else:
        ex = oracle.Experts(w_gate_up=p["w_gate_up"], w_down=p["w_down"])
    per_step = wl["layers"] if wl.get("chain") else 1
    # Each step is one oracle call on a bounded sample of the step's token rows, sized
    # from a timed calibration call so that the K timed steps take about REF_BUDGET_S
    # (at least one row per step): any --steps stays within a few minutes.
    rows = _oracle_rows(shape)

    def host_x(i, n):
        return synth.torch_x(shape, 1234, i, "cpu")[:n].contiguous().view(torch.int16).numpy().view(np.uint16)

    tc = time.perf_counter()
    oracle.block_forward(host_x(0, rows), p, ex, shape.k, shape.eps, bias)
    per_row = (time.perf_counter() - tc) / rows
    rows = max(1, min(rows, int(REF_BUDGET_S / (args.steps * per_row))))
    xs = [host_x(i, rows) for i in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        oracle.block_forward(xs[i], p, ex, shape.k, shape.eps, bias)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.block_forward(xs[args.warmup + i], p, ex, shape.k, shape.eps, bias)
    el = time.perf_counter() - t0
    v = round(args.steps * rows / el / per_step, 3)
    sample = (f"{args.steps} timed oracle block calls of {rows} of the {shape.T} tokens of a "
              f"step each ({wl['name']}; layer 0)") + (
        f"; one layer per call, rate divided by {per_step} layers" if per_step > 1 else "")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el * 1e3 / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": workload_config(wl, world, args.layers or wl["layers"], alpha),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default=None,
                    help="one workload only (default: the decode headline, then every other "
                         "workload on one GPU)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None, help="layer copies to rotate over")
    args = ap.parse_args()
    sweep = args.workload is None
    wl = WORKLOADS[args.workload or "decode"]
    if args.impl == "reference":
        args.steps = args.steps if args.steps is not None else 10
        args.warmup = args.warmup if args.warmup is not None else 3
    else:
        args.steps = args.steps if args.steps is not None else wl["steps"]
        args.warmup = args.warmup if args.warmup is not None else wl["warmup"]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, wl, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        res = run_ours(args, wl, rank, world, device)
        if sweep and world == 1:
            # every other workload, each with its own step counts; its weights are freed
            # before the next one is built
            res["workloads"] = {}
            for name, (k, w) in SWEEP.items():
                torch.cuda.empty_cache()
                res["workloads"][name] = run_ours(args, WORKLOADS[name], rank, world, device,
                                                  K=k, W=w, headline=False)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
