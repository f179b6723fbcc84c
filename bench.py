#!/usr/bin/env python3
"""Throughput of the W4A4 + low-rank linear layer on B200.

Workload (one GPU): the Llama-3-8B attention projection in the decode
regime, K = N = 4096, rank 32, Hadamard block 128, M = 16 tokens (other M via
--m).  One "step" is one pass of the hot path -- rotation, per-token INT4
codes, X L1, INT4 GEMM with INT32 accumulation, bf16 low-rank branch and the
shared epilogue, one tq_w4a4_lr_layer call (one fused kernel) per layer --
over 16 distinct layers, so the 16 x 9.2 MB of operands (147 MB) exceed the
126 MB L2 and every layer streams its weights from HBM.  The offline weight
packing is not part of a step.  A step is replayed as one CUDA graph.
--workload prefill_gateup|prefill_down|large_gateup|large_down|sweep times
tq_quantize_act + tq_w4a4_lr_gemm on the prefill and sweep shapes instead;
--workload sweeps runs the roofline sweeps at K = N = 4096 (M from 1 to 8192
at rank 64, rank from 0 to 512 at M = 4096) through tq_w4a4_lr_layer;
--workload gateup_swiglu times the MLP's gate and up projections as one
shared-input pair with the SwiGLU epilogue (tq_w4a4_lr_gate_up) against the
two projections as separate tq_w4a4_lr_layer calls; --workload qlr times the
layer with the INT4 low-rank branch against the same layer with the bf16
branch (prefill gate/up shape).

Metric: algorithmic GB/s of the layer (X + L1^T + Wq + s_w + L2^T + Y bytes
per layer), the decode roofline quantity; TOPS (2 M N K) is reported beside it.

--impl reference times the CPU oracle (fp64 C, the parity reference) on a
bounded sample of the same workload.

Multi-GPU (torchrun): every rank runs its own independent batch of layers
(weak scaling, no data-path collective); rank 0 prints max-over-ranks time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4+low-rank linear TOPS and GB/s at Llama-3 shapes; % of INT8/HBM roofline"
K_DIM = N_DIM = 4096
RANK = 32
HAD = 128
LAYERS = 16


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--m", type=int, default=16, help="tokens per layer")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--no-sweep", action="store_true", help="skip the M=1/128 side measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill configurations and the rank-overhead point")
    ap.add_argument("--profile", action="store_true",
                    help="replay only the timed step graph (for a profiler); prints one status line")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "prefill_gateup", "prefill_down", "large_gateup",
                             "large_down", "sweep", "sweeps", "gateup_swiglu", "qlr", "qkv", "rht"],
                    help="decode is the default workload; the others are the prefill "
                         "shapes, scored in TOPS against the dense INT8 peak")
    ap.add_argument("--rank", type=int, default=None, help="low-rank r override (sweep)")
    return ap.parse_args()


def layer_bytes(M, K, N, r):
    """Algorithmic bytes of one layer: X + L1^T + Wq + s_w + L2^T + Y."""
    return 2 * M * K + 2 * r * K + K * N // 2 + 4 * N + 2 * N * r + 2 * M * N


def gemm_bytes(M, K, N, r):
    """Compulsory bytes of the GEMM kernel: Xq + s_x + XL1 + Wq + s_w + L2^T + Y."""
    return M * K // 2 + 4 * M + 4 * M * r + K * N // 2 + 4 * N + 2 * N * r + 2 * M * N


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return 6650.0, "fallback (6.65 TB/s, earlier measurement on this pool)"


def int8_peak(sustained: bool):
    """Dense INT8 tensor peak: the measured bf16 cuBLAS peak times the nominal
    INT8/bf16 ratio of B200 (4.5 / 2.25 = 2)."""
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return 2.0 * float(d[key]), f"measured bf16 ({key}) x 2 nominal INT8/bf16 ratio"
    except Exception:
        return 2.0 * (1400.0 if sustained else 1590.0), "fallback bf16 x 2"


def profiled_traffic(kernel_src: str, profile: str):
    """DRAM bytes per launch recorded in a committed ncu summary, or None when
    the summary is missing or was taken on a different kernel source."""
    try:
        txt = open(os.path.join(ROOT, "profiles", profile)).read()
        src = open(os.path.join(ROOT, kernel_src), "rb").read()
    except OSError:
        return None
    m_h = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    m_t = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m_h or not m_t or m_h.group(1) != hashlib.sha256(src).hexdigest():
        return None
    return float(m_t.group(1))


class ClockSampler:
    """Samples SM clocks and throttle reasons through NVML while running."""

    def __init__(self, index: int, period: float = 0.005):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksThrottleReasonSwPowerCap", 0x4),
        }
        while True:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            if self._stop.wait(self.period):
                break

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2] if s else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(s)}


# ----------------------------------------------------------------- GPU arm

def build_layers(tq, torch, M, L, seed0, device):
    import synth
    sh = synth.CONFIGS["decode"].with_(M=M)
    layers = []
    for i in range(L):
        w = synth.make_weights(sh, seed=seed0 + 10 * i, device="cuda")
        Rt = w["Rt"].to(device)
        Wq, s_w = tq.tq_pack_weight(Rt, HAD)
        lay = {
            "Rt": Rt if i == 0 else None,
            "X": synth.make_activations(sh, seed=seed0 + 10 * i).to(device),
            "L1t": w["L1t"].to(device), "L2t": w["L2t"].to(device), "Wq": Wq, "s_w": s_w,
            "Xq": torch.empty(M, K_DIM // 2, dtype=torch.uint8, device=device),
            "s_x": torch.empty(M, dtype=torch.float32, device=device),
            "XL1": torch.empty(M, RANK, dtype=torch.float32, device=device),
            "Y": torch.empty(M, N_DIM, dtype=torch.bfloat16, device=device),
            "ws": torch.zeros(tq.tq_gemm_workspace_bytes(M, N_DIM, K_DIM, RANK),
                              dtype=torch.uint8, device=device),
            "lws": torch.zeros(tq.tq_layer_workspace_bytes(M, N_DIM, K_DIM, RANK),
                               dtype=torch.uint8, device=device),
        }
        layers.append(lay)
    # a stack of layers as in a decode step: layer i reads layer i-1's output
    # (K = N), so every layer waits for its predecessor and finds its input in
    # L2, as a model's next layer does; layer 0 reads the synthetic X
    for prev, lay in zip(layers, layers[1:]):
        lay["X"] = prev["Y"]
    torch.cuda.synchronize()
    return layers


def layer_call(tq, lay, ev=None):
    """The layer through tq_w4a4_lr_layer (one fused kernel at these sizes)."""
    if ev is not None:
        ev[0].record()
    tq.tq_w4a4_lr_layer(lay["X"], lay["L1t"], lay["Wq"], lay["s_w"], lay["L2t"], HAD,
                        Y=lay["Y"], workspace=lay["lws"])
    if ev is not None:
        ev[1].record()


def layer_call_two(tq, lay):
    """The same layer through the two-call path (tq_quantize_act, tq_w4a4_lr_gemm)."""
    tq.tq_quantize_act(lay["X"], HAD, lay["L1t"], Xq=lay["Xq"], s_x=lay["s_x"], XL1=lay["XL1"])
    tq.tq_w4a4_lr_gemm(lay["Xq"], lay["s_x"], lay["Wq"], lay["s_w"], lay["XL1"], lay["L2t"],
                       Y=lay["Y"], workspace=lay["ws"])


def capture(torch, fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # one eager pass (function attributes, tensor maps) before capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The slowest rank's value (every rank gets it); identity on one rank.
    The tensor lives on `device`: a CUDA device under NCCL, the CPU under gloo."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank: int) -> int:
    """Seed base of a rank's independent batch of layers (weak scaling: every
    rank streams its own weights, no data-path collective)."""
    return 1000 * rank


def whole_job(per_rank_units: float, world: int, ms: float) -> float:
    """Units per second of all ranks together, timed by the slowest rank."""
    return world * per_rank_units / (ms * 1e-3)


def time_graph(torch, g, steps, warmup, dist=None):
    for _ in range(warmup):
        g.replay()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return e0.elapsed_time(e1) / steps  # ms per step


def run_tq(args, rank, world, local_rank, dist):
    import torch

    import rank_int4_gemm_b200 as tq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    M, L = args.m, args.layers
    layers = build_layers(tq, torch, M, L, seed0=replica_seed(rank), device=dev)

    def step():
        for lay in layers:
            layer_call(tq, lay)

    g = capture(torch, step)
    if args.profile:
        time_graph(torch, g, args.steps, args.warmup)
        return {"profile": "decode step graph", "layers": L, "steps": args.steps, "warmup": args.warmup}

    with ClockSampler(local_rank) as clk:
        ms = time_graph(torch, g, args.steps, args.warmup, dist if world > 1 else None)
    clocks = clk.summary()
    ms = max_over_ranks(ms, dist if world > 1 else None, dev)

    # per-kernel durations of the same step, events captured in the graph
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in layers]

    def step_ev():
        for lay, ev in zip(layers, evs):
            layer_call(tq, lay, ev)

    g_ev = capture(torch, step_ev)
    reps = max(1, min(args.steps, 50))
    gemm_ms = []
    for _ in range(max(3, args.warmup)):
        g_ev.replay()
    for _ in range(reps):
        g_ev.replay()
        torch.cuda.synchronize()
        gemm_ms.extend(a.elapsed_time(b) for a, b in evs)
    gemm_ms_avg = sum(gemm_ms) / len(gemm_ms)

    # end to end: the step's input (layer 0's X) from pinned host memory in,
    # its result (the last layer's Y) to pinned host memory out, every step
    hx = [layers[0]["X"].cpu().pin_memory()]
    hy = [torch.empty_like(layers[-1]["Y"], device="cpu").pin_memory()]

    def step_e2e():
        layers[0]["X"].copy_(hx[0], non_blocking=True)
        step()
        hy[0].copy_(layers[-1]["Y"], non_blocking=True)

    g_e2e = capture(torch, step_e2e)
    ms_e2e = time_graph(torch, g_e2e, args.steps, args.warmup, dist if world > 1 else None)
    ms_e2e = max_over_ranks(ms_e2e, dist if world > 1 else None, dev)

    # the two-call path on the same layers, for comparison
    g_two = capture(torch, lambda: [layer_call_two(tq, l) for l in layers])
    ms_two = time_graph(torch, g_two, args.steps, args.warmup)
    del g_two

    sweep = {}
    if not args.no_sweep and world == 1:
        for m2 in (1, 128):
            if m2 == M:
                continue
            ls = build_layers(tq, torch, m2, L, seed0=7, device=dev)

            def st(ls=ls):
                for lay in ls:
                    layer_call(tq, lay)

            g2 = capture(torch, st)
            ms2 = time_graph(torch, g2, args.steps, args.warmup)
            b2 = L * layer_bytes(m2, K_DIM, N_DIM, RANK)
            sweep[f"M={m2}"] = {"GB/s": round(b2 / ms2 / 1e6, 1), "us_per_layer": round(ms2 * 1e3 / L, 3),
                                "TOPS": round(L * 2 * m2 * N_DIM * K_DIM / ms2 / 1e9, 3)}
            del ls, g2

    bytes_step = L * layer_bytes(M, K_DIM, N_DIM, RANK)
    value = whole_job(bytes_step, world, ms) / 1e9        # GB/s, all ranks
    e2e = whole_job(bytes_step, world, ms_e2e) / 1e9
    peak, peak_src = measured_peaks()
    gb = layer_bytes(M, K_DIM, N_DIM, RANK)   # the fused kernel reads X, writes Y
    # the step is L launches of the one fused kernel, back to back (each
    # overlaps its predecessor's tail): average launch duration = step / L
    kernel_ms = ms / L
    achieved = gb / (kernel_ms * 1e-3) / 1e9
    traffic = profiled_traffic("rank_int4_gemm_b200/csrc/tq_decode.cu",
                               "w4a4_lr_decode_m16.md") if M == 16 else None
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4",
        "data": "synthetic (seeded N(0,1) activations with 1% x30 outlier channels; "
                "W = U diag(i^-1/2) V^T at std 0.02, random-init, no checkpoint)",
        "config": {
            "workload": f"Llama-3-8B attention projection, decode: M={M} tokens, K=N=4096, "
                        f"rank {RANK}, Hadamard block {HAD}; a stack of {L} distinct layers per "
                        f"step, each reading the previous one's output",
            "M": M, "K": K_DIM, "N": N_DIM, "r": RANK, "had_block": HAD,
            "layers_per_step": L,
            "chain": "layer i reads layer i-1's output (a decode step through a stack of "
                     "layers); layer 0 reads the synthetic X",
            "l2": f"inputs larger than L2: {L} layers x {gb / 1e6:.1f} MB of GEMM operands",
            "parallelism": f"{world} independent replica(s), no data-path collective",
            "graph": "one CUDA graph per step; one tq_w4a4_lr_layer launch per layer "
                     "(fused decode kernel), launched with programmatic dependent launch",
        },
        "TOPS": round(world * L * 2 * M * N_DIM * K_DIM / ms / 1e9, 3),
        "us_per_layer": round(ms * 1e3 / L, 3),
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "kernel": "w4a4_lr_decode_kernel (whole layer, split-K cluster of K/256 CTAs)",
            "kernel_us": round(kernel_ms * 1e3, 3),
            "kernel_us_isolated": round(gemm_ms_avg * 1e3, 3),
            "algorithmic_bytes_per_launch": gb, "peak_source": peak_src,
        },
        "e2e": {"value": round(e2e, 1), "unit": "GB/s",
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in hx),
                "d2h_bytes_per_step": sum(y.numel() * y.element_size() for y in hy),
                "ms_per_step": round(ms_e2e, 5)},
        "gpu_launches": L * args.steps,
        "clocks": clocks,
        "two_call_path": {"GB/s": round(world * bytes_step / ms_two / 1e6, 1),
                          "us_per_layer": round(ms_two * 1e3 / L, 3),
                          "calls": "tq_quantize_act + tq_w4a4_lr_gemm"},
    }
    if sweep:
        out["sweep"] = sweep

    # the flip fraction of the decode layers: codes of the bench's first
    # layer from the timed path, against the oracle (in the baseline leg)
    dec_codes = decode_codes_sample(tq, torch, layers[0])
    dec_cpu = {k: v.cpu() for k, v in decode_cpu_inputs(layers[0]).items()}
    del layers, g, g_ev, g_e2e

    # the prefill configurations and the rank overhead, measured in the same
    # process (one GPU only: they are reported beside the decode metric)
    prefill, pre_cpu = {}, {}
    if world == 1 and not args.no_prefill:
        import synth
        steps_p, warm_p = max(5, min(args.steps, 20)), max(3, min(args.warmup, 5))
        for name in PREFILL_CONFIGS:
            sh = synth.CONFIGS[name]
            lays, per_layer = prefill_layers(tq, torch, sh, sh.M, dev, rank, keep_cpu=True)
            pt, _ = prefill_point(tq, torch, sh, sh.M, lays, per_layer, steps_p, warm_p, rank,
                                  local_rank)
            prefill[name] = pt
            pre_cpu[name] = (sh, lays[0]["cpu"],
                             prefill_codes_sample(tq, torch, lays[0], sh, range(CPU_SLICE)))
            del lays
            torch.cuda.empty_cache()
        out["prefill"] = prefill
        ro = {}
        for r in (0, 64):
            sh = synth.CONFIGS["sweep"].with_(r=r)
            lays, per_layer = prefill_layers(tq, torch, sh, sh.M, dev, rank)
            ro[r], _ = prefill_point(tq, torch, sh, sh.M, lays, per_layer, steps_p, warm_p, rank,
                                     local_rank)
            del lays
            torch.cuda.empty_cache()
        out["rank_overhead"] = {
            "workload": "roofline sweep point M = K = N = 4096, Hadamard block 128: rank 64 "
                        "against rank 0, layer time (activation kernel + GEMM)",
            "us_rank0": ro[0]["us_per_layer"], "us_rank64": ro[64]["us_per_layer"],
            "ratio": round(ro[64]["us_per_layer"] / ro[0]["us_per_layer"], 4),
            "gemm_us_rank0": ro[0]["gemm_us"], "gemm_us_rank64": ro[64]["gemm_us"],
            "gemm_ratio": round(ro[64]["gemm_us"] / ro[0]["gemm_us"], 4),
            "target_ratio_at_most": 1.10,
            "TOPS_rank0": ro[0]["TOPS"], "TOPS_rank64": ro[64]["TOPS"],
            "clocks": ro[64]["clocks"],
        }
    if rank == 0 and not args.no_cpu_baseline:
        cb, parity = cpu_baseline(M, budget_s=12.0, decode=(dec_cpu, dec_codes),
                                  prefill=pre_cpu)
        out["cpu_baseline"] = cb
        out["parity"] = parity
    return out


def decode_cpu_inputs(lay):
    return {"X": lay["X"], "L1t": lay["L1t"], "L2t": lay["L2t"], "Rt": lay["Rt"]}


def decode_codes_sample(tq, torch, lay):
    """Codes and scales of the decode layer's tokens as the timed kernel
    makes them (its debug hook: the same kernel, also storing its codes), and
    its weight codes (host copies), for the flip fraction."""
    _, q, s_x, _ = tq.tq_debug_w4a4_lr_layer_decode(lay["X"], lay["L1t"], lay["Wq"], lay["s_w"],
                                                     lay["L2t"], HAD)
    torch.cuda.synchronize()
    return {"q": q.cpu().numpy(), "s_x": s_x.cpu().numpy(), "Wq": lay["Wq"].cpu().numpy(),
            "s_w": lay["s_w"].cpu().numpy(), "b": HAD,
            "source": "the timed decode kernel's own codes (tq_debug_w4a4_lr_layer_decode) on "
                      "the bench's first layer; all weight codes"}


# --------------------------------------------------------------- prefill arm

PREFILL_CONFIGS = ("prefill_gateup", "prefill_down", "large_gateup", "large_down")


def prefill_layers(tq, torch, sh, M, dev, rank, layers_cap=16, keep_cpu=False):
    """Distinct layers of one prefill shape, enough that a step's operands
    exceed L2 (about 200 MB), with every buffer the timed calls use."""
    K, N, r, b = sh.K, sh.N, sh.r, sh.had_block
    per_layer = 2 * M * K + K * N // 2 + 2 * M * N
    L = max(1, min(layers_cap, -(-200_000_000 // per_layer)))
    import synth
    layers = []
    for i in range(L):
        seed = replica_seed(rank) + 10 * i
        w = synth.make_weights(sh, seed=seed, device="cuda")
        X = synth.make_activations(sh, seed=seed, M=M)
        Wq, s_w = tq.tq_pack_weight(w["Rt"].to(dev), b)
        lay = {
            "X": X.to(dev), "L1t": w["L1t"].to(dev) if r else None,
            "L2t": w["L2t"].to(dev) if r else None, "Wq": Wq, "s_w": s_w,
            "Xq": torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
            "Xq8": torch.empty(M, K, dtype=torch.int8, device=dev),
            "s_x": torch.empty(M, dtype=torch.float32, device=dev),
            "XL1": torch.empty(M, r, dtype=torch.float32, device=dev) if r else None,
            "XL1b": torch.empty(M, r, dtype=torch.bfloat16, device=dev) if r else None,
            "Y": torch.empty(M, N, dtype=torch.bfloat16, device=dev),
            "ws": torch.zeros(tq.tq_gemm_a8_workspace_bytes(M, N, K, r), dtype=torch.uint8,
                              device=dev),
        }
        if keep_cpu and i == 0:
            lay["cpu"] = {"X": X, "Rt": w["Rt"], "L1t": w["L1t"], "L2t": w["L2t"]}
        del w
        layers.append(lay)
    torch.cuda.synchronize()
    return layers, per_layer


def prefill_point(tq, torch, sh, M, layers, per_layer, steps, warmup, rank, local_rank,
                  dist=None, world=1, packed_too=False):
    """Times one prefill shape: a step is one layer call (activation kernel +
    GEMM, the kernels tq_w4a4_lr_layer runs for the shape) per distinct
    layer, replayed as a CUDA graph.  Reports the layer's TOPS (2 M N K per
    layer over the layer time, the quantity the INT8 target is set on) and
    the GEMM's alone, both as fractions of the dense INT8 peak."""
    K, N, r, b = sh.K, sh.N, sh.r, sh.had_block
    L = len(layers)
    a8 = tq.tq_layer_path(M, N, K, r, b) == "codes_i8"

    def one(lay, ev=None, packed=not a8):
        if ev is not None:
            ev[2].record()
        if packed:
            tq.tq_quantize_act(lay["X"], b, lay["L1t"], Xq=lay["Xq"], s_x=lay["s_x"],
                               XL1=lay["XL1"])
        else:
            tq.tq_quantize_act_i8(lay["X"], b, lay["L1t"], Xq8=lay["Xq8"], s_x=lay["s_x"],
                                  XL1b=lay["XL1b"])
        if ev is not None:
            ev[0].record()
        if packed:
            tq.tq_w4a4_lr_gemm(lay["Xq"], lay["s_x"], lay["Wq"], lay["s_w"], lay["XL1"],
                               lay["L2t"], Y=lay["Y"], workspace=lay["ws"])
        else:
            tq.tq_w4a4_lr_gemm_a8(lay["Xq8"], lay["s_x"], lay["Wq"], lay["s_w"], lay["XL1b"],
                                  lay["L2t"], Y=lay["Y"], workspace=lay["ws"])
        if ev is not None:
            ev[1].record()

    g = capture(torch, lambda: [one(l) for l in layers])
    with ClockSampler(local_rank) as clk:
        ms = time_graph(torch, g, steps, warmup, dist if world > 1 else None)
    ms = max_over_ranks(ms, dist if world > 1 else None, torch.device("cuda", local_rank))
    del g
    evs = [tuple(torch.cuda.Event(enable_timing=True, external=True) for _ in range(3))
           for _ in layers]
    g_ev = capture(torch, lambda: [one(l, e) for l, e in zip(layers, evs)])
    gemm_ms, act_ms = [], []
    for _ in range(3):
        g_ev.replay()
    for _ in range(max(1, min(steps, 20))):
        g_ev.replay()
        torch.cuda.synchronize()
        gemm_ms.extend(e[0].elapsed_time(e[1]) for e in evs)
        act_ms.extend(e[2].elapsed_time(e[0]) for e in evs)
    del g_ev
    gemm_us = sum(gemm_ms) / len(gemm_ms) * 1e3
    act_us = sum(act_ms) / len(act_ms) * 1e3
    layer_us = ms * 1e3 / L
    packed_us = None
    if a8 and packed_too:
        g_p = capture(torch, lambda: [one(l, packed=True) for l in layers])
        packed_us = time_graph(torch, g_p, steps, warmup) * 1e3 / L
        del g_p
    ops = 2 * M * N * K
    peak, src = int8_peak(sustained=False)
    peak_s, _ = int8_peak(sustained=True)
    tops_layer = ops / (layer_us * 1e-6) / 1e12
    tops_gemm = ops / (gemm_us * 1e-6) / 1e12
    c = clk.summary()
    out = {
        "workload": f"{sh.name}: M={M}, K={K}, N={N}, rank {r}, Hadamard block {b}",
        "M": M, "K": K, "N": N, "r": r, "had_block": b, "layers_per_step": L,
        "l2": "inputs larger than L2" if L * per_layer > 126e6 else "L2-resident",
        "steps": steps, "warmup": warmup,
        "us_per_layer": round(layer_us, 2), "act_us": round(act_us, 2),
        "gemm_us": round(gemm_us, 2),
        "TOPS": round(tops_layer, 1), "TOPS_gemm": round(tops_gemm, 1),
        "roofline": {"bound": "tensor", "unit": "TOPS", "peak": round(peak, 1),
                     "peak_source": src, "achieved": round(tops_layer, 1),
                     "frac": round(tops_layer / peak, 4),
                     "frac_gemm": round(tops_gemm / peak, 4),
                     "frac_sustained_peak": round(tops_layer / peak_s, 4),
                     "kernel": "w4a4_lr_gemm_a8_kernel" if a8 else
                               "w4a4_lr_gemm_kernel (prefill tiling)",
                     "lowrank_flops_per_layer": 2 * M * r * (K + N)},
        "path": ("tq_quantize_act_i8 + tq_w4a4_lr_gemm_a8 (codes one per byte)" if a8
                 else "tq_quantize_act + tq_w4a4_lr_gemm"),
        "clocks": c,
    }
    if c.get("sm_mhz"):
        out["kcycles_per_layer"] = round(layer_us * c["sm_mhz"] / 1e3, 1)
    if packed_us is not None:
        out["packed_code_path_us_per_layer"] = round(packed_us, 3)
    return out, ops * L / (ms * 1e-3)


def prefill_codes_sample(tq, torch, lay, sh, rows):
    """The timed path's codes and scales of sampled tokens (host copies), for
    the flip fraction against the oracle."""
    b = sh.had_block
    idx = torch.as_tensor(rows, device=lay["Xq8"].device)
    return {"qx": lay["Xq8"][idx].cpu().numpy(), "s_x": lay["s_x"][idx].cpu().numpy(),
            "Wq": lay["Wq"].cpu().numpy(), "s_w": lay["s_w"].cpu().numpy(), "b": b}


def run_prefill(args, rank, world, local_rank, dist):
    """One prefill shape per run (--workload): one layer call per distinct
    layer per step; TOPS = 2 M N K per layer / layer time."""
    import torch

    import rank_int4_gemm_b200 as tq
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    sh = synth.CONFIGS[args.workload]
    if args.rank is not None:
        sh = sh.with_(r=args.rank)
    M = args.m if args.m != 16 else sh.M
    layers, per_layer = prefill_layers(tq, torch, sh, M, dev, rank, layers_cap=args.layers)
    if args.profile:
        a8 = tq.tq_layer_path(M, sh.N, sh.K, sh.r, sh.had_block) == "codes_i8"

        def step():
            for l in layers:
                if a8:
                    tq.tq_quantize_act_i8(l["X"], sh.had_block, l["L1t"], Xq8=l["Xq8"],
                                          s_x=l["s_x"], XL1b=l["XL1b"])
                    tq.tq_w4a4_lr_gemm_a8(l["Xq8"], l["s_x"], l["Wq"], l["s_w"], l["XL1b"],
                                          l["L2t"], Y=l["Y"], workspace=l["ws"])
                else:
                    tq.tq_quantize_act(l["X"], sh.had_block, l["L1t"], Xq=l["Xq"],
                                       s_x=l["s_x"], XL1=l["XL1"])
                    tq.tq_w4a4_lr_gemm(l["Xq"], l["s_x"], l["Wq"], l["s_w"], l["XL1"],
                                       l["L2t"], Y=l["Y"], workspace=l["ws"])
        g = capture(torch, step)
        time_graph(torch, g, args.steps, args.warmup)
        return {"profile": f"{args.workload} step graph", "layers": len(layers),
                "steps": args.steps, "warmup": args.warmup}
    pt, ops_per_s = prefill_point(tq, torch, sh, M, layers, per_layer, args.steps, args.warmup,
                                  rank, local_rank, dist, world, packed_too=True)
    L = len(layers)
    out = {
        "metric": METRIC, "value": round(world * ops_per_s / 1e12, 2), "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(L * pt["us_per_layer"] / 1e3, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int4", "data": "synthetic",
        "config": {"workload": pt["workload"] + f"; {L} distinct layer(s) per step",
                   "M": M, "K": sh.K, "N": sh.N, "r": sh.r, "had_block": sh.had_block,
                   "layers_per_step": L, "l2": pt["l2"]},
        "GB/s": round(world * L * per_layer / (L * pt["us_per_layer"] * 1e-6) / 1e9, 1),
        "gpu_launches": 2 * L * args.steps,
    }
    out.update({k: v for k, v in pt.items() if k not in ("workload", "l2")})
    return out


SWEEP_M = (1, 4, 16, 64, 256, 1024, 4096, 8192)
SWEEP_R = (0, 32, 64, 128, 256, 512)


def run_sweeps(args, rank, world, local_rank, dist):
    """The roofline sweeps at K = N = 4096, Hadamard block 128, through the
    public layer entry tq_w4a4_lr_layer (whichever kernels it routes to): M
    over SWEEP_M at rank 64 and rank over SWEEP_R at M = 4096.  Each point
    replays one CUDA graph over enough distinct layers that the step's
    operands exceed L2 (weights shared between points of the same rank, X
    and Y per point).  Reports GB/s of algorithmic bytes and TOPS (2 M N K)
    with their fractions of the measured HBM and INT8 peaks, the
    memory-to-compute crossover (the smallest M whose INT8 fraction is above
    its HBM fraction) and each rank's latency against rank 0."""
    import torch

    import rank_int4_gemm_b200 as tq
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    base = synth.CONFIGS["sweep"]
    K, N, b = base.K, base.N, base.had_block
    hbm, hbm_src = measured_peaks()
    i8, i8_src = int8_peak(sustained=False)
    pools = {}

    def weights(r, n):
        pool = pools.setdefault(r, [])
        sh = base.with_(r=r)
        while len(pool) < n:
            w = synth.make_weights(sh, seed=replica_seed(rank) + 10 * len(pool), device="cuda")
            Rt = w["Rt"].to(dev)
            Wq, s_w = tq.tq_pack_weight(Rt, b)
            del Rt
            pool.append({"Wq": Wq, "s_w": s_w, "L1t": w["L1t"].to(dev) if r else None,
                         "L2t": w["L2t"].to(dev) if r else None})
        return pool[:n]

    def point(M, r):
        per_layer = layer_bytes(M, K, N, r)
        L = max(2, min(16, -(-250_000_000 // per_layer)))
        sh = base.with_(r=r)
        lays = []
        for i, w in enumerate(weights(r, L)):
            lays.append(dict(w, X=synth.make_activations(sh, seed=replica_seed(rank) + 10 * i, M=M).to(dev),
                             Y=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                             ws=torch.zeros(tq.tq_layer_workspace_bytes(M, N, K, r),
                                            dtype=torch.uint8, device=dev)))
        torch.cuda.synchronize()

        def step():
            for l in lays:
                tq.tq_w4a4_lr_layer(l["X"], l["L1t"], l["Wq"], l["s_w"], l["L2t"], b, Y=l["Y"],
                                    workspace=l["ws"])
        g = capture(torch, step)
        ms = time_graph(torch, g, max(5, min(args.steps, 50)), max(3, args.warmup))
        del g, lays
        us = ms * 1e3 / L
        gbs = per_layer / (us * 1e-6) / 1e9
        tops = 2 * M * N * K / (us * 1e-6) / 1e12
        return {"M": M, "r": r, "path": tq.tq_layer_path(M, N, K, r, b), "layers": L,
                "us_per_layer": round(us, 3), "GB/s": round(gbs, 1), "TOPS": round(tops, 2),
                "frac_hbm": round(gbs / hbm, 4), "frac_int8": round(tops / i8, 4)}

    with ClockSampler(local_rank) as clk:
        pts_m = [point(M, 64) for M in SWEEP_M]
        pts_r = [p for p in pts_m if p["M"] == 4096] + [point(4096, r) for r in SWEEP_R if r != 64]
    pts_r.sort(key=lambda p: p["r"])
    r0 = next(p for p in pts_r if p["r"] == 0)["us_per_layer"]
    for p in pts_r:
        p["vs_rank0"] = round(p["us_per_layer"] / r0, 4)
    cross = next((p["M"] for p in pts_m if p["frac_int8"] > p["frac_hbm"]), None)
    ref = next(p for p in pts_m if p["M"] == 4096)
    return {
        "metric": METRIC, "value": ref["TOPS"], "unit": "TOPS", "n_gpus": world,
        "steps": max(5, min(args.steps, 50)), "warmup": max(3, args.warmup),
        "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4", "data": "synthetic",
        "config": {"workload": f"roofline sweeps: K = N = {K}, Hadamard block {b}; M over "
                               f"{list(SWEEP_M)} at rank 64, rank over {list(SWEEP_R)} at M = 4096",
                   "l2": "each point: distinct layers whose operands exceed L2"},
        "sweep_m": pts_m, "sweep_r": pts_r, "crossover_M": cross,
        "rank64_vs_rank0": next(p for p in pts_r if p["r"] == 64)["vs_rank0"],
        "peaks": {"hbm_gbs": hbm, "hbm_source": hbm_src, "int8_tops": i8, "int8_source": i8_src},
        "clocks": clk.summary(),
    }


def run_gateup(args, rank, world, local_rank, dist):
    """Gate and up projections of the prefill MLP shape (M = 2048, K = 4096,
    N = 14336 each, rank 64 each) as one shared-input pair: one activation
    pass and one GEMM over the 2N interleaved channels with the SwiGLU
    epilogue.  TOPS counts both projections (2 x 2 M N K); the comparison is
    the two projections as separate layer calls (without the SwiGLU)."""
    import torch

    import rank_int4_gemm_b200 as tq
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    sh = synth.CONFIGS["prefill_gateup"]
    M = args.m if args.m != 16 else sh.M
    K, N, r, b = sh.K, sh.N, sh.r, sh.had_block
    per_pair = 2 * M * K + K * N + 2 * M * N
    L = max(2, min(args.layers, -(-200_000_000 // per_pair)))
    pairs = []
    for i in range(L):
        seed = replica_seed(rank) + 10 * i
        ws = [synth.make_weights(sh, seed=seed + k, device="cuda") for k in (0, 5)]
        packed = []
        for w in ws:
            Wq, s_w = tq.tq_pack_weight(w["Rt"].to(dev), b)
            packed.append((Wq, s_w, w["L1t"].to(dev), w["L2t"].to(dev)))
        (Wg, sg, L1g, L2g), (Wu, su, L1u, L2u) = packed
        Wq2, s_w2, L1t2, L2t2 = tq.tq_pack_gate_up(Wg, sg, L1g, L2g, Wu, su, L1u, L2u)
        pairs.append({"X": synth.make_activations(sh, seed=seed, M=M).to(dev), "g": packed[0],
                      "u": packed[1], "Wq2": Wq2, "s_w2": s_w2, "L1t2": L1t2, "L2t2": L2t2,
                      "Y": torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                      "Yg": torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                      "Yu": torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                      "ws": tq.Workspace(dev), "wsg": tq.Workspace(dev), "wsu": tq.Workspace(dev)})
        del ws
    torch.cuda.synchronize()

    def fused():
        for p in pairs:
            tq.tq_w4a4_lr_gate_up(p["X"], p["L1t2"], p["Wq2"], p["s_w2"], p["L2t2"], b, Y=p["Y"],
                                  workspace=p["ws"])

    def separate():
        for p in pairs:
            for (Wq, s_w, L1t, L2t), Y, w in ((p["g"], p["Yg"], p["wsg"]), (p["u"], p["Yu"], p["wsu"])):
                tq.tq_w4a4_lr_layer(p["X"], L1t, Wq, s_w, L2t, b, Y=Y, workspace=w)

    g1 = capture(torch, fused)
    g2 = capture(torch, separate)
    steps, warm = max(5, min(args.steps, 50)), max(3, args.warmup)
    with ClockSampler(local_rank) as clk:
        ms = time_graph(torch, g1, steps, warm, dist if world > 1 else None)
    ms = max_over_ranks(ms, dist if world > 1 else None, dev)
    ms2 = time_graph(torch, g2, steps, warm)
    ops = 2 * (2 * M * N * K)
    peak, src = int8_peak(sustained=False)
    return {
        "metric": METRIC, "value": round(whole_job(L * ops, world, ms) / 1e12, 2), "unit": "TOPS",
        "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4",
        "data": "synthetic",
        "config": {"workload": f"gate/up pair with SwiGLU: M={M}, K={K}, N={N} per projection, "
                               f"rank {r} each, Hadamard block {b}; {L} distinct pairs per step",
                   "M": M, "K": K, "N": N, "r": r, "had_block": b, "pairs_per_step": L,
                   "l2": "inputs larger than L2" if L * per_pair > 126e6 else "L2-resident"},
        "us_per_pair": round(ms * 1e3 / L, 3),
        "frac_int8": round(ops / (ms * 1e3 / L * 1e-6) / 1e12 / peak, 4), "peak_source": src,
        "separate_layers_us": round(ms2 * 1e3 / L, 3),
        "speedup_vs_separate": round(ms2 / ms, 3),
        "gpu_launches": 2 * L * steps,
        "clocks": clk.summary(),
    }


def run_qlr(args, rank, world, local_rank, dist):
    """The prefill gate/up layer (M = 2048, K = 4096, N = 14336, rank 64) with
    the INT4 low-rank branch (activation codes, X L1 in INT32, requantized,
    second integer product) against the same layer with the bf16 branch;
    TOPS = 2 M N K per layer."""
    import torch

    import rank_int4_gemm_b200 as tq
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    sh = synth.CONFIGS["prefill_gateup"]
    M = args.m if args.m != 16 else sh.M
    K, N, r, b = sh.K, sh.N, sh.r, sh.had_block
    per_layer = 2 * M * K + K * N // 2 + 2 * M * N
    L = max(2, min(args.layers, -(-200_000_000 // per_layer)))
    lays = []
    for i in range(L):
        seed = replica_seed(rank) + 10 * i
        w = synth.make_weights(sh, seed=seed, device="cuda")
        Wq, s_w = tq.tq_pack_weight(w["Rt"].to(dev), b)
        L1t, L2t = w["L1t"].to(dev), w["L2t"].to(dev)
        lays.append({"X": synth.make_activations(sh, seed=seed, M=M).to(dev), "Wq": Wq, "s_w": s_w,
                     "L1t": L1t, "L2t": L2t, "q": tq.tq_pack_lowrank_q4(L1t, L2t, b),
                     "Y": torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                     "wa": tq.Workspace(dev), "wg": tq.Workspace(dev)})
        del w
    torch.cuda.synchronize()

    def int4_branch():
        for l in lays:
            qL1, s_L1, qL2, s_L2 = l["q"]
            Xq8, s_x, XL1q, s_xl1 = tq.tq_quantize_act_qlr_i8(l["X"], b, qL1, s_L1, workspace=l["wa"])
            tq.tq_w4a4_lr_gemm_a8_qlr(Xq8, s_x, l["Wq"], l["s_w"], XL1q, s_xl1, qL2, s_L2, Y=l["Y"],
                                      workspace=l["wg"])

    def bf16_branch():
        for l in lays:
            Xq8, s_x, XL1b = tq.tq_quantize_act_i8(l["X"], b, l["L1t"])
            tq.tq_w4a4_lr_gemm_a8(Xq8, s_x, l["Wq"], l["s_w"], XL1b, l["L2t"], Y=l["Y"],
                                  workspace=l["wg"])

    g1, g2 = capture(torch, int4_branch), capture(torch, bf16_branch)
    steps, warm = max(5, min(args.steps, 50)), max(3, args.warmup)
    with ClockSampler(local_rank) as clk:
        ms = time_graph(torch, g1, steps, warm, dist if world > 1 else None)
    ms = max_over_ranks(ms, dist if world > 1 else None, dev)
    ms2 = time_graph(torch, g2, steps, warm)
    ops = 2 * M * N * K
    return {
        "metric": METRIC, "value": round(whole_job(L * ops, world, ms) / 1e12, 2), "unit": "TOPS",
        "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4",
        "data": "synthetic",
        "config": {"workload": f"INT4 low-rank branch: M={M}, K={K}, N={N}, rank {r}, Hadamard "
                               f"block {b}; {L} distinct layers per step",
                   "M": M, "K": K, "N": N, "r": r, "had_block": b, "layers_per_step": L,
                   "l2": "inputs larger than L2" if L * per_layer > 126e6 else "L2-resident"},
        "us_per_layer": round(ms * 1e3 / L, 3),
        "bf16_branch_us_per_layer": round(ms2 * 1e3 / L, 3),
        "gpu_launches": 5 * L * steps,
        "clocks": clk.summary(),
    }


def _time_pair(torch, f1, f2, steps, warm, local_rank):
    g1, g2 = capture(torch, f1), capture(torch, f2)
    with ClockSampler(local_rank) as clk:
        ms1 = time_graph(torch, g1, steps, warm)
    ms2 = time_graph(torch, g2, steps, warm)
    del g1, g2
    return ms1, ms2, clk.summary()


def run_qkv(args, rank, world, local_rank, dist):
    """Llama-3-8B attention's Q, K and V projections (K = 4096; N = 4096,
    1024, 1024 under grouped-query attention; rank 32 each) packed as one
    shared-input layer (tq_pack_shared_input, one activation pass and one
    GEMM) against the three projections as separate tq_w4a4_lr_layer calls,
    at decode (M = 16, a stack of layers) and prefill (M = 2048)."""
    import torch

    import rank_int4_gemm_b200 as tq
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    K, Ns, r, b = 4096, (4096, 1024, 1024), 32, 128
    steps, warm = max(5, min(args.steps, 50)), max(3, args.warmup)
    out = {"metric": METRIC, "unit": "TOPS", "n_gpus": world, "steps": steps, "warmup": warm,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4",
           "data": "synthetic", "config": {"workload": "Llama-3-8B attention QKV: K=4096, N = "
                                                       "4096 + 1024 + 1024, rank 32 each, block 128"}}
    for M, L in ((16, 16), (2048, 3)):
        lays = []
        for i in range(L):
            projs = []
            for j, N in enumerate(Ns):
                sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r)
                w = synth.make_weights(sh, seed=replica_seed(rank) + 10 * i + j, device="cuda")
                Wq, s_w = tq.tq_pack_weight(w["Rt"].to(dev), b)
                projs.append((Wq, s_w, w["L1t"].to(dev), w["L2t"].to(dev)))
            Wc, sc, L1c, L2c, _ = tq.tq_pack_shared_input(projs)
            X = synth.make_activations(synth.CONFIGS["decode"].with_(M=M), seed=i, M=M).to(dev)
            lays.append({"X": X, "p": projs, "c": (Wc, sc, L1c, L2c),
                         "Y": torch.empty(M, sum(Ns), dtype=torch.bfloat16, device=dev),
                         "Ys": [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for N in Ns],
                         "ws": tq.Workspace(dev), "wss": [tq.Workspace(dev) for _ in Ns]})
        torch.cuda.synchronize()

        def packed():
            for l in lays:
                Wc, sc, L1c, L2c = l["c"]
                tq.tq_w4a4_lr_layer(l["X"], L1c, Wc, sc, L2c, b, Y=l["Y"], workspace=l["ws"])

        def separate():
            for l in lays:
                for (Wq, s_w, L1t, L2t), Y, w in zip(l["p"], l["Ys"], l["wss"]):
                    tq.tq_w4a4_lr_layer(l["X"], L1t, Wq, s_w, L2t, b, Y=Y, workspace=w)

        ms1, ms2, clk = _time_pair(torch, packed, separate, steps, warm, local_rank)
        ops = 2 * M * sum(Ns) * K
        out[f"M={M}"] = {"us_packed": round(ms1 * 1e3 / L, 3), "us_separate": round(ms2 * 1e3 / L, 3),
                         "TOPS_packed": round(ops / (ms1 * 1e-3 / L) / 1e12, 2),
                         "path_packed": tq.tq_layer_path(M, sum(Ns), K, 3 * r, b),
                         "path_separate": [tq.tq_layer_path(M, N, K, r, b) for N in Ns],
                         "clocks": clk}
        del lays
        torch.cuda.empty_cache()
    out["value"] = out["M=2048"]["TOPS_packed"]
    out["gpu_launches"] = None
    return out


def run_rht(args, rank, world, local_rank, dist):
    """The layer with the randomized Hadamard (a sign mask before the
    Hadamard blocks) against the plain layer: the decode projection (M = 16,
    a stack of 16 layers, the one-kernel path) and the Llama-3-8B gate/up
    prefill shape (M = 2048: the tensor-core activation kernel, which negates
    the masked columns of each staged X block, then the int8-code GEMM; the
    plain layer runs the same kernels without the mask)."""
    import torch

    import rank_int4_gemm_b200 as tq
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    steps, warm = max(5, min(args.steps, 50)), max(3, args.warmup)
    out = {"metric": METRIC, "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": warm,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4",
           "data": "synthetic", "config": {"workload": "randomized Hadamard against the plain "
                                                       "Hadamard, decode and prefill shapes"}}
    for name, L in (("decode", 16), ("prefill_gateup", 2)):
        sh = synth.CONFIGS[name]
        M, K, N, r, b = sh.M, sh.K, sh.N, sh.r, sh.had_block
        gen = torch.Generator().manual_seed(77)
        signs = torch.randint(-2 ** 31, 2 ** 31 - 1, (K // 32,), generator=gen,
                              dtype=torch.int64).to(torch.int32).to(dev)
        lays = []
        for i in range(L):
            w = synth.make_weights(sh, seed=replica_seed(rank) + 10 * i, device="cuda")
            Rt = w["Rt"].to(dev)
            lays.append({"X": synth.make_activations(sh, seed=i).to(dev), "L1t": w["L1t"].to(dev),
                         "L2t": w["L2t"].to(dev), "plain": tq.tq_pack_weight(Rt, b),
                         "rht": tq.tq_pack_weight_rht(Rt, b, signs),
                         "Y": torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                         "ws": tq.Workspace(dev)})
            del Rt
        torch.cuda.synchronize()

        def plain():
            for l in lays:
                tq.tq_w4a4_lr_layer(l["X"], l["L1t"], *l["plain"], l["L2t"], b, Y=l["Y"],
                                    workspace=l["ws"])

        def signed():
            for l in lays:
                tq.tq_w4a4_lr_layer_rht(l["X"], signs, l["L1t"], *l["rht"], l["L2t"], b, Y=l["Y"],
                                        workspace=l["ws"])

        ms_s, ms_p, clk = _time_pair(torch, signed, plain, steps, warm, local_rank)
        byt = layer_bytes(M, K, N, r)
        out[name] = {"M": M, "K": K, "N": N, "r": r, "us_signed": round(ms_s * 1e3 / L, 3),
                     "us_plain": round(ms_p * 1e3 / L, 3),
                     "GB/s_signed": round(byt / (ms_s * 1e-3 / L) / 1e9, 1),
                     "TOPS_signed": round(2 * M * N * K / (ms_s * 1e-3 / L) / 1e12, 2),
                     "clocks": clk}
        del lays
        torch.cuda.empty_cache()
    out["value"] = out["decode"]["GB/s_signed"]
    out["gpu_launches"] = None
    return out


# ------------------------------------------------------------ oracle (CPU)

CPU_SLICE = 64  # tokens of a prefill layer the oracle evaluates (time extrapolated)


def _flips(gpu_q, orc_q, orc_t, rel=1e-6):
    """Fraction of codes that differ from the oracle's, and how many of those
    differ outside the midpoint allowance (a difference of exactly one where
    the oracle's v/s lies within rel*|v/s| of the midpoint)."""
    import numpy as np
    g = np.asarray(gpu_q).astype(np.int32)
    o = np.asarray(orc_q).astype(np.int32)
    d = g - o
    bad = d != 0
    n = int(bad.sum())
    if n == 0:
        return 0.0, 0, int(g.size)
    mid = (g[bad] + o[bad]) / 2.0
    t = np.asarray(orc_t)[bad]
    ok = (np.abs(d[bad]) == 1) & (np.abs(t - mid) <= rel * np.abs(t))
    return n / g.size, int((~ok).sum()), int(g.size)


def _one_layer(oracle, X, L1t, L2t, w, b):
    """One evaluation of the layer by the oracle (weights packed beforehand);
    returns the per-stage times and the activation codes."""
    t0 = time.perf_counter()
    a = oracle.quantize_act(X, b)
    t1 = time.perf_counter()
    acc = oracle.int_gemm(a["qx"], w["qw"])
    t2 = time.perf_counter()
    lr = None
    if L1t is not None and L1t.shape[0] > 0:
        _, lr = oracle.lowrank(X, L1t, L2t)
    t3 = time.perf_counter()
    oracle.epilogue(a["s_x"], w["s_w"], acc, lr)
    t4 = time.perf_counter()
    return {"rotate_quantize": t1 - t0, "int_gemm": t2 - t1, "lowrank": t3 - t2,
            "epilogue": t4 - t3}, a


def cpu_baseline(M, budget_s=12.0, decode=None, prefill=None):
    """The fp64 C oracle, as it stands, on bounded samples of the workloads.

    * decode: repeated evaluations of one decode layer (the bench's first
      layer) on all host threads for about budget_s, with the time of each
      stage (rotation + codes, integer GEMM, low-rank branch, epilogue);
    * one thread: one evaluation of the tiny layer and of the decode layer;
    * prefill: the first 64 tokens of each prefill layer (weights packed
      beforehand, untimed); the layer time is extrapolated linearly in M.
    Also returns the flip fractions of the timed path's codes against the
    oracle's on those samples (the reported fraction of midpoint flips)."""
    import numpy as np

    import oracle
    import synth

    threads = oracle.num_threads()
    if decode is not None:
        dec_in, dec_codes = decode
        X, L1t, L2t, Rt = dec_in["X"], dec_in["L1t"], dec_in["L2t"], dec_in["Rt"]
    else:
        dec_codes = None
        L = synth.make_layer(synth.CONFIGS["decode"].with_(M=M), seed=0)
        X, L1t, L2t, Rt = L["X"], L["L1t"], L["L2t"], L["Rt"]
    w = oracle.pack_weight(Rt, HAD)          # offline, untimed
    n, t0, stages, a = 0, time.perf_counter(), None, None
    while True:
        st, a = _one_layer(oracle, X, L1t, L2t, w, HAD)
        stages = st if stages is None else {k: stages[k] + st[k] for k in st}
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = (time.perf_counter() - t0) / n
    val = layer_bytes(M, K_DIM, N_DIM, RANK) / dt / 1e9
    cb = {"value": round(val, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
          "sample": f"{n} evaluations of one decode layer (M={M}, K=N=4096, r=32), "
                    f"{dt:.3f} s each on {threads} threads; weights packed outside the timing",
          "s_per_layer": round(dt, 4),
          "stages_s_per_layer": {k: round(v / n, 5) for k, v in stages.items()}}
    parity = {"rule": "a code may differ by one only where the oracle's v/s lies within "
                      "1e-6 relative of the rounding midpoint; outside = codes breaking it"}
    if dec_codes is not None:
        f, bad, cnt = _flips(dec_codes["q"], a["qx"], a["t_x"])
        fw, badw, cntw = _flips(oracle.unpack_int4(dec_codes["Wq"]), w["qw"], w["t_w"])
        parity["decode"] = {"activation_flip_fraction": f, "activation_codes": cnt,
                            "outside_allowance": bad, "weight_flip_fraction": fw,
                            "weight_codes": cntw, "weight_outside_allowance": badw,
                            "source": dec_codes["source"]}

    # one thread: the tiny layer and the decode layer
    one = {}
    oracle.set_num_threads(1)
    try:
        tl = synth.make_layer(synth.CONFIGS["tiny"], seed=0)
        tw = oracle.pack_weight(tl["Rt"], 256)
        reps, t0 = 0, time.perf_counter()
        while reps < 3 or time.perf_counter() - t0 < 0.5:
            _one_layer(oracle, tl["X"], tl["L1t"], tl["L2t"], tw, 256)
            reps += 1
        dtt = (time.perf_counter() - t0) / reps
        one["tiny"] = {"s_per_layer": round(dtt, 6),
                       "GB/s": round(layer_bytes(16, 256, 256, 16) / dtt / 1e9, 5)}
        t0 = time.perf_counter()
        st1, _ = _one_layer(oracle, X, L1t, L2t, w, HAD)
        dt1 = time.perf_counter() - t0
        one["decode"] = {"s_per_layer": round(dt1, 4),
                         "GB/s": round(layer_bytes(M, K_DIM, N_DIM, RANK) / dt1 / 1e9, 5),
                         "stages_s": {k: round(v, 5) for k, v in st1.items()}}
    finally:
        oracle.set_num_threads(threads)
    cb["one_thread"] = one
    del w

    # prefill: the first CPU_SLICE tokens of each configuration, extrapolated
    ext = {}
    for name, (sh, cpu, codes) in (prefill or {}).items():
        b = sh.had_block
        w = oracle.pack_weight(cpu["Rt"], b)
        Xs = cpu["X"][:CPU_SLICE]
        t0 = time.perf_counter()
        st, a = _one_layer(oracle, Xs, cpu["L1t"], cpu["L2t"], w, b)
        ds = time.perf_counter() - t0
        full = ds * sh.M / CPU_SLICE
        ext[name] = {"tokens": CPU_SLICE, "s_slice": round(ds, 3),
                     "s_layer_extrapolated": round(full, 2),
                     "TOPS_extrapolated": round(2 * sh.M * sh.N * sh.K / full / 1e12, 6),
                     "stages_s_slice": {k: round(v, 4) for k, v in st.items()},
                     "label": "extrapolated"}
        f, bad, cnt = _flips(codes["qx"], a["qx"], a["t_x"])
        fw, badw, cntw = _flips(oracle.unpack_int4(codes["Wq"]), w["qw"], w["t_w"])
        parity[name] = {"activation_flip_fraction": f, "activation_codes": cnt,
                        "outside_allowance": bad, "weight_flip_fraction": fw,
                        "weight_codes": cntw, "weight_outside_allowance": badw,
                        "source": f"tq_quantize_act_i8 codes of the first {CPU_SLICE} tokens "
                                  f"of the timed layer; all weight codes"}
        del w, a
    if ext:
        cb["prefill_slices"] = ext
    return cb, parity


def run_reference(args):
    """The oracle as the reference arm: each step a bounded sample (one layer
    of the same workload), timed on the host cores."""
    import oracle
    import synth

    M = args.m
    sh = synth.CONFIGS["decode"].with_(M=M)
    L = synth.make_layer(sh, seed=0)
    w = oracle.pack_weight(L["Rt"], HAD)
    X, L1t, L2t = L["X"], L["L1t"], L["L2t"]

    def one():
        a = oracle.quantize_act(X, HAD)
        acc = oracle.int_gemm(a["qx"], w["qw"])
        _, lr = oracle.lowrank(X, L1t, L2t)
        oracle.epilogue(a["s_x"], w["s_w"], acc, lr)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    val = layer_bytes(M, K_DIM, N_DIM, RANK) / dt / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"Llama-3-8B attention projection, decode: M={M} tokens, "
                               f"K=N=4096, rank {RANK}, Hadamard block {HAD}; each step one layer",
                   "M": M, "K": K_DIM, "N": N_DIM, "r": RANK, "had_block": HAD},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": "one decode layer per step (rotation, codes, X L1, integer "
                                   "GEMM, low-rank branch, epilogue); weights packed untimed"},
        "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)))
        return 0
    dist = None
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if args.workload == "decode":
        out = run_tq(args, rank, world, local_rank, dist)
    elif args.workload == "sweeps":
        out = run_sweeps(args, rank, world, local_rank, dist)
    elif args.workload == "gateup_swiglu":
        out = run_gateup(args, rank, world, local_rank, dist)
    elif args.workload == "qlr":
        out = run_qlr(args, rank, world, local_rank, dist)
    elif args.workload == "qkv":
        out = run_qkv(args, rank, world, local_rank, dist)
    elif args.workload == "rht":
        out = run_rht(args, rank, world, local_rank, dist)
    else:
        out = run_prefill(args, rank, world, local_rank, dist)
    if rank == 0:
        print(json.dumps(out))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
