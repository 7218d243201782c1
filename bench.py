"""Benchmark of the NVFP4 W4A4 MoE expert layer (one JSON line on rank 0).

Headline workload: the Qwen3-30B-A3B-shaped expert layer -- 16384 tokens,
hidden 2048, 128 experts, top-8 softmax routing, gate_up 2048 -> 2x768 with
SwiGLU and NVFP4 requantization, down 768 -> 2048 -- on seeded synthetic BF16
data.  A step is one moe_expert_layer call (every kernel of the path).
Per-token scaling (the token-wise path) is the default; --per-tensor switches.
At one GPU the same line also carries the other synthetic workloads (toy,
dense Qwen3-4B-shaped, the Zipf-skewed 65536-token MoE layer) under
"workloads", each with its own throughput, roofline, e2e and CPU baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU under torchrun; each rank runs the layer on its
own tokens with its own replica of the weights (data parallel, no data-path
collective: "scaling": "weak").  Time is the max over ranks of the device
time.  --impl reference times the CPU oracle (the reference arm of this
build) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_moe_grouped_token_b200 import workloads  # noqa: E402

METRIC = "NVFP4 MoE expert-layer tokens/s & TFLOPS (% of FP4 peak); quantizer GB/s"
FP4_PER_BF16 = 4.0        # nominal dense FP4 : BF16 tensor throughput (9 : 2.25 PFLOP/s)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="moe30b")
    ap.add_argument("--per-tensor", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-experts", type=int, default=8,
                    help="experts whose routed rows form the cpu_baseline sample (~10 s of oracle work)")
    ap.add_argument("--ref-experts", type=int, default=2,
                    help="experts whose routed rows form each step of --impl reference (~2 s per step)")
    ap.add_argument("--workloads", default="toy,dense4b,moe30b_skew",
                    help="extra workloads measured at one GPU and reported under 'workloads' ('' = none)")
    ap.add_argument("--workload-steps", type=int, default=20)
    ap.add_argument("--no-backward", action="store_true", help="skip timing the BF16 backward")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip timing the W4A16 and W4A8 activation-precision variants")
    ap.add_argument("--no-fast-combine", action="store_true",
                    help="skip measuring the non-strict (FP32-reduction) combine beside the headline")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons of one GPU, sampled while
    the timed loop runs: read-only NVML queries every 5 ms, else nvidia-smi
    every 200 ms.  Samples between mark_begin() and mark_end() are the ones
    reported."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, index: int):
        self.index = index
        self.samples = []          # (host time, sm MHz, max sm MHz, set of active reasons)
        self.t0 = self.t1 = None
        self.source = None
        self.proc = None
        self.thread = None
        self.stop_event = threading.Event()

    def _nvml(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            props = torch.cuda.get_device_properties(self.index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def start(self):
        try:
            nv, h = self._nvml()

            def loop():
                while not self.stop_event.is_set():
                    try:
                        t = time.perf_counter()
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
                        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((t, sm, mx, {n for n, b in self.REASONS if bits & b}))
                    except Exception:
                        pass
                    self.stop_event.wait(0.005)
            self.source = "nvml"
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                     "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (FileNotFoundError, OSError):
                self.proc = None
                return

            def loop():
                names = [n for n, _ in self.REASONS]
                for ln in self.proc.stdout:
                    p = [x.strip() for x in ln.split(",")]
                    if len(p) < 9:
                        continue
                    try:
                        self.samples.append((time.perf_counter(), float(p[1]), float(p[2]),
                                             {n for n, v in zip(names, p[5:9]) if v.lower() == "active"}))
                    except ValueError:
                        continue
            self.source = "nvidia-smi"
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def mark_begin(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        self.stop_event.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml and nvidia-smi unavailable"]}
        inside = [x for x in self.samples
                  if self.t0 is not None and self.t1 is not None and self.t0 <= x[0] <= self.t1]
        use = inside if inside else self.samples[-3:]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": self.source}
        return {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": max(x[2] for x in use),
                "reasons": sorted(set().union(*(x[3] for x in use))), "samples": len(use),
                "in_timed_region": bool(inside), "source": self.source}


def layer_flops(cfg) -> dict:
    R = cfg.T * cfg.k
    gu = 2.0 * R * cfg.H * (2 * cfg.I)
    dn = 2.0 * R * cfg.I * cfg.H
    return {"gate_up": gu, "down": dn, "total": gu + dn}


def stage_bytes(cfg, per_tensor: bool = False, fused_requant: bool = False) -> dict:
    """Algorithmic HBM bytes per stage (each tensor read or written once).

    h leaves the gate_up GEMM in BF16 and a second pass requantizes it; with
    the requantization fused into the GEMM (per-token scales only) the GEMM's
    output is h's NVFP4 codes and scales and there is no requant stage."""
    fused = fused_requant and not per_tensor
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    R = T * k
    nv = 0.5 + 1.0 / 16                 # NVFP4 bytes per element (codes + UE4M3 scale)
    w_gu = E * 2 * I * H * nv
    w_dn = E * H * I * nv
    out = {
        "quantize_permute": T * H * 2 + R * H * nv + R * 8,
        "gate_up_swiglu": R * H * nv + w_gu + (R * I * nv if fused else R * I * 2),
        "down": R * I * nv + w_dn + R * H * 2,
        "combine": R * H * 2 + T * H * 2 + R * 8,
    }
    if not fused:
        out["requant_h"] = R * I * 2 + R * I * nv
    return out


# ------------------------------------------------------- multi-rank ----

def rank_config(cfg, rank: int, world: int):
    """Data-parallel replicas: every rank runs the same layer shape on its own
    tokens (seed shifted by rank), with a full copy of the weights."""
    return cfg if world == 1 else workloads.scaled(cfg, seed=cfg.seed + 1000 * rank)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's time (the job's time) via all_reduce(MAX)."""
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms_max * 1e-3)


# --------------------------------------------------------------- ours ----

def fp4_peak(reps: int = 3) -> dict:
    """The block-scaled FP4 MMA's measured throughput on this GPU (the GEMM's
    instruction and tile shape, operands in shared memory), best of `reps`
    launches, with and without the scale writes the GEMM's feeders issue."""
    from nvfp4_moe_grouped_token_b200 import ops
    pure = max(ops.mma_peak(4000, scale_writes=False)["tflops"] for _ in range(reps))
    fed = max(ops.mma_peak(4000, scale_writes=True)["tflops"] for _ in range(reps))
    return {"mma_only": pure, "with_scale_writes": fed}


def kernel_rooflines(cfg, stage_ms: dict, per_tensor: bool, pk: dict, fp4: dict, traffic, fused_requant=False):
    """Every stage of the step against its own bound: HBM stages against the
    measured copy bandwidth, the GEMMs against the measured FP4 MMA peak (and
    the down GEMM, whose BF16 output dominates its bytes, against HBM too)."""
    fl = layer_flops(cfg)
    sb = stage_bytes(cfg, per_tensor, fused_requant)
    out = []
    for name, ms in stage_ms.items():
        if name not in sb and name != "route":
            continue
        sec = ms * 1e-3
        row = {"stage": name, "ms": ms}
        if name == "route":
            row.update(bound="latency", note="histogram + scan of the routing metadata (~1 MB)")
        elif name in ("gate_up_swiglu", "down"):
            f = fl["gate_up" if name == "gate_up_swiglu" else "down"]
            row.update(bound="tensor" if name == "gate_up_swiglu" else "hbm",
                       tflops=f / sec / 1e12, frac_fp4_peak=f / sec / 1e12 / fp4["mma_only"],
                       gbs=sb[name] / sec / 1e9, frac_hbm=sb[name] / sec / 1e9 / pk["hbm_gbs"],
                       algorithmic_bytes=sb[name], flop=f)
            if name == "gate_up_swiglu":
                row["traffic"] = traffic
        else:
            row.update(bound="hbm", gbs=sb[name] / sec / 1e9, frac_hbm=sb[name] / sec / 1e9 / pk["hbm_gbs"],
                       algorithmic_bytes=sb[name])
        out.append(row)
    return out


FAST_COMBINE_FLAG = 0x80     # NVFP4MOE_FAST_COMBINE
FUSED_REQUANT_FLAG = 0x100   # NVFP4MOE_FUSED_REQUANT


def measure_layer(cfg, args, world, dev, steps, warmup, fp4, clocks_for_timed=True, extra_flags=0):
    """Time `steps` layer steps (inputs resident in HBM) and the same number of
    end-to-end steps from pinned host buffers.  Returns the measurement dict."""
    from nvfp4_moe_grouped_token_b200 import ops

    flags = (0 if args.per_tensor else ops.SCALE_PER_TOKEN) | extra_flags
    inp = workloads.layer_inputs(cfg)
    x = inp["x"].to(dev)
    idx = inp["topk_idx"].to(dev)
    w = inp["topk_w"].to(dev)
    wgu = ops.nvfp4_prepare_weights(inp["w_gate_up"].to(dev), gate_up=True)
    wdn = ops.nvfp4_prepare_weights(inp["w_down"].to(dev), gate_up=False)
    del inp["w_gate_up"], inp["w_down"]
    ws = torch.empty(ops.moe_expert_layer_workspace_size(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, flags),
                     dtype=torch.uint8, device=dev)
    y = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    for _ in range(warmup):
        ops.moe_expert_layer(x, idx, w, wgu, wdn, y, ws, flags)
    torch.cuda.synchronize()
    assert ops.device_status(ws) == 0

    # ---- timed region: K steps through the public API, inputs resident in
    # HBM, with CUDA events only around the gate_up GEMM (the roofline's
    # kernel); then K more steps with an event between every two kernels for
    # the stage breakdown (each event record costs a step a few microseconds,
    # so the timed steps carry two)
    nstage = len(ops.STAGES)
    gu_stage = ops.STAGES.index("gate_up_swiglu")
    gu_evs = [[None] * (nstage + 1) for _ in range(steps)]
    for row in gu_evs:
        row[gu_stage] = torch.cuda.Event(enable_timing=True)
        row[gu_stage + 1] = torch.cuda.Event(enable_timing=True)
        row[gu_stage].record(stream)
        row[gu_stage + 1].record(stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage + 1)] for _ in range(steps)]
    for row in evs:                          # materialise the events before timing
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index) if clocks_for_timed else None
    if clocks is not None:
        clocks.start()
        time.sleep(0.2)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.mark_begin()
    t_start.record(stream)
    for i in range(steps):
        ops.moe_expert_layer_profiled(x, idx, w, wgu, wdn, y, ws, gu_evs[i], flags)
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    p_start = torch.cuda.Event(enable_timing=True)
    p_end = torch.cuda.Event(enable_timing=True)
    p_start.record(stream)
    for i in range(steps):
        ops.moe_expert_layer_profiled(x, idx, w, wgu, wdn, y, ws, evs[i], flags)
    p_end.record(stream)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.mark_end()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks is not None else None
    assert ops.device_status(ws) == 0

    total_ms = t_start.elapsed_time(t_end)
    profiled_ms = max_over_ranks(p_start.elapsed_time(p_end) / steps, world, dev)
    step_ms = [evs[i][0].elapsed_time(evs[i][nstage]) for i in range(steps)]
    stage_ms = {name: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps))
                for j, name in enumerate(ops.STAGES)}
    if flags & FUSED_REQUANT_FLAG:
        stage_ms.pop("requant_h")              # fused into gate_up: an empty interval
    # the roofline kernel's time from the timed steps themselves
    gate_up_timed_ms = statistics.mean(gu_evs[i][gu_stage].elapsed_time(gu_evs[i][gu_stage + 1])
                                       for i in range(steps))
    ms = max_over_ranks(total_ms / steps, world, dev)

    # ---- the same K steps replayed from one CUDA graph ----------------------
    # (the layer makes no host synchronization or allocation, so a step
    # captures as is; a small workload is launch-bound without it)
    graph_ms = None
    if world == 1:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(steps):
                ops.moe_expert_layer(x, idx, w, wgu, wdn, y, ws, flags)
        g.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        graph_ms = g0.elapsed_time(g1) / steps
        del g
        assert ops.device_status(ws) == 0

    # ---- end to end through the public API with host buffers ----------------
    # Every step copies its inputs from pinned host memory and reads its whole
    # output back.  The copies run on two copy streams with double-buffered
    # device inputs and outputs, so step i+1's input copies and step i-1's
    # output copy overlap step i's kernels (PCIe is full duplex).
    xh = inp["x"].pin_memory()
    ih = inp["topk_idx"].pin_memory()
    wh = inp["topk_w"].pin_memory()
    yh = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    idd = [torch.empty_like(idx) for _ in range(2)]
    wd = [torch.empty_like(w) for _ in range(2)]
    yd = [torch.empty_like(y) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e_ in ev_in + ev_done + ev_out:
        e_.record(stream)

    def e2e_step(i):
        b = i % 2
        s_in.wait_event(ev_done[b])              # step i-2 no longer reads input buffer b
        with torch.cuda.stream(s_in):
            xd[b].copy_(xh, non_blocking=True)
            idd[b].copy_(ih, non_blocking=True)
            wd[b].copy_(wh, non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])             # step i-2's output has left buffer b
        ops.moe_expert_layer(xd[b], idd[b], wd[b], wgu, wdn, yd[b], ws, flags)
        ev_done[b].record(stream)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            yh[b].copy_(yd[b], non_blocking=True)
        ev_out[b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, steps)
    e0.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    assert torch.equal(yh[(n_e2e - 1) % 2].view(torch.int16), yd[(n_e2e - 1) % 2].cpu().view(torch.int16))
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, dev)

    fl = layer_flops(cfg)
    pk = peaks()
    traffic = load_traffic("gate_up_swiglu") if cfg.name == "moe30b" else None
    kern = kernel_rooflines(cfg, stage_ms, args.per_tensor, pk, fp4, traffic, bool(flags & FUSED_REQUANT_FLAG))
    gu_tflops = fl["gate_up"] / (gate_up_timed_ms * 1e-3) / 1e12
    bf16x4 = pk["bf16_tflops"] * FP4_PER_BF16
    launches_per_step = 7 + (1 if args.per_tensor else 0) - (1 if flags & FUSED_REQUANT_FLAG else 0)
    return {
        "value": job_throughput(cfg.T, world, ms),
        "ms_per_step": ms,
        "tflops": world * fl["total"] / (ms * 1e-3) / 1e12,
        "stages_ms": stage_ms,
        "stage_timing": "K further steps right after the timed ones, with a CUDA event between the kernels on the "
                        "launching stream; their mean step time is profiled_ms_per_step",
        "profiled_ms_per_step": profiled_ms,
        "graph_ms_per_step": graph_ms,
        "step_ms_min_max": [min(step_ms), max(step_ms)],
        "roofline": {"kernel": "k_grouped_gemm (gate_up + SwiGLU epilogue)",
                     "bound": "tensor", "achieved": gu_tflops, "peak": fp4["mma_only"], "unit": "TFLOP/s",
                     "frac": gu_tflops / fp4["mma_only"], "traffic": traffic,
                     "kernel_ms": gate_up_timed_ms,
                     "kernel_timing": "CUDA events around the kernel in every timed step, on its launching stream",
                     "peak_note": "block-scaled FP4 MMA (M128 N256 K64) measured in this process, operands in "
                                  "shared memory (nvfp4moe_mma_peak)",
                     "peak_with_scale_writes": fp4["with_scale_writes"],
                     "frac_vs_bf16_burst_x4": gu_tflops / bf16x4,
                     "bf16_burst_x4": bf16x4, "bf16_source": pk["source"],
                     "frac_vs_nominal_9pf": gu_tflops / 9000.0,
                     "kernels": kern},
        "e2e": {"value": job_throughput(cfg.T, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": xh.numel() * 2 + ih.numel() * 4 + wh.numel() * 4,
                "d2h_bytes_per_step": yh[0].numel() * 2,
                "pipeline": "input copies (copy stream 1), the layer (launching stream) and the output copy (copy "
                            "stream 2) of consecutive steps overlap; double-buffered device inputs and outputs"},
        "gpu_launches": steps * launches_per_step,
        "launches_per_step": launches_per_step,
        "clocks": clk,
    }


def backward_flops(cfg) -> dict:
    """The BF16 backward's products (2 * rows * K * N each): the recomputed
    gate_up, dgrad of down, dgrad of gate_up, and the two weight gradients."""
    R = cfg.T * cfg.k
    H, I = cfg.H, cfg.I
    f = {"gate_up_recompute": 2.0 * R * H * 2 * I, "dgrad_down": 2.0 * R * H * I, "dgrad_gate_up": 2.0 * R * 2 * I * H,
         "wgrad_down": 2.0 * R * H * I, "wgrad_gate_up": 2.0 * R * 2 * I * H}
    f["total"] = sum(f.values())
    return f


def measure_backward(cfg, dev, steps, warmup):
    """Time moe_expert_layer_backward (BF16 backward of the layer, FP32 weight
    gradients) on the workload, inputs resident in HBM."""
    from nvfp4_moe_grouped_token_b200 import ops

    inp = workloads.layer_inputs(cfg)
    x, idx, w = inp["x"].to(dev), inp["topk_idx"].to(dev), inp["topk_w"].to(dev)
    wgu, wdn = inp["w_gate_up"].to(dev), inp["w_down"].to(dev)
    g = torch.Generator().manual_seed(77)
    dy = torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16).to(dev)
    ws = torch.empty(ops.moe_expert_layer_backward_workspace_size(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8,
                     device=dev)
    dx = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    dtw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    dwgu = torch.empty(cfg.E, 2 * cfg.I, cfg.H, dtype=torch.bfloat16, device=dev)
    dwdn = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.bfloat16, device=dev)

    def step():
        ops.moe_expert_layer_backward(x, idx, w, wgu, wdn, dy, dx, dtw, ws, dw_gate_up_bf16=dwgu, dw_down_bf16=dwdn)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert ops.device_status(ws) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    assert ops.device_status(ws) == 0
    ms = e0.elapsed_time(e1) / steps
    fl = backward_flops(cfg)
    pk = peaks()
    tf = fl["total"] / (ms * 1e-3) / 1e12
    return {"ms_per_step": ms, "tokens_per_s": cfg.T / (ms * 1e-3), "tflops": tf, "flop": fl["total"],
            "frac_bf16_burst": tf / pk["bf16_tflops"], "bf16_peak": pk["bf16_tflops"], "bf16_source": pk["source"],
            "weight_grads": "bf16", "steps": steps,
            "note": "BF16-backward mode: exact gradient of the unquantized layer on BF16 operands (gate_up recomputed)"}


def measure_variant(cfg, dev, steps, warmup, kind):
    """Time the W4A16 or W4A8 layer (NVFP4 weights; BF16 or MXFP8
    activations, products on the BF16 tensor cores) on the workload, inputs
    resident in HBM, outside the headline's timed region.  The rate reported
    is the layer's GEMM FLOPs over the whole step time (routing, gather, both
    GEMMs and the combine), against the BF16 peak; the GEMM's own share of
    the step is in the ncu launch list under profiles/."""
    from nvfp4_moe_grouped_token_b200 import ops

    inp = workloads.layer_inputs(cfg)
    x, idx, w = inp["x"].to(dev), inp["topk_idx"].to(dev), inp["topk_w"].to(dev)
    wgu = ops.nvfp4_prepare_weights(inp["w_gate_up"].to(dev), gate_up=True)
    wdn = ops.nvfp4_prepare_weights(inp["w_down"].to(dev), gate_up=False)
    size = ops.moe_expert_layer_w4a8_workspace_size if kind == "w4a8" else ops.moe_expert_layer_w4a16_workspace_size
    call = ops.moe_expert_layer_w4a8 if kind == "w4a8" else ops.moe_expert_layer_w4a16
    ws = torch.empty(size(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8, device=dev)
    y = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)

    def step():
        call(x, idx, w, wgu, wdn, y, ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert ops.device_status(ws) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    assert ops.device_status(ws) == 0
    ms = e0.elapsed_time(e1) / steps
    fl = layer_flops(cfg)["total"]
    pk = peaks()
    tf = fl / (ms * 1e-3) / 1e12
    act = "MXFP8 (E4M3, E8M0 per 32)" if kind == "w4a8" else "BF16"
    return {"ms_per_step": ms, "tokens_per_s": cfg.T / (ms * 1e-3), "tflops": tf, "flop": fl,
            "frac_bf16_burst": tf / pk["bf16_tflops"], "bf16_peak": pk["bf16_tflops"], "bf16_source": pk["source"],
            "steps": steps, "activations": act, "weights": "NVFP4 (the headline's prepared weights)",
            "note": "weights stay 4-bit in HBM and are converted to BF16 per K-step in shared memory; "
                    "kind::f16 tensor cores; the whole step (routing, gather, both GEMMs, combine) is timed"}


def measure_router(cfg, dev, steps, warmup):
    """Time the dense router GEMM (moe_router_logits: logits = x W_r^T, BF16
    operands, FP32 out) on the workload's shapes, W_r ~ N(0, 0.02)."""
    from nvfp4_moe_grouped_token_b200 import ops

    g = torch.Generator().manual_seed(91)
    x = torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16).to(dev)
    w = (torch.randn(cfg.E, cfg.H, generator=g) * 0.02).to(torch.bfloat16).to(dev)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        ops.moe_router_logits(x, w, logits, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        ops.moe_router_logits(x, w, logits, ws)
    e1.record()
    torch.cuda.synchronize()
    assert ops.device_status(ws) == 0
    ms = e0.elapsed_time(e1) / steps
    fl = 2.0 * cfg.T * cfg.H * cfg.E
    byt = cfg.T * cfg.H * 2 + cfg.E * cfg.H * 2 + cfg.T * cfg.E * 4
    pk = peaks()
    return {"us": ms * 1e3, "tflops": fl / (ms * 1e-3) / 1e12, "gbs": byt / (ms * 1e-3) / 1e9,
            "frac_hbm": byt / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], "bound": "hbm",
            "note": "x read once (67 MB for moe30b): HBM-bound at E = 128; tcgen05 kind::f16"}


def measure_ep(cfg, dev, steps, warmup, G):
    """The expert-parallel pipeline (nvfp4_moe_grouped_token_b200.ep) with G
    ranks driven by this process on one GPU: dispatch, exchanges as device
    copies, arrange, experts, return, combine, including the one host read of
    the offsets per rank that sizes the exchange.  Reports the step time and
    the bytes that would cross NVLink per step (NVFP4 rows out, BF16 D back)."""
    from nvfp4_moe_grouped_token_b200 import ep, ops

    inp = workloads.layer_inputs(cfg)
    wgu = ops.nvfp4_prepare_weights(inp["w_gate_up"].to(dev), gate_up=True)
    wdn = ops.nvfp4_prepare_weights(inp["w_down"].to(dev), gate_up=False)
    b = [cfg.T * g // G for g in range(G + 1)]
    xs = [inp["x"][b[g]:b[g + 1]].contiguous().to(dev) for g in range(G)]
    idxs = [inp["topk_idx"][b[g]:b[g + 1]].contiguous().to(dev) for g in range(G)]
    tws = [inp["topk_w"][b[g]:b[g + 1]].contiguous().to(dev) for g in range(G)]
    ys = [torch.empty(b[g + 1] - b[g], cfg.H, dtype=torch.bfloat16, device=dev) for g in range(G)]
    wgus = [ep.local_weights(wgu, g, G) for g in range(G)]
    wdns = [ep.local_weights(wdn, g, G) for g in range(G)]

    def step():
        return ep.moe_expert_layer_ep_local(xs, idxs, tws, wgus, wdns, ys, cfg.E)

    for _ in range(warmup):
        assert step() == 0
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    # rows that leave their rank: each routed row whose expert lives elsewhere
    idx = inp["topk_idx"]
    owner = idx // (cfg.E // G)
    src = torch.repeat_interleave(torch.arange(G), torch.tensor([b[g + 1] - b[g] for g in range(G)]))
    remote = int((owner != src[:, None]).sum())
    row_out = cfg.H // 2 + cfg.H // 16 + 4
    return {"simulated_ranks": G, "ms_per_step": ms, "tokens_per_s": cfg.T / (ms * 1e-3),
            "remote_rows": remote, "nvlink_bytes_per_step": remote * (row_out + 2 * cfg.H),
            "bf16_dispatch_bytes_would_be": remote * (2 * cfg.H + 2 * cfg.H),
            "note": "one GPU drives all ranks (exchanges are device copies); results equal the strict layer "
                    "bit for bit (tests/test_gpu_ep.py)"}


WORKLOAD_NAMES = {
    "toy": "toy NVFP4 MoE layer (E=4, T=256, top-2, K=256 -> N=512)",
    "dense4b": "dense Qwen3-4B-shaped W4A4 MLP (T=8192, 2560 -> 2x9728 -> 2560, 0.1% outlier channels x30)",
    "moe30b": "Qwen3-30B-A3B-shaped MoE expert layer (moe30b)",
    "moe30b_skew": "Qwen3-30B-A3B-shaped MoE layer, 65536 tokens, Zipf(1.2) skewed routing (moe30b_skew)",
}


def run_ours(args, rank, world, local_rank):
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = rank_config(workloads.CONFIGS[args.config], rank, world)
    fp4 = fp4_peak()
    m = measure_layer(cfg, args, world, dev, args.steps, args.warmup, fp4)
    result = {
        "metric": METRIC,
        "value": m["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 scales) -> f32 accumulate, bf16 out",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights, softmax top-8 routing)",
        "config": {"workload": WORKLOAD_NAMES.get(cfg.name.split("+")[0], cfg.name), "tokens_per_gpu": cfg.T,
                   "hidden": cfg.H, "intermediate": cfg.I, "experts": cfg.E, "top_k": cfg.k,
                   "scaling_mode": "per-tensor" if args.per_tensor else "per-token",
                   "parallelism": f"dp{world} (replicas, no data-path collective)",
                   "l2": "no flush: per-step working set ~1.5 GB (weights 340 MB + activations) > 126 MB L2"},
        "tflops": m["tflops"],
        "stages_ms": m["stages_ms"],
        "stage_timing": m["stage_timing"],
        "profiled_ms_per_step": m["profiled_ms_per_step"],
        "graph_ms_per_step": m["graph_ms_per_step"],
        "step_ms_min_max": m["step_ms_min_max"],
        "quantizer_gbs": next(r["gbs"] for r in m["roofline"]["kernels"] if r["stage"] == "quantize_permute"),
        "roofline": m["roofline"],
        "e2e": m["e2e"],
        "gpu_launches": m["gpu_launches"],
        "clocks": m["clocks"],
        "fp4_mma_peak_tflops": fp4,
    }
    if world == 1 and not args.per_tensor and not args.no_fast_combine:
        # the non-strict combine (FP32 reductions from the down GEMM's epilogue,
        # no D round trip): measured beside the headline strict-order step
        fc = measure_layer(cfg, args, world, dev, max(10, args.steps // 2), max(3, args.warmup), fp4,
                           clocks_for_timed=False, extra_flags=FAST_COMBINE_FLAG)
        result["fast_combine"] = {"value": fc["value"], "ms_per_step": fc["ms_per_step"],
                                  "stages_ms": fc["stages_ms"],
                                  "note": "NVFP4MOE_FAST_COMBINE: non-strict (reduction order varies), "
                                          "not bitwise reproducible; the headline value is the strict-order path"}
    if world == 1 and not args.per_tensor and not args.no_fast_combine:
        # the requantization fused into the gate_up GEMM (opt-in): measured
        # beside the headline's separate pass
        fr = measure_layer(cfg, args, world, dev, max(10, args.steps // 2), max(3, args.warmup), fp4,
                           clocks_for_timed=False, extra_flags=FUSED_REQUANT_FLAG)
        result["fused_requant"] = {"value": fr["value"], "ms_per_step": fr["ms_per_step"],
                                   "stages_ms": fr["stages_ms"],
                                   "note": "NVFP4MOE_FUSED_REQUANT: requantization inside the gate_up GEMM "
                                           "(bitwise the same outputs); off by default because it is slower"}
    if world == 1 and not args.no_backward:
        result["backward"] = measure_backward(cfg, dev, max(5, args.steps // 5), 2)
        torch.cuda.empty_cache()
    if world == 1 and not args.no_variants:
        result["router_gemm"] = measure_router(cfg, dev, 20, 3)
        result["expert_parallel"] = measure_ep(cfg, dev, 5, 2, 4)
        torch.cuda.empty_cache()
        for kind in ("w4a16", "w4a8"):
            result[kind] = measure_variant(cfg, dev, max(5, args.steps // 5), 3, kind)
            torch.cuda.empty_cache()
        torch.cuda.empty_cache()
    if world == 1 and args.workloads:
        extra = {}
        for name in [w for w in args.workloads.split(",") if w and w != args.config]:
            wcfg = workloads.CONFIGS[name]
            wm = measure_layer(wcfg, args, world, dev, args.workload_steps, max(3, args.warmup), fp4,
                               clocks_for_timed=False)
            extra[name] = {"workload": WORKLOAD_NAMES.get(name, name), "value": wm["value"], "unit": "tokens/s",
                           "ms_per_step": wm["ms_per_step"], "graph_ms_per_step": wm["graph_ms_per_step"],
                           "tflops": wm["tflops"], "steps": args.workload_steps,
                           "stages_ms": wm["stages_ms"], "roofline": wm["roofline"], "e2e": wm["e2e"],
                           "gpu_launches": wm["gpu_launches"],
                           "config": {"tokens": wcfg.T, "hidden": wcfg.H, "intermediate": wcfg.I,
                                      "experts": wcfg.E, "top_k": wcfg.k, "routing": wcfg.routing}}
            result["gpu_launches"] += wm["gpu_launches"]
            torch.cuda.empty_cache()
        result["workloads"] = extra
    return result, cfg


def load_traffic(kernel_key: str):
    """DRAM bytes per launch of a GEMM launch from profiles/traffic.txt (one ncu
    capture), or None when the kernel source changed since that capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    src = os.path.join(ROOT, "nvfp4_moe_grouped_token_b200", "csrc", "gemm.cu")
    if not os.path.exists(path) or not os.path.exists(src):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 2 and not line.startswith("#"):
                vals[parts[0]] = parts[1]
    with open(src, "rb") as f:
        if hashlib.sha1(f.read()).hexdigest() != vals.get("gemm_sha1"):
            return None
    v = vals.get(kernel_key)
    return None if v is None else int(v)


# ------------------------------------------------------- oracle (CPU) ----

def oracle_sample(cfg, inp, n_experts: int, per_token: bool, wq=None, max_rows: int = 1 << 30):
    """Time the C++ CPU oracle on the routed rows of the first n_experts
    experts, at most max_rows of them (a bounded slice of the same workload):
    quantize the tokens, permute, gate_up GEMM, SwiGLU, BF16, requantize h,
    down GEMM, BF16 D.  The weights are quantized once, outside the timed
    part.  Returns (seconds, rows, weights)."""
    import numpy as np
    from oracle import cpp

    idx = inp["topk_idx"].numpy()
    if wq is None:
        def deq(w):
            out = np.empty(w.shape, np.float64)
            for e in range(w.shape[0]):
                q = cpp.quantize(w[e], False)
                out[e] = cpp.dequantize(q["q"], q["sf"], q["s_dec"])
            return out
        wq = (deq(inp["w_gate_up"][:n_experts].float().numpy()), deq(inp["w_down"][:n_experts].float().numpy()))
    x = inp["x"].float().numpy()
    t0 = time.perf_counter()
    info = cpp.permutation(idx, cfg.E)
    hi = min(int(info["offsets"][n_experts]), max_rows)
    tok = info["perm"][:hi] // cfg.k
    utok = np.unique(tok)
    if per_token:
        qx = cpp.quantize(x[utok], True)
        a = cpp.dequantize(qx["q"], qx["sf"], qx["s_dec"])[np.searchsorted(utok, tok)]
    else:
        qx = cpp.quantize(x, False)
        a = cpp.dequantize(qx["q"], qx["sf"], qx["s_dec"])[tok]
    off = np.minimum(info["offsets"][: n_experts + 1], hi).astype(np.int32)
    gu = cpp.grouped_gemm(a, off, wq[0])
    h = cpp.round_to_bf16(cpp.swiglu(gu, cfg.I))
    qh = cpp.quantize(h, per_token)
    hh = cpp.dequantize(qh["q"], qh["sf"], qh["s_dec"])
    d = cpp.round_to_bf16(cpp.grouped_gemm(hh, off, wq[1]))
    _ = d.sum()
    return time.perf_counter() - t0, hi, wq


def cpu_cores_used():
    """Threads the C++ oracle runs its GEMMs on (one per host core)."""
    from oracle import cpp
    return cpp.threads()


def cpu_baseline(cfg, n_experts: int, per_token: bool, max_rows: int = 1 << 30):
    inp = workloads.layer_inputs(cfg)
    n_experts = min(n_experts, cfg.E)
    secs, rows, _ = oracle_sample(cfg, inp, n_experts, per_token, max_rows=max_rows)
    return {"value": rows / cfg.k / secs, "unit": "tokens/s", "cores": cpu_cores_used(), "kind": "oracle",
            "sample": f"the first {rows} of the {cfg.T * cfg.k} routed rows (experts 0..{n_experts - 1}), "
                      f"rate reported per token = rows/s / k; {secs:.1f} s of CPU time"}


# experts whose routed rows form each extra workload's cpu_baseline sample
WORKLOAD_CPU_EXPERTS = {"toy": 4, "dense4b": 1, "moe30b_skew": 2}
WORKLOAD_CPU_ROWS = {"dense4b": 1024}      # dense4b's one expert holds all 8192 rows (~50 s of oracle work)


def run_reference(args, rank, world):
    cfg = workloads.CONFIGS[args.config]
    per_token = not args.per_tensor
    if rank != 0:
        return None
    inp = workloads.layer_inputs(cfg)
    wq = None
    for _ in range(args.warmup):
        _, _, wq = oracle_sample(cfg, inp, args.ref_experts, per_token, wq)
    secs, rows = 0.0, 0
    for _ in range(args.steps):
        s, r, wq = oracle_sample(cfg, inp, args.ref_experts, per_token, wq)
        secs += s
        rows += r
    value = rows / cfg.k / secs
    sample = (f"routed rows of experts 0..{args.ref_experts - 1} per step ({rows // args.steps} rows), "
              f"rate per token = rows/s / k")
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (C++ oracle)", "data": "synthetic",
        "config": {"workload": f"Qwen3-30B-A3B-shaped MoE expert layer ({cfg.name})",
                   "tokens_per_gpu": cfg.T, "hidden": cfg.H, "intermediate": cfg.I, "experts": cfg.E,
                   "top_k": cfg.k, "scaling_mode": "per-tensor" if args.per_tensor else "per-token"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores; other ranks have no work
        res = run_reference(args, rank, world)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res, cfg = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(cfg, args.cpu_experts, not args.per_tensor)
            for name, wl in res.get("workloads", {}).items():
                # a smaller sample per extra workload (a few seconds each)
                wl["cpu_baseline"] = cpu_baseline(workloads.CONFIGS[name], WORKLOAD_CPU_EXPERTS.get(name, 8),
                                                  not args.per_tensor, max_rows=WORKLOAD_CPU_ROWS.get(name, 1 << 30))
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
