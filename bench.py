"""Benchmark of the NVFP4 W4A4 MoE expert layer (one JSON line on rank 0).

Workload: the Qwen3-30B-A3B-shaped expert layer -- 16384 tokens, hidden 2048,
128 experts, top-8 softmax routing, gate_up 2048 -> 2x768 with SwiGLU and
NVFP4 requantization, down 768 -> 2048 -- on seeded synthetic BF16 data.  A
step is one moe_expert_layer call (every kernel of the path).  Per-token
scaling (the token-wise path) is the default; --per-tensor switches.

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
    ap.add_argument("--cpu-experts", type=int, default=30,
                    help="experts whose routed rows form the cpu_baseline sample (~10 s of oracle work)")
    ap.add_argument("--ref-experts", type=int, default=6,
                    help="experts whose routed rows form each step of --impl reference (~2 s per step)")
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


def stage_bytes(cfg, counts_pad_rows: int) -> dict:
    """Algorithmic HBM bytes per stage (each tensor read or written once)."""
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    R = T * k
    nv = 0.5 + 1.0 / 16                 # NVFP4 bytes per element (codes + UE4M3 scale)
    w_gu = E * 2 * I * H * nv
    w_dn = E * H * I * nv
    return {
        "quantize_permute": T * H * 2 + R * H * nv + R * 8,
        "gate_up_swiglu": R * H * nv + w_gu + R * I * 2,
        "requant_h": R * I * 2 + R * I * nv,
        "down": R * I * nv + w_dn + R * H * 2,
        "combine": R * H * 2 + T * H * 2 + R * 8,
    }


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

def run_ours(args, rank, world, local_rank):
    from nvfp4_moe_grouped_token_b200 import ops

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = rank_config(workloads.CONFIGS[args.config], rank, world)
    flags = 0 if args.per_tensor else ops.SCALE_PER_TOKEN
    inp = workloads.layer_inputs(cfg)
    x = inp["x"].to(dev)
    idx = inp["topk_idx"].to(dev)
    w = inp["topk_w"].to(dev)
    wgu = ops.nvfp4_prepare_weights(inp["w_gate_up"].to(dev), gate_up=True)
    wdn = ops.nvfp4_prepare_weights(inp["w_down"].to(dev), gate_up=False)
    ws = torch.empty(ops.moe_expert_layer_workspace_size(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, flags),
                     dtype=torch.uint8, device=dev)
    y = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ops.moe_expert_layer(x, idx, w, wgu, wdn, y, ws, flags)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ops.device_status(ws) == 0

    # ---- timed region: K steps, stage events on the launching stream -----
    nstage = len(ops.STAGES)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage + 1)] for _ in range(args.steps)]
    for row in evs:                          # materialise the events before timing
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.2)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks.mark_begin()
    t_start.record(stream)
    for i in range(args.steps):
        ops.moe_expert_layer_profiled(x, idx, w, wgu, wdn, y, ws, evs[i], flags)
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert ops.device_status(ws) == 0

    total_ms = t_start.elapsed_time(t_end)
    step_ms = [evs[i][0].elapsed_time(evs[i][nstage]) for i in range(args.steps)]
    stage_ms = {name: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                for j, name in enumerate(ops.STAGES)}
    ms = max_over_ranks(total_ms / args.steps, world, dev)

    # ---- end to end through the public API with host buffers ----------------
    xh = inp["x"].pin_memory()
    ih = inp["topk_idx"].pin_memory()
    wh = inp["topk_w"].pin_memory()
    yh = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
    xd, idd, wd = torch.empty_like(x), torch.empty_like(idx), torch.empty_like(w)

    def e2e_step():
        xd.copy_(xh, non_blocking=True)
        idd.copy_(ih, non_blocking=True)
        wd.copy_(wh, non_blocking=True)
        ops.moe_expert_layer(xd, idd, wd, wgu, wdn, y, ws, flags)
        yh.copy_(y, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 2)
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, dev)

    fl = layer_flops(cfg)
    pk = peaks()
    fp4_peak_sustained = pk["bf16_tflops_sustained"] * FP4_PER_BF16
    gu_ms = stage_ms["gate_up_swiglu"]
    gu_tflops = fl["gate_up"] / (gu_ms * 1e-3) / 1e12
    traffic = load_traffic("gate_up_swiglu")
    sb = stage_bytes(cfg, 0)
    result = {
        "metric": METRIC,
        "value": job_throughput(cfg.T, world, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 scales) -> f32 accumulate, bf16 out",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights, softmax top-8 routing)",
        "config": {"workload": f"Qwen3-30B-A3B-shaped MoE expert layer ({cfg.name})", "tokens_per_gpu": cfg.T,
                   "hidden": cfg.H, "intermediate": cfg.I, "experts": cfg.E, "top_k": cfg.k,
                   "scaling_mode": "per-tensor" if args.per_tensor else "per-token",
                   "parallelism": f"dp{world} (replicas, no data-path collective)",
                   "l2": "no flush: per-step working set ~1.5 GB (weights 340 MB + activations) > 126 MB L2"},
        "tflops": world * fl["total"] / (ms * 1e-3) / 1e12,
        "stages_ms": stage_ms,
        "step_ms_min_max": [min(step_ms), max(step_ms)],
        "gemm": {"gate_up_tflops": gu_tflops,
                 "down_tflops": fl["down"] / (stage_ms["down"] * 1e-3) / 1e12,
                 "fp4_peak_tflops_sustained": fp4_peak_sustained,
                 "down_hbm_gbs": sb["down"] / (stage_ms["down"] * 1e-3) / 1e9},
        "quantizer_gbs": sb["quantize_permute"] / (stage_ms["quantize_permute"] * 1e-3) / 1e9,
        "requant_gbs": sb["requant_h"] / (stage_ms["requant_h"] * 1e-3) / 1e9,
        "combine_gbs": sb["combine"] / (stage_ms["combine"] * 1e-3) / 1e9,
        "roofline": {"kernel": "k_grouped_gemm (gate_up + SwiGLU epilogue)", "bound": "tensor",
                     "achieved": gu_tflops, "peak": fp4_peak_sustained, "unit": "TFLOP/s",
                     "frac": gu_tflops / fp4_peak_sustained,
                     "peak_note": f"{pk['source']} sustained bf16 x {FP4_PER_BF16:g} (nominal FP4:BF16 ratio)",
                     "traffic": traffic},
        "e2e": {"value": job_throughput(cfg.T, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": xh.numel() * 2 + ih.numel() * 4 + wh.numel() * 4,
                "d2h_bytes_per_step": yh.numel() * 2},
        "gpu_launches": args.steps * (7 + (1 if args.per_tensor else 0)),
        "clocks": clk,
    }
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

def oracle_sample(cfg, inp, n_experts: int, per_token: bool, wq=None):
    """Time the CPU oracle on the routed rows of the first n_experts experts
    (a bounded slice of the same workload).  Returns (seconds, rows, weights)."""
    import numpy as np
    from oracle import moe, nvfp4

    idx = inp["topk_idx"].numpy()
    if wq is None:
        wgu = inp["w_gate_up"][:n_experts].float().numpy()
        wdn = inp["w_down"][:n_experts].float().numpy()
        wq = (moe.QuantWeights(wgu), moe.QuantWeights(wdn))
        for e in range(n_experts):
            wq[0].dequant(e), wq[1].dequant(e)
    x = inp["x"].float().numpy()
    t0 = time.perf_counter()
    info = moe.permutation(idx, cfg.E)
    hi = int(info["offsets"][n_experts])
    rows = np.arange(hi)
    tok = info["perm"][rows] // cfg.k
    utok = np.unique(tok)
    qx = nvfp4.quantize(x[utok], per_token) if per_token else nvfp4.quantize(x, False)
    xh_rows = nvfp4.dequantize(qx["q"], qx["sf"], qx["s_dec"])
    if per_token:
        a = xh_rows[np.searchsorted(utok, tok)]
    else:
        a = xh_rows[tok]
    off = info["offsets"][: n_experts + 1]
    gu = moe.grouped_gemm(a, off, wq[0].dequant)
    h = nvfp4.round_to_bf16(moe.swiglu(gu, cfg.I))
    qh = nvfp4.quantize(h, per_token)
    hh = nvfp4.dequantize(qh["q"], qh["sf"], qh["s_dec"])
    d = nvfp4.round_to_bf16(moe.grouped_gemm(hh, off, wq[1].dequant))
    _ = d.sum()
    return time.perf_counter() - t0, hi, wq


def cpu_cores_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(cfg, n_experts: int, per_token: bool):
    inp = workloads.layer_inputs(cfg)
    secs, rows, _ = oracle_sample(cfg, inp, n_experts, per_token)
    return {"value": rows / cfg.k / secs, "unit": "tokens/s", "cores": cpu_cores_used(), "kind": "oracle",
            "sample": f"routed rows of experts 0..{n_experts - 1} ({rows} of {cfg.T * cfg.k} rows), "
                      f"rate reported per token = rows/s / k; {secs:.1f} s of CPU time"}


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
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
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
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
