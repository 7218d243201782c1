"""bench.py on the CPU: the reference arm's JSON line and the pure helpers
that turn event times into the reported throughput and roofline figures."""
import json
import os
import subprocess
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from nvfp4_moe_grouped_token_b200 import workloads  # noqa: E402


def test_layer_flops_closed_form():
    cfg = workloads.CONFIGS["moe30b"]
    f = bench.layer_flops(cfg)
    # 2 * rows * K * N for each GEMM, rows = T * k = 131072
    assert f["gate_up"] == 2 * 131072 * 2048 * 1536
    assert f["down"] == 2 * 131072 * 768 * 2048
    assert abs(f["total"] - 1.237e12) / 1.237e12 < 1e-3


def test_stage_bytes_count_each_tensor_once():
    cfg = workloads.CONFIGS["moe30b"]
    R, H, I, E = 131072, 2048, 768, 128
    nv = 0.5625
    # separate requantization: h leaves gate_up in BF16 and a second pass requantizes it
    for per_tensor in (False, True):
        b = bench.stage_bytes(cfg, per_tensor=per_tensor)
        assert b["combine"] == R * H * 2 + 16384 * H * 2 + R * 8
        assert b["down"] == R * I * nv + E * H * I * nv + R * H * 2
        assert b["gate_up_swiglu"] == R * H * nv + E * 2 * I * H * nv + R * I * 2
        assert b["requant_h"] == R * I * (2 + nv)
    # fused into gate_up (per-token only): the GEMM writes h's codes, no requant stage
    b = bench.stage_bytes(cfg, per_tensor=False, fused_requant=True)
    assert b["gate_up_swiglu"] == R * H * nv + E * 2 * I * H * nv + R * I * nv
    assert "requant_h" not in b
    # the whole step moves about 2 GB at the moe30b shape (the survey's figure)
    total = sum(bench.stage_bytes(cfg, per_tensor=False, fused_requant=True).values())
    assert 1.6e9 < total < 2.1e9


def test_kernel_rooflines_fractions_follow_from_the_times():
    cfg = workloads.CONFIGS["moe30b"]
    stage_ms = {"route": 0.02, "quantize_permute": 0.05, "gate_up_swiglu": 0.2, "down": 0.15, "combine": 0.1}
    pk = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}
    fp4 = {"mma_only": 8000.0, "with_scale_writes": 7500.0}
    rows = {r["stage"]: r for r in bench.kernel_rooflines(cfg, stage_ms, False, pk, fp4, None)}
    fl = bench.layer_flops(cfg)
    sb = bench.stage_bytes(cfg, False)
    gu = rows["gate_up_swiglu"]
    assert abs(gu["tflops"] - fl["gate_up"] / 0.2e-3 / 1e12) < 1e-6
    assert abs(gu["frac_fp4_peak"] - gu["tflops"] / 8000.0) < 1e-12
    assert rows["route"]["bound"] == "latency"
    for name in ("quantize_permute", "down", "combine"):
        r = rows[name]
        assert abs(r["gbs"] - sb[name] / (stage_ms[name] * 1e-3) / 1e9) < 1e-6
        assert abs(r["frac_hbm"] - r["gbs"] / 6500.0) < 1e-12


def test_job_throughput_is_all_tokens_over_slowest_rank():
    assert bench.job_throughput(16384, 1, 1.0) == 16384e3
    assert bench.job_throughput(16384, 4, 2.0) == 4 * 16384 / 2e-3


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                          "--ref-experts", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_clock_sampler_reports_the_timed_window_from_nvml(monkeypatch):
    """A fake NVML: idle clocks before the window, loaded clocks with the power
    cap active inside it, thermal slowdown after it."""
    import time
    import types

    phase = {"p": "before"}
    fake = types.ModuleType("pynvml")
    fake.NVML_CLOCK_SM = 0
    fake.nvmlInit = lambda: None
    fake.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)

    def by_bus(_):
        raise RuntimeError("no such bus id")
    fake.nvmlDeviceGetHandleByPciBusId = by_bus
    fake.nvmlDeviceGetClockInfo = lambda h, kind: {"before": 300, "in": 1900, "after": 1100}[phase["p"]]
    fake.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: {"before": 0x1, "in": 0x4, "after": 0x40}[phase["p"]]
    monkeypatch.setitem(sys.modules, "pynvml", fake)

    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.05)
    phase["p"] = "in"
    time.sleep(0.02)
    c.mark_begin()
    time.sleep(0.08)
    c.mark_end()
    time.sleep(0.02)
    phase["p"] = "after"
    time.sleep(0.05)
    r = c.stop()
    assert r["source"] == "nvml" and r["in_timed_region"] is True
    assert r["samples"] >= 3
    assert r["sm_mhz"] == 1900 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]
