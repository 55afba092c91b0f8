"""bench.py's own arm keeps the JSON contract on a GPU: one line with the
metric, throughput, the roofline of the dominant kernel, the end-to-end
number through host buffers, clocks sampled during the timed region, the
oracle baseline and the count of the library's launches."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


@pytest.mark.timeout(900)
def test_bench_line_step16k():
    d = _run("--steps", "4", "--warmup", "3", "--cpu-seconds", "2")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3 and d["value"] > 0
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["config"]["workload"].startswith("step16k")
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9 and 0 < r["frac"] < 1.3
    assert r["traffic"] is None or r["traffic"] > 0
    e = d["e2e"]
    assert e["value"] > 0 and e["unit"] == d["unit"] and e["value"] < d["value"]
    assert e["h2d_bytes_per_step"] == 2 * 16384 * 768 * 2 and e["d2h_bytes_per_step"] == 2 * 16384 * 768 * 2
    # the copies alone bound the end-to-end step
    assert 0 < e["value"] <= 1.5 * e["copy_bound"]["value"]  # (loose: both are timed once)
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["value"] > 0 and c["cores"] >= 1 and c["sample"]
    clk = d["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(clk)
    assert d["gpu_launches"] >= 8 * d["steps"]
    assert d["device_status"] == 0
    # the step against the measured peaks and against the datasheet peaks
    sr = d["step_roofline"]
    assert abs(sr["frac"] - sr["roofline_ms"] / sr["measured_ms"]) < 1e-9
    sp = sr["spec"]
    assert sp["peaks"]["bf16_tflops"] == 2250.0 and sp["peaks"]["fp8_tflops"] == 4500.0
    assert 0 < sp["frac"] < sr["frac"] and 0 < sp["fwd_frac"] < sr["fwd_frac"]
    # the other two MLP workloads, run by the same command
    for wl, metric_word in (("fwd16k", "fwd tokens/s"), ("train49k", "fwd+bwd tokens/s")):
        o = d["also"][wl]
        assert "error" not in o, o
        assert o["config"].startswith(wl) and metric_word in o["metric"] and o["value"] > 0
        assert o["steps"] == d["steps"] and o["warmup"] == d["warmup"]
        assert 0 < o["step_roofline_frac"] < 1.3 and o["device_status"] == 0


@pytest.mark.timeout(900)
def test_bench_line_ce16k_small():
    d = _run("--workload", "ce16k", "--tokens", "2048", "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    assert d["config"]["workload"].startswith("ce16k") and d["value"] > 0
    assert d["roofline"]["kernel"] in ("ce_fwd", "ce_bwd_dlogits", "dx", "dw")
    assert d["gpu_launches"] > 0 and d["device_status"] == 0


@pytest.mark.timeout(900)
def test_bench_line_fwd16k():
    d = _run("--workload", "fwd16k", "--steps", "5", "--warmup", "3", "--cpu-seconds", "2")
    assert d["config"]["workload"].startswith("fwd16k") and d["value"] > 0
    assert d["roofline"]["kernel"] == "up_fused" and 0 < d["roofline"]["frac"] < 1.3
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 16384 * 768 * 2 and e["d2h_bytes_per_step"] == 16384 * 768 * 2
    assert 0 < e["value"] <= 1.5 * e["copy_bound"]["value"]  # (loose: both are timed once)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["gpu_launches"] >= 3 * d["steps"]
    assert d["device_status"] == 0
