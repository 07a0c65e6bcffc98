"""The benchmark's JSON line, produced on the GPU: every key its contract
names, for a tensor-bound layer (CTA-pair GEMMs), a weight-streaming decode
step (HBM-bound) and a small float32 layer (one kernel, CUDA cores)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

COMMON = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
          "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
          "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"}


def run_bench(*args, timeout=600):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-3000:]
    return json.loads(lines[0])


@pytest.mark.parametrize("workload,bound,unit,dtype", [
    ("mixtral_shape_t1024_d4096_f14336_e2_k2_bf16", "tensor", "TFLOP/s", "bf16"),
    ("decode_t32_d4096_f14336_e8_k1_bf16", "hbm", "GB/s", "bf16"),
    ("silu_gated_t64_d64_f128_e8_k2_f32", "alu", "TFLOP/s", "f32"),
])
def test_bench_line_keeps_its_contract(workload, bound, unit, dtype):
    steps, warmup = 5, 3
    d = run_bench("--workload", workload, "--steps", str(steps), "--warmup", str(warmup),
                  "--no-workloads", "--cpu-seconds", "1")
    assert COMMON <= d.keys(), COMMON - d.keys()
    assert d["n_gpus"] == 1 and d["steps"] == steps and d["warmup"] == warmup
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == dtype and d["unit"] == "tokens/s"
    assert d["config"]["workload"] == workload
    # tokens/s is the step's tokens over its time
    T = d["config"]["T"]
    assert d["value"] == pytest.approx(T / (d["ms_per_step"] / 1e3), rel=1e-2)   # ms rounded to 4 places

    r = d["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= r.keys()
    assert r["bound"] == bound and r["unit"] == unit
    assert r["achieved"] > 0 and r["peak"] > 0
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-2)
    assert r["frac"] < 1.5                 # far above 1 would mean the timed kernel skipped work

    e = d["e2e"]
    assert {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"} <= e.keys()
    assert e["unit"] == d["unit"] and e["value"] > 0
    x_bytes = T * d["config"]["D"] * (2 if dtype == "bf16" else 4)
    assert e["h2d_bytes_per_step"] == x_bytes and e["d2h_bytes_per_step"] == x_bytes

    # the library's own launches in the timed region: a whole number per forward
    n = d["gpu_launches"]
    assert n > 0 and n % steps == 0 and 1 <= n // steps <= 9

    c = d["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= c.keys()

    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    assert cb["unit"] == d["unit"] and cb["sample"]
