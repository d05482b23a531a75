"""The JSON line bench.py prints, both arms: the keys and the relations between
them that a reader of the line relies on.

The reference arm (the oracle on the host cores) runs here on CPU; the
library arm needs the GPU and runs a 2-layer step."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(args, timeout):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def _common(d, steps, warmup):
    assert d["metric"] and d["unit"] == "TFLOP/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == steps and d["warmup"] == warmup
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["data"] == "synthetic"
    assert d["config"]["workload"]


def test_reference_arm_line():
    d = _line(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "2"], 600)
    _common(d, 1, 3)
    assert d["impl"] == "reference" and d["dtype"] == "f64"
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["sample"]
    assert cpu["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


@pytest.mark.gpu
def test_library_arm_line():
    steps, warmup, layers = 3, 3, 2
    d = _line(["--layers", str(layers), "--steps", str(steps), "--warmup", str(warmup),
               "--no-cpu-baseline", "--no-configs"], 900)
    _common(d, steps, warmup)
    assert d.get("impl", "ours") != "reference"
    assert d["device_status"] == 0
    # the launches of the timed region: 11 per layer plus the amax pass of
    # layer 0's input, every step
    assert d["gpu_launches"] == (11 * layers + 1) * steps
    rl = d["roofline"]
    assert rl["bound"] == "tensor" and rl["unit"] == "TFLOP/s"
    assert rl["achieved"] > 0 and rl["peak"] > 0
    assert abs(rl["frac"] - rl["achieved"] / rl["peak"]) < 1e-9
    assert "traffic" in rl
    e2e = d["e2e"]
    assert e2e["unit"] == d["unit"] and e2e["value"] > 0
    # one bf16 2640 x 3072 input up and one output down per step
    assert e2e["h2d_bytes_per_step"] == 2640 * 3072 * 2
    assert e2e["d2h_bytes_per_step"] == 2640 * 3072 * 2
    # end to end cannot beat the device-resident step
    assert e2e["ms_per_step"] >= 0.98 * d["ms_per_step"]
    assert e2e["eager"]["value"] > 0 and e2e["eager"]["ms_per_step"] > 0
    clk = d["clocks"]
    assert clk is None or {"sm_mhz", "sm_max_mhz", "reasons"} <= set(clk)
