"""bench.py's one JSON line on a small set: every key of the output contract, with values
that agree with each other (work, time, launches, copies).  Needs a B200."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def line():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--config", "1", "--steps", "4",
                        "--warmup", "3", "--no-cpu-baseline"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_contract_keys(line):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["steps"] == 4 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["dtype"] == "bf16"
    assert line["data"] == "synthetic" and "workload" in line["config"]


def test_values_agree(line):
    import synth
    from muon_newton_schulz_06_b200 import cost
    shapes = [(s.rows, s.cols) for s in synth.config_shapes(1)]
    work = cost.ns_flops(shapes)["algorithmic"]
    # value = algorithmic TFLOP per step / device time per step
    assert line["value"] == pytest.approx(work / (line["ms_per_step"] / 1e3) / 1e12, rel=1e-6)
    roof = line["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in roof, k
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"], rel=1e-9)
    e2e = line["e2e"]
    grads = sum(r * c * 2 for r, c in shapes)  # bf16 gradients in, bf16 weights out
    assert e2e["h2d_bytes_per_step"] == grads and e2e["d2h_bytes_per_step"] == grads
    assert e2e["value"] > 0
    # the persistent launch on this set: 3 momentum-pass kernels + 1 per step
    assert line["gpu_launches"] == 4 * line["steps"]
    assert line["clocks"]["sm_max_mhz"] and "reasons" in line["clocks"]
