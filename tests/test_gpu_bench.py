"""bench.py on the GPU, on small cases: the line carries every field the
measurement needs (value, roofline with its peak and fraction, the oracle's CPU
figure, the end-to-end figure with its copied bytes, clocks, launch count), and
the log-quantizer mode reports its issue roofline.  The full-size line is the
benchmark itself; these runs only check its shape, on workloads small enough to
finish in seconds."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    return json.loads(p.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("workload,coords", [("normal_seg_d2^30_w8_ef", 1 << 22),
                                             ("gpt2s_laplace_w8", 1 << 22)])
def test_bench_line_fields(workload, coords):
    line = run_bench("--workload", workload, "--coords", str(coords), "--steps", "4",
                     "--warmup", "3", "--no-extras")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "config", "roofline", "clocks",
                "e2e", "gpu_launches", "cpu_baseline", "cpu_baseline_threads"):
        assert key in line, key
    assert line["value"] > 0 and line["gpu_launches"] == 8
    assert line["config"]["workload"] == workload and line["config"]["d"] == coords
    roof = line["roofline"]
    assert roof["bound"] == "hbm" and roof["peak"] > 0 and 0 < roof["frac"] < 2
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-3
    e2e = line["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] == 4 * 8 * coords
    assert e2e["api"].startswith("pipelined") and 0 < e2e["frac_of_host_link"] < 1.2
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] == 1 and cpu["value"] > 0


def test_lq_mode_reports_its_issue_roofline():
    line = run_bench("--lq", "--steps", "10", "--no-cpu-baseline")
    assert [r["rank"] for r in line["rows"]] == [1, 4, 7]
    for r in line["rows"]:
        roof = r["roofline"]
        # the committed instruction count matches the sources: the roofline is the issue peak
        assert roof["bound"] == "alu", roof.get("note")
        assert 0 < roof["frac"] < 1.0
        assert roof["decode_sum_kernel"]["avg_launch_ms"] > 0


def test_power_mode_reports_clocks_per_segment():
    line = run_bench("--power")
    assert line["mode"] == "power" and len(line["rows"]) == 9
    for r in line["rows"]:
        assert 0 < r["frac"] < 2 and r["sm_mhz"] and r["sm_mhz"] > 0
        assert r["frac_at_max_clock"] >= r["frac"] - 1e-9
