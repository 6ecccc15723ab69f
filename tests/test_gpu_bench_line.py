"""The bench's JSON line on the GPU: one short run per kind of workload
(single instance with an end-to-end host-streamed rate, batched with the
per-step copy rate) must carry every key of the reporting contract, with
values that are consistent with each other."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches",
        "value_call", "value_graph_call", "phases"]


def _bench(*args):
    p = subprocess.run([sys.executable, "bench.py", "--steps", "3", "--warmup", "3", "--min-timed-s", "0.05",
                        "--cpu-seconds", "0.5", *args], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert p.returncode == 0, p.stderr[-2000:]
    return json.loads(p.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("workload", ["small_f32", "batch512_k256"])
def test_bench_line_carries_the_contract(workload):
    d = _bench("--workload", workload)
    for k in KEYS:
        assert k in d, k
    assert d["config"]["workload"] == workload
    # value is the iteration rate of ms_per_step (rounded to 0.1 us in the line)
    assert d["value"] > 0 and abs(d["value"] * d["ms_per_step"] / 1e3 - 1) < 0.01
    assert d["gpu_launches"] > 0 and d["gpu_launches_per_repeat"] * d["repeats"] == d["gpu_launches"]
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert d["value_graph_call"] > 0 and d["value_call"] > 0
    rf = d["roofline"]
    assert rf["bound"] in ("tensor", "hbm") and 0 < rf["frac"] < 2 and rf["achieved"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
