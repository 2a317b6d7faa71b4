"""The benchmark's reference arm (the oracle on host cores) on CPU: it reports
the megakernel arm's metric, unit and workload with exactly K timed and W
warm-up steps, and only rank 0 prints."""
import json
import os
import subprocess
import sys
from types import SimpleNamespace

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _run(extra_env, *args):
    env = dict(os.environ, MK_REF_BUDGET_S="5", **extra_env)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          *args], capture_output=True, text=True, env=env, timeout=600, check=True)
    return [ln for ln in out.stdout.splitlines() if ln.startswith("{")]


def test_reference_line_matches_the_megakernel_arm_workload():
    lines = _run({}, "--workload", "qwen05b", "--steps", "3", "--warmup", "3")
    assert len(lines) == 1
    d = json.loads(lines[0])
    spec = bench.workload_spec(SimpleNamespace(workload="qwen05b", layers=0, steps=3, warmup=3))
    assert d["impl"] == "reference"
    assert (d["metric"], d["unit"], d["config"]["workload"]) == (spec.metric, spec.unit,
                                                                 spec.workload)
    assert (d["steps"], d["warmup"], d["higher_is_better"]) == (3, 3, False)
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_on_rank_zero_only():
    assert _run({"RANK": "1"}, "--workload", "qwen05b", "--steps", "3", "--warmup", "3") == []


def test_workload_spec_per_workload():
    def spec(wl, steps=504, warmup=8):
        return bench.workload_spec(SimpleNamespace(workload=wl, layers=0, steps=steps,
                                                   warmup=warmup))
    d = spec("llama8b")
    assert (d.n, d.lens, d.K, d.W, d.unit, d.metric) == (1, [39], 504, 8, "ms/token", bench.METRIC)
    assert "steps 47..550 timed" in d.workload
    d = spec("llama8b-32k")
    assert (d.lens, d.K, d.unit) == ([32768], 248, "ms/token")   # 256 decode steps in all
    d = spec("llama8b-batch8")
    assert d.n == 8 and d.K == 248 and d.unit == "ms/step" and "8 requests" in d.metric
    assert all(32 <= n <= 2048 for n in d.lens)
    d = spec("qwen05b", steps=10, warmup=3)
    assert d.model.name.startswith("qwen") and "Qwen2.5-0.5B-shape" in d.metric and d.K == 10
