"""The reference arm of bench.py (the fp64 oracle on the host cores) on CPU: one JSON line with the
contract's keys, the same workload string as the CUDA arm, and nothing printed by ranks other than 0."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run(args, env=None):
    e = dict(os.environ, **(env or {}))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                       capture_output=True, text=True, timeout=600, env=e, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.strip()]


@pytest.mark.parametrize("workload,args", [
    ("decode_int4", ["--steps", "1", "--warmup", "3"]),
    ("quant_int4", ["--steps", "1", "--warmup", "3", "--cpu-seconds", "1"]),
])
def test_reference_line(workload, args):
    lines = _run(["--workload", workload, *args])
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    if workload in bench.WORKLOADS:
        E, fmt, T, _ = bench.WORKLOADS[workload]
        assert d["config"]["workload"] == bench.layer_workload(workload, E, fmt, T)
        assert d["unit"] == "tokens/s" and d["metric"] == bench.METRIC
    else:
        E, fmt = bench.QUANT_WORKLOADS[workload]
        assert d["config"]["workload"] == bench.quant_workload(workload, E, fmt)


def test_other_ranks_print_nothing():
    assert _run(["--workload", "quant_int4", "--steps", "1", "--warmup", "3", "--cpu-seconds", "1"],
                env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []
