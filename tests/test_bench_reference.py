"""bench.py's reference arm (the float64 oracle on the host cores): one JSON
line with the keys of the benchmark contract, for a decode step and for a
verification step (CPU only, a tiny workload and a short time budget)."""
import json
import os
import subprocess
import sys

import pytest

import bench
from kv_cache_bandwidth_b200.workloads import WORKLOADS, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_reference(*extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "2", "--warmup", "3", "--oracle-seconds", "0.05", *extra]
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("extra", [(), ("--query-tokens", "3")], ids=["decode", "verify3"])
def test_reference_line(extra):
    d = run_reference(*extra)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    # the same workload description as the GPU arm's line (no plan in it)
    assert d["config"] == bench.config_dict(WORKLOADS["tiny"], make_inputs(WORKLOADS["tiny"]),
                                            int(extra[1]) if extra else 1)
    if extra:
        assert d["config"]["query_tokens"] == 3
        assert "3 query tokens" in d["cpu_baseline"]["sample"]
