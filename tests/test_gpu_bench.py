"""bench.py end to end on the GPU: one short run of the decode step, checked for
the keys of its JSON line and for an end-to-end figure that moved host bytes."""
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("workload", ["gqa70b", "fp8_prefix"])
def test_bench_decode_line(workload):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", workload,
           "--steps", "5", "--warmup", "3", "--e2e-steps", "50", "--no-cpu-baseline"]
    run = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stderr[-2000:]
    lines = [l for l in run.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, run.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "roofline", "e2e", "gpu_launches", "clocks", "config"):
        assert key in d, key
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["gpu_launches"] > 0
    assert d["roofline"]["achieved"] > 0 and d["roofline"]["peak"] > 0
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert e["eager_ms_per_step"] > 0
    # the reported form is the faster of those timed
    times = [t for t in (e["eager_ms_per_step"], e["graph_ms_per_step"]) if t is not None]
    assert abs(e["ms_per_step"] - min(times)) <= 1e-4
