"""The synthetic layer-stack step of bench.py (--layers): runs on the GPU, stays finite,
and reports the speed-ups it is meant to report."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_layer_step_mode_runs_and_reports():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--layers", "2", "--workload", "tiny",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["unit"] == "x" and line["config"]["layers"] == 2
    for k in ("lazyflash", "dense"):
        assert line["ms_per_step"][k] > 0 and line["attention_fwd_bwd"]["ms"][k] > 0
    assert line["value"] > 0 and line["attention_fwd_bwd"]["speedup"] > 0
