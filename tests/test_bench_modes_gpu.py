"""bench.py's paged and joint-value modes (full and latent output) run end to end on a small
workload and print one JSON line with the contract's keys (the timing itself is not checked)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("mode,call", [(["--paged"], "stief_append_decode_paged"),
                                       (["--joint"], "stief_decode_attention_joint_v"),
                                       (["--latent", "--joint"], "stief_decode_latent_joint_v")])
def test_bench_mode_runs(mode, call):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), *mode, "--workload", "tiny",
           "--steps", "3", "--warmup", "3", "--decode-iters", "3", "--no-cpu-baseline",
           "--clock-window", "0"]
    run = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert run.returncode == 0, run.stdout[-2000:] + run.stderr[-2000:]
    line = json.loads(run.stdout.strip().splitlines()[-1])
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["steps"] == 3
    assert call in line["config"]["step"] and call in line["roofline"]["kernel"]
    assert line["roofline"]["traffic"] is None
    assert line["e2e"]["value"] > 0 and line["gpu_launches"] == 3
