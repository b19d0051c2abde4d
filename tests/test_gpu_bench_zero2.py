"""bench.py's ZeRO-2 mode on one rank: the degenerate form of the whole-model
ZeRO-2 step (one slice, no peers, the stream barriers a no-op), run the way
the driver runs bench.py, so that the multi-GPU form has a tested entry."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_zero2_bench_mode_on_one_rank():
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    out = subprocess.run([sys.executable, "bench.py", "--zero2", "--workload", "tiny", "--steps", "3", "--warmup", "3"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["n_gpus"] == 1 and line["steps"] == 3 and line["scaling"] == "strong"
    assert line["config"]["numel_model"] == line["config"]["numel_per_rank"] == 1 << 20
    assert line["gpu_launches"] == 9          # per step: pass 1, the decision, pass 2
    assert line["nvlink"]["bytes_per_rank_per_step"] == 0 and line["roofline"]["bound"] == "hbm"
    assert line["value"] > 0 and line["ms_per_step"] > 0
