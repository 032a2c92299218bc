"""`bench.py --gpus N` started as one plain process launches N ranks itself
(under torch.distributed.run on 127.0.0.1); rank 0 alone prints the line,
with n_gpus = N and the max-over-ranks time. Checked on CPU through the
launch-only dry run (gloo process group, no workload)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("extra", [[], ["--eager"]], ids=["graph", "eager"])
def test_bench_gpus_2_launches_two_ranks(extra):
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                            "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run"] + extra,
                       capture_output=True, text=True, timeout=240, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2
    assert d["ms_per_step"] == 2.0            # max over ranks of (1 + rank)
