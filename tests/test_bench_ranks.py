"""bench.py under a multi-rank launch (host logic, no GPU): the one-GPU workloads (schedule
replays, paged prefill, the E4M3 decode) run on rank 0 only; any other rank exits 0 at
once, printing nothing and touching no GPU."""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", ["sharing_B", "prefill_opt13b_t16", "opt13b_fp8"])
def test_other_ranks_do_nothing(workload):
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "bench.py", "--workload", workload, "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
