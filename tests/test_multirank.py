"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

The attention path needs no exchange step, so N GPUs run N independent replicas; what crosses
ranks is only the timing (maximum over ranks) and the work done (sum over ranks), which give the
whole-job throughput.  Here two processes on the host run those reductions through bench.py's own
helpers with the gloo backend, and the reference arm's rule that only rank 0 runs and prints.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["REPO"])
import torch.distributed as dist
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank, world = dist.get_rank(), dist.get_world_size()
local_ms = [2.0, 5.0][rank]               # rank 1 is the slow one
local_bytes = [3e9, 7e9][rank]
out = {
    "max": bench.max_over_ranks(world, local_ms),
    "sum": bench.sum_over_ranks(world, local_bytes),
    "whole_job": bench.whole_job(world, local_bytes, local_ms),
}
bench.barrier(world)
dist.destroy_process_group()
print(json.dumps(out))
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(script: str, world: int = 2, extra_env=None, timeout: int = 120):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), REPO=ROOT, CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, e[-2000:]
        outs.append(o)
    return outs


def test_reductions_and_whole_job_rate_over_two_gloo_ranks():
    outs = [json.loads(o.strip().splitlines()[-1]) for o in _run_ranks(RANK_SCRIPT)]
    for o in outs:                         # every rank sees the same reduced values
        assert o["max"] == 5.0
        assert o["sum"] == 10e9
        rate, ms = o["whole_job"]
        assert ms == 5.0 and abs(rate - 10e9 / 5e-3) < 1.0   # all ranks' bytes over the slowest time


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(1, 3.0) == 3.0 and bench.sum_over_ranks(1, 4.0) == 4.0
    assert bench.whole_job(1, 8e9, 2.0) == (8e9 / 2e-3, 2.0)


def test_reference_arm_runs_on_rank_zero_only():
    # rank 1 of 2 returns at once and prints nothing (the oracle timing runs on rank 0 alone)
    script = r"""
import os, sys
sys.path.insert(0, os.environ["REPO"])
import bench
sys.argv = ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
bench.main()
"""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", REPO=ROOT, CUDA_VISIBLE_DEVICES="")
    p = subprocess.run([sys.executable, "-c", script], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=120)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""
