"""The benchmark's replica plumbing at world size 2, on CPU (gloo): process-group start-up
from the launcher's environment, the barrier, the max-over-ranks time and the
sum-over-ranks token count; and the reference arm, which only rank 0 runs."""
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import importlib.util, json, os, sys
spec = importlib.util.spec_from_file_location("bench_rank", os.path.join(sys.argv[1], "bench.py"))
b = importlib.util.module_from_spec(spec)
spec.loader.exec_module(b)
ws, rank, local = b.dist_init()
b.barrier(ws)
out = {"ws": ws, "rank": rank, "max": b.max_over_ranks(1.5 + rank, ws), "sum": b.sum_over_ranks(10.0 * (rank + 1), ws)}
b.barrier(ws)
import torch.distributed as dist
backend = dist.get_backend()
dist.destroy_process_group()
out["backend"] = backend
print(json.dumps(out), flush=True)
"""


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_env(rank, ws, port):
    env = dict(os.environ, WORLD_SIZE=str(ws), RANK=str(rank), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
    return env


def test_two_ranks_reduce_max_time_and_total_tokens():
    import json
    port = free_port()
    procs = [subprocess.Popen([sys.executable, "-c", RANK_SCRIPT, ROOT], env=rank_env(r, 2, port),
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True) for r in range(2)]
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=120)
        assert p.returncode == 0, e
        outs.append(json.loads(o.strip().splitlines()[-1]))
    for o in outs:
        assert o["ws"] == 2 and o["backend"] == "gloo"
        assert o["max"] == 2.5           # the slower rank's time
        assert o["sum"] == 30.0          # every rank's tokens
    assert sorted(o["rank"] for o in outs) == [0, 1]


def test_reference_arm_runs_on_rank_zero_only():
    env = rank_env(1, 2, free_port())
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""
