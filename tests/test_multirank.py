"""The N > 1 path of bench.py, on the CPU: one process per rank joins the
process group through the helpers the bench uses (gloo here, NCCL on GPUs),
the ranks take the max of their step times (the slowest replica sets the job's
time) and agree on the whole-job throughput; the reference arm prints on rank
0 only, and the other ranks exit 0 without work."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, os, sys
sys.path.insert(0, {root!r})
import torch
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
joined = bench.init_ranks(world, backend="gloo")
ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"), joined)
value = bench.job_throughput(131072, world, ms)
print(json.dumps({{"rank": rank, "joined": joined, "ms": ms, "value": value}}), flush=True)
torch.distributed.barrier()
torch.distributed.destroy_process_group()
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _env(rank, world, port):
    env = dict(os.environ)
    env.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
               WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return env


def test_two_gloo_ranks_take_the_slowest_step():
    port, world = _free_port(), 2
    code = WORKER.format(root=ROOT)
    procs = [subprocess.Popen([sys.executable, "-c", code], env=_env(r, world, port), cwd=ROOT,
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
             for r in range(world)]
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(o["rank"] for o in outs) == [0, 1]
    for o in outs:
        assert o["joined"] is True
        assert o["ms"] == 15.0                      # the slower rank's time
        assert o["value"] == 131072 * world / 0.015  # tokens of every rank / that time


def test_one_rank_joins_no_group():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_ranks(1) is False
    assert bench.max_over_ranks(3.5, torch.device("cpu"), False) == 3.5
    assert bench.job_throughput(1000, 1, 500.0) == 2000.0


def test_reference_arm_prints_on_rank_zero_only():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT,
                       env=_env(1, 2, _free_port()), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
