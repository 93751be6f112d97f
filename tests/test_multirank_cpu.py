"""The multi-rank plumbing of bench.py on CPU: two gloo ranks over 127.0.0.1 (barrier, the
max over ranks that the timing takes), and the reference arm under torchrun, which rank 0
alone runs and prints."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["SDPA_ROOT"])
import bench, torch
rank, world, _ = bench.init_dist(2, backend="gloo")
bench.barrier(world)
ms = bench.max_over_ranks(1.5 + rank, world)
bench.barrier(world)
print(json.dumps({"rank": rank, "world": world, "max_ms": ms}))
torch.distributed.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    env = dict(os.environ)
    env.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
               WORLD_SIZE=str(world), SDPA_ROOT=ROOT, CUDA_VISIBLE_DEVICES="")
    return env


def test_two_gloo_ranks_agree_on_the_slowest_time():
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, "-c", WORKER], env=_env(r, 2, port), stdout=subprocess.PIPE,
                              stderr=subprocess.PIPE, text=True) for r in range(2)]
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("gloo ranks did not finish")
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(o["rank"] for o in outs) == [0, 1]
    assert all(o["world"] == 2 and o["max_ms"] == 2.5 for o in outs)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "3",
           "--reference-heads", "1"]
    p = subprocess.run(cmd, env=_env(rank, 2, _free_port()), capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    if rank == 1:
        assert p.stdout.strip() == ""
    else:
        line = json.loads(p.stdout.strip().splitlines()[-1])
        assert line["impl"] == "reference" and line["n_gpus"] == 2
        assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
