"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.

bench.py runs one process per GPU under torchrun; its process group carries
only a barrier and the max-reduce of the ranks' timings, and the reported
value is the units all ranks processed over the slowest rank's time.  These
tests run that plumbing with world size 2 on the gloo backend (no GPU), and
check that the reference arm does no work on ranks other than 0.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

_WORKER = r"""
import json, os, sys, time
sys.path.insert(0, {root!r})
import bench
rank, world, local = bench.dist_setup(2, backend="gloo")
bench.barrier(world)
t_local = 0.25 + 0.5 * rank          # rank 1 is the slower one
t = bench.max_over_ranks(t_local, world)
value = bench.job_throughput(100, world, t)
bench.barrier(world)
if rank == 0:
    print(json.dumps({{"world": world, "t": t, "value": value}}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(code, world):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=120)
        except subprocess.TimeoutExpired:
            p.kill()
            o, e = p.communicate()
        outs.append((p.returncode, o, e))
    return outs


def test_two_gloo_ranks_take_the_max_time_and_sum_the_units():
    outs = _launch(_WORKER.format(root=ROOT), 2)
    for rc, o, e in outs:
        assert rc == 0, e
    import json
    line = json.loads(outs[0][1].strip().splitlines()[-1])
    assert line["world"] == 2
    assert line["t"] == pytest.approx(0.75)
    assert line["value"] == pytest.approx(2 * 100 / 0.75)
    assert outs[1][1].strip() == ""  # only rank 0 prints


def test_job_throughput_single_rank():
    assert bench.job_throughput(20000, 1, 0.5) == pytest.approx(40000.0)


def test_reference_arm_does_nothing_on_other_ranks():
    code = (f"import sys; sys.path.insert(0, {ROOT!r}); import bench, time\n"
            "class A: steps = 10**9; warmup = 3; gpus = 2\n"
            "t0 = time.time(); bench.run_reference(A()); print(round(time.time() - t0, 3))\n")
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert float(r.stdout.strip()) < 1.0
