"""The bench's multi-rank plumbing on host ranks (gloo, world size 2): the
process group from torchrun's environment, the barrier, the max over ranks of
the device time, and the reference arm's rank-0-only output."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_setup(backend="gloo")
    bench.barrier(w)
    longest = bench.max_over_ranks(10.0 + 5.0 * r, w, device="cpu")
    bench.barrier(w)
    q.put((r, w, local, longest))
    torch.distributed.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 2, 0, 15.0), (1, 2, 1, 15.0)]


def _bench(env_extra):
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", **env_extra)
    return subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
         "--steps", "1", "--warmup", "3", "--gpus", "2"],
        env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_on_rank_zero_only():
    # under torchrun every rank runs bench.py; only rank 0 times the oracle
    # and prints, the others exit 0 without output
    r1 = _bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _bench({"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"})
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["n_gpus"] == 2 and line["e2e"]["h2d_bytes_per_step"] == 0
