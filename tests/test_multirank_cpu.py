"""Multi-rank plumbing of bench.py on CPU with the gloo backend (world size 2).

The hot path shards by independent (b, h) units, so ranks share no data:
the only cross-rank steps are barriers, the max-over-ranks of the timings and
rank 0 printing the JSON line.  These tests run those steps in two real
processes."""

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


def _max_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench._world()
        bench._barrier(w)
        got = bench._max_over_ranks(w, 10.0 + rank, torch.device("cpu"))
        out[rank] = got
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of this multi-threaded process
        out = m.dict()
        mp.spawn(_max_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 11.0, 1: 11.0}


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_world2():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "single_tile_N128_d64"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=280, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2 and res["value"] > 0
    assert res["e2e"]["h2d_bytes_per_step"] == 0
