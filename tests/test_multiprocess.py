"""The multi-process (N > 1) paths of bench.py on CPU, two ranks over gloo: every rank
runs an independent replica, the slowest rank's time is the job's, and rank 0 alone prints
the JSON line; no GPU."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench
        out[rank] = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_max_worker, args=(2, port, out), nprocs=2, start_method="spawn")
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.25, torch.device("cpu")) == 0.25


@pytest.mark.timeout(600)
def test_reference_arm_two_ranks_under_torchrun():
    """The driver's launch of the reference arm at N = 2: rank 0 prints one JSON line,
    rank 1 exits cleanly, over the gloo process group."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny",
           "--ref-budget", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=580,
                       env={**os.environ, "OMP_NUM_THREADS": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
