"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): ranks time
their own batch (weak scaling, no collective on the data path) and the job's
time is the slowest rank's."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms, kern = bench.max_over_ranks([1.0 + rank, 5.0 - rank])
    out[rank] = (ms, kern, bench.whole_job_tokens(32768, world))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2(root):
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert dict(out) == {0: (2.0, 5.0, 65536), 1: (2.0, 5.0, 65536)}


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([3.5, 1.25]) == [3.5, 1.25]
    assert bench.whole_job_tokens(32768, 1) == 32768


def test_reference_arm_under_torchrun_two_ranks(root):
    """`bench.py --impl reference` launched as the driver launches N > 1: rank
    0 alone times the oracle and prints one JSON line, the other rank exits 0
    without work."""
    import json
    import subprocess
    import sys
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "3", "--workload", "tiny_l256"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["config"]["workload"] == "tiny_l256"
    # rank 0 gives the oracle every core even though the launcher pins one thread
    assert line["cpu_baseline"]["cores"] == len(os.sched_getaffinity(0))
