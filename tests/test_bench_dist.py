"""bench.py's multi-rank plumbing on CPU (world_size 2 over gloo): the step
time every rank reports is the maximum over the ranks, and the reference arm
under torchrun prints exactly one JSON line, from rank 0."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench
        got = bench.max_over_ranks(1.5 + 2.0 * rank, world)    # rank 1 is the slower one
        bench.barrier(world)
        np.save(f"{path}.{rank}.npy", np.array([got]))
    finally:
        dist.destroy_process_group()


def test_step_time_is_the_max_over_ranks(tmp_path):
    world, port = 2, _free_port()
    path = str(tmp_path / "t")
    mp.start_processes(_worker, args=(world, port, path), nprocs=world, start_method="spawn")
    for r in range(world):
        assert float(np.load(f"{path}.{r}.npy")[0]) == 3.5


def test_reference_arm_under_torchrun_prints_one_line():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
