"""The multi-process (N > 1) bookkeeping of bench.py, on CPU with gloo and two ranks.

On GPUs each rank runs the same fixed work on its own GPU (replicas: the path has no
exchange step), so what N > 1 adds is host logic: the process group, the barriers, the
slowest rank's time, the whole-job rate, and a reference arm that only rank 0 runs.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup()
    try:
        assert (w, r, local) == (world, rank, rank)
        assert dist.get_backend() == "gloo"
        bench.barrier(w)
        slowest = bench.max_over_ranks(1.0 + rank, w)            # rank r took 1 + r seconds
        rate, t_max = bench.job_rate(10.0, 1.0 + rank, w)        # 10 units per rank
        bench.barrier(w)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "rate": rate, "t_max": t_max}, f)
    finally:
        dist.destroy_process_group()


def test_replica_bookkeeping_two_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    for r in range(world):
        got = json.loads((tmp_path / f"rank{r}.json").read_text())
        assert got["slowest"] == 2.0                  # the max over ranks, seen by every rank
        assert got["t_max"] == 2.0
        assert got["rate"] == pytest.approx(10.0 * world / 2.0)


def test_reference_arm_under_torchrun_prints_once():
    # two ranks on the host: rank 0 times the oracle and prints one line, rank 1 exits 0
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
