"""The benchmark's own N > 1 plumbing on the CPU (gloo, world size 2): its
max-over-ranks reduction and barrier, and its reference arm launched under
torchrun the way `bench.py --gpus N` is launched (rank 0 alone runs the oracle
and prints the line, the other ranks exit 0 without work).  The GPU arm's
per-rank kernels need a GPU each and are not run here."""
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
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    bench.init_pg("gloo", w)
    try:
        # each rank's "device time"; the benchmark reports the slowest rank
        got = bench.max_over_ranks(1.5 + 2.0 * rank, w)
        bench.barrier(w)
        np.save(os.path.join(result_dir, f"max{rank}.npy"), np.array([got]))
    finally:
        dist.destroy_process_group()


def test_bench_max_over_ranks_and_barrier_gloo(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    for rank in range(world):
        assert float(np.load(tmp_path / f"max{rank}.npy")[0]) == 3.5


def test_bench_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3", "--workload", "gdn_tiny_fp32"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout  # rank 0 alone prints
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["config"]["workload"] == "gdn_tiny_fp32"
    assert rec["value"] > 0 and rec["unit"] == "tokens/s"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
