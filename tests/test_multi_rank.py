"""The bench's multi-rank logic on CPU: two gloo ranks (no GPU, no NCCL).

bench.py --gpus N runs N independent replicas (no data-path collective); what
crosses ranks is the barrier around the timed region, the max-over-ranks time
and the sum of the bytes all ranks moved.  The reference arm prints from rank 0
only; the other ranks exit 0 without work."""
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


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank), "W1_BENCH_BACKEND": "gloo"})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    bench.barrier(w)
    res = {
        "world": w, "rank": r,
        "max": bench.max_over_ranks(w, 1.5 * (r + 1)),        # per-rank times 1.5, 3.0
        "sum": bench.sum_over_ranks(w, 1000.0 * (r + 1)),     # per-rank bytes 1000, 2000
    }
    bench.barrier(w)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks_reduce_time_and_bytes(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    for r, g in enumerate(got):
        assert g["world"] == world and g["rank"] == r
        assert g["max"] == 3.0          # max over ranks, identical everywhere
        assert g["sum"] == 3000.0       # total bytes of all ranks


def test_reference_arm_under_torchrun_prints_once(tmp_path):
    """torchrun --nproc-per-node 2: rank 0 prints one JSON line, rank 1 exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, W1_BENCH_BACKEND="gloo", OMP_NUM_THREADS="2")
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
