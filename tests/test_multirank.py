"""The N > 1 path of bench.py on CPU: world-size-2 process groups (gloo, 127.0.0.1).

bench.py runs N independent replicas (one per GPU, no data-path collective): its only cross-rank steps are the
barrier and the max over ranks of every device time, and the whole-job value is all ranks' bytes over the
slowest rank's time.  The reference arm runs on rank 0 alone; the other ranks exit 0 without work.
"""
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


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    slowest = bench.max_over_ranks(1.5 + rank, world, "cpu")  # rank r "took" 1.5 + r ms
    dist.barrier()
    value = bench.replica_throughput(step_bytes=1e6, steps=10, elapsed_ms_max=slowest, world=world)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"slowest": slowest, "value": value}, f)
    dist.destroy_process_group()


def test_max_over_ranks_and_replica_throughput_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["slowest"] == pytest.approx(2.5)  # every rank sees the slowest rank's time
        # 2 replicas x 1 MB per step over 0.25 ms per step (10 steps in 2.5 ms)
        assert g["value"] == pytest.approx(2 * 1e6 / 0.25e-3 / 1e9)


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-rows", "16"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env={**os.environ, "OMP_NUM_THREADS": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0
