"""The multi-GPU path of bench.py is replicas only; its cross-rank logic runs here on CPU ranks (gloo, world 2)."""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world)  # rank 1 is the slow one
    dist.barrier()
    value = bench.job_throughput(1024, world, 20, slowest)
    results[rank] = (slowest, value)
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_world2():
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    mp.start_processes(_worker, args=(2, port, results), nprocs=2, join=True, start_method="spawn")
    assert results[0] == results[1]
    slowest, value = results[0]
    assert slowest == 15.0
    assert value == pytest.approx(2 * 1024 * 20 / 0.015)


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1024, 1, 10, 20.0) == pytest.approx(1024 * 10 / 0.02)


def test_reference_arm_prints_on_rank0_only():
    """Under torchrun only rank 0 times the CPU oracle; the other ranks exit 0 without output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3", "--workload", "dsa-tiny-N4096-L256"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "dsa-tiny-N4096-L256"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_bench_starts_its_own_ranks():
    """`bench.py --gpus 2` without a torch.distributed environment starts two ranks itself (torch.distributed.run
    on 127.0.0.1); the dry run exercises that launch and the cross-rank max on CPU ranks."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                           "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "5",
                          "--warmup", "3", "--dry-run"], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(ln) for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    line = lines[0]
    assert line["dry_run"] and line["n_gpus"] == 2 and line["steps"] == 5
    assert line["ms_per_step"] >= 2.0 * 0.9  # the slower rank (2 ms per step) sets the time
