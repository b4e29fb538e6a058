"""The N > 1 host logic of bench.py on two gloo ranks (CPU): the slowest rank's time is
what every rank reports, the weak-scaling value counts every rank's work, and the
reference arm under torchrun prints from rank 0 only."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    local_ms = [3.0, 5.0][rank]
    m = bench.max_over_ranks(local_ms, dist)
    out[rank] = (m, bench.weak_scaling_value(1e12, 10, world, m))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_on_gloo():
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == out[1]
    m, val = out[0]
    assert m == 5.0
    assert val == pytest.approx(1e12 * 10 * 2 / 5e-3 / 1e12)


def test_reference_arm_prints_from_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
