"""The N > 1 host logic of bench.py on two gloo ranks (CPU): every rank times
its own device work, the reported time is the maximum over ranks, the value
is all ranks' bytes over that time, and only rank 0 reports."""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        own_ms = 100.0 + 50.0 * rank
        ms = bench.max_over_ranks(own_ms, world, dist, "cpu")
        q.put((rank, ms, bench.throughput_gbs(world, 8.0e9, 3, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive and all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 150.0                       # the slower rank's time on every rank
        assert value == pytest.approx(2 * 8.0e9 * 3 / 0.150 / 1e9)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_grouping_roofline_arithmetic():
    import bench
    # LLaMA-3.1-8B-shaped 64K key cache: 2^32 bf16 keys; 4 power iterations = 10 passes
    n = 32 * 8 * 65536 * 128
    r = bench.grouping_roofline(43.8, n, 2, 4, 148)
    assert r["peak"] == 74.4                       # 148 x 128 x 2 x 1.965 GHz
    flops = 10 * 2 * 16 * n
    assert abs(r["achieved"] - flops / 43.8e-3 / 1e12) < 0.01
    assert r["key_gb_read"] == round(10 * n * 2 / 1e9, 2)
    assert r["bound"] == "alu" and 0 < r["frac"] < 1
