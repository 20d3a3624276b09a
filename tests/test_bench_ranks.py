"""bench.py's multi-rank host logic on CPU: two gloo ranks, as torch.distributed.run would
launch them, agree on the max-over-ranks time and the whole-job throughput, and the
reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ranks = bench.Ranks(world, torch.device("cpu"), sync_cuda=False)
    ranks.barrier()
    slowest = ranks.max(10.0 + rank)          # rank r took 10 + r ms
    tflops = bench.job_tflops(1e12, world, slowest)
    ranks.barrier()
    dist.destroy_process_group()
    out.put((rank, slowest, tflops))


def test_two_gloo_ranks_agree_on_max_and_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, tflops in res:
        assert slowest == 11.0                  # the max over ranks, seen by every rank
        # 2 ranks x 1e12 flops in 11 ms: the whole job's throughput, not one rank's
        assert tflops == pytest.approx(2e12 / 11e-3 / 1e12)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    r = bench.Ranks(1, None, sync_cuda=False)
    assert r.max(3.5) == 3.5
    assert bench.job_tflops(2e12, 1, 4.0) == pytest.approx(500.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "single_s256_h2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
