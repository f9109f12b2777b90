"""The N > 1 host logic of bench.py on two gloo ranks (CPU, no GPU):
rank discovery from the torchrun environment, the max-over-ranks time,
the whole-job throughput of independent replicas, and the reference arm
running on rank 0 only."""
import os
import socket
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


def _worker(rank, world, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                          MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import bench
        from datetime import timedelta
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=timedelta(seconds=60))
        ws, r, local = bench.dist_env()
        assert (ws, r, local) == (world, rank, rank)
        my_ms = 10.0 + 5.0 * rank
        worst = bench.max_over_ranks(my_ms, "cpu")
        bench.barrier()
        value = bench.whole_job_tflops(1e12, 4, ws, worst)

        class A:
            workload, steps, warmup = "tiny", 3, 3
        ref = bench.run_reference(A(), ws, r) if r != 0 else "rank0"
        dist.destroy_process_group()
        q.put((rank, worst, value, ref))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e), None))


def test_two_rank_host_logic():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, worst, value, ref = q.get(timeout=120)
        results[rank] = (worst, value, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (worst, value, ref) in results.items():
        assert worst != "error", value
        assert worst == 15.0                       # the slowest rank's time
        assert value == pytest.approx(1e12 * 4 * 2 / 15e-3 / 1e12)
    assert results[1][2] is None                   # reference arm: rank 0 only
