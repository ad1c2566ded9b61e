"""bench.py's multi-GPU bookkeeping, run as two gloo ranks on the CPU.

With N GPUs the benchmark runs N independent replicas of the boundary (the
emulated t ranks live inside each GPU; replicas share nothing), so the only
cross-rank steps are host-side: the job time is the slowest rank's and the
throughput counts every rank's bytes.  These tests run that logic on two
processes over gloo."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}",
                            rank=rank, world_size=world)
    try:
        local = [12.5, 20.0][rank]          # rank 1 is the slow one
        mx = bench.max_over_ranks(local, "cpu")
        v = bench.job_throughput(1e9, 10, world, mx)
        # the NCCL arm's record: each collective at its slowest rank
        coll = bench.collective_record(1 << 20, [0.5, 0.75][rank], [0.9, 0.6][rank],
                                       world, "cpu")
        dist.barrier()
        q.put((rank, mx, v, coll))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in (0, 1)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, v, coll in out:
        assert mx == 20.0
        # 2 ranks x 10 steps x 1 GB in 20 ms
        assert v == pytest.approx(2 * 10 * 1e9 / 0.020 / 1e9)
        assert coll["all_reduce_ms"] == 0.75 and coll["rs_ag_ms"] == 0.9
        assert coll["rs_ag_over_all_reduce"] == pytest.approx(1.2)
        # 2 (t-1)/t of the tensor per rank: the whole tensor at t = 2
        assert coll["wire_bytes_per_rank"] == float(1 << 20)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.job_throughput(2e9, 5, 1, 10.0) == pytest.approx(1000.0)
