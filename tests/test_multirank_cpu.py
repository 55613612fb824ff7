"""World-size-2 checks (gloo, CPU) of the benchmark's multi-rank logic.

The decode path shards by sequence with no data exchange, so N GPUs run N
independent replicas: each rank gets its own seeded workload, and the only
collectives are a barrier and the max of the elapsed times, from which the
whole-job rate is computed.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method="env://")
    try:
        import bench
        w = bench.workload_for_rank("continuous_batching_b64", rank)
        ms_local = 10.0 + 5.0 * rank                   # rank 1 is the slowest
        bench.barrier()
        ms = bench.max_over_ranks(ms_local, torch.device("cpu"))
        rate = bench.whole_job_rate(w.batch * w.num_layers, world, ms)
        q.put((rank, w.seed, int(w.seq_lens(1).sum()), ms, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, seed0, tok0, ms0, rate0), (r1, seed1, tok1, ms1, rate1) = res
    assert seed0 != seed1 and tok0 != tok1          # independent replicas
    assert ms0 == ms1 == 15.0                       # both ranks report the max
    assert rate0 == rate1 == pytest.approx(2 * 64 * 16 / 0.015)


def test_single_process_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.whole_job_rate(100, 1, 1000.0) == pytest.approx(100.0)
