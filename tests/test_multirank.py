"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The path shards by independent batches: every rank scans its own batch
with no collective on the data path; ranks meet only for a barrier and the
maximum of their step times.  These tests run two gloo ranks in child
processes and check the per-rank seeds, the max-over-ranks timing and the
whole-job throughput.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from selective_state_space_momentum_b200 import workloads as wl
        r, wsz, local = bench.dist_env()
        seed = bench.rank_seed(wl.SCAN_MEDIUM.seed_index, r)
        inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=1, seqlen=32, dim=8, seed=seed)
        slowest = bench.max_over_ranks(10.0 + 5.0 * r, "cpu")
        dist.barrier()
        q.put((r, wsz, local, seed, float(inp["x"].sum()), slowest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_batches_and_time_by_the_slowest():
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, w0, l0, s0, x0, m0), (r1, w1, l1, s1, x1, m1) = res
    assert (r0, r1, w0, w1, l0, l1) == (0, 1, 2, 2, 0, 1)
    assert s0 != s1 and x0 != x1          # each rank its own batch
    assert m0 == m1 == 15.0               # both ranks see the slowest rank's time


def test_whole_job_rate_counts_every_rank():
    import bench
    assert bench.whole_job_rate(1e9, 4, 2.0) == pytest.approx(4e9 / 2e-3)
    assert bench.max_over_ranks(3.5, "cpu") == 3.5      # no process group: unchanged
