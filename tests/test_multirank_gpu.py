"""Batch-sharded ranks running the product kernels, checked shard by shard.

The multi-GPU form of the path shards by independent batches: every rank
scans its own batch with no collective on the data path and the ranks meet
only for a barrier and the maximum of their step times (bench.py).  Here two
ranks run as processes on the one GPU this pool gives (their kernels are
independent: nothing waits on the other rank), with a gloo group standing in
for NCCL for the host-side collective.  Each rank draws its shard from its
own seed exactly as bench.py does, runs the scan through the C ABI -- the
register-resident path, and the sequence-split path with its clusters --
and compares its whole output with the fp64 oracle; the ranks then agree on
the slowest rank's device time.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

F32_TOL = 1e-4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import bench
        import oracle
        import selective_state_space_momentum_b200 as mm
        from selective_state_space_momentum_b200 import workloads as wl
        torch.cuda.set_device(0)
        r, wsz, _ = bench.dist_env()
        seed = bench.rank_seed(wl.SCAN_MEDIUM.seed_index, r)
        out = {"rank": r, "world": wsz, "seed": seed}
        for path, seg in ((1, 0), (2, 256)):
            inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=2, seqlen=1536, dim=48, seed=seed)
            dev = {k: torch.from_numpy(v).cuda().contiguous() for k, v in inp.items()}
            mm.mm_scan_set_path(path, seg)
            try:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                y, hT, vT = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.9, alpha=1.0)
                e1.record()
                torch.cuda.synchronize()
                mm.mm_device_status()
            finally:
                mm.mm_scan_set_path(0, 0)
            yr, hr, vr = oracle.scan_seq(**inp, beta=0.9, alpha=1.0)
            L, N = inp["x"].shape[2], inp["A"].shape[1]
            yg = y.cpu().numpy().reshape(-1, L)
            out[f"y_err_{path}"] = float(np.abs(yg - yr).max() / np.abs(yr).max())
            out[f"h_err_{path}"] = float(np.abs(hT.cpu().numpy().reshape(-1, N) - hr).max() / np.abs(hr).max())
            out[f"sum_{path}"] = float(yg.sum())
            ms = e0.elapsed_time(e1)
            out[f"ms_{path}"] = ms
            out[f"slowest_{path}"] = bench.max_over_ranks(ms, "cpu")
        dist.barrier()
        q.put(out)
    finally:
        dist.destroy_process_group()


def test_two_ranks_scan_their_own_shards_and_agree_on_the_slowest():
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
    res = sorted((q.get(timeout=10) for _ in range(2)), key=lambda d: d["rank"])
    assert [d["rank"] for d in res] == [0, 1] and all(d["world"] == 2 for d in res)
    assert res[0]["seed"] != res[1]["seed"]
    for path in (1, 2):
        assert res[0][f"sum_{path}"] != res[1][f"sum_{path}"], "the ranks scanned the same batch"
        for d in res:
            assert d[f"y_err_{path}"] <= F32_TOL, f"rank {d['rank']} path {path}: y error {d[f'y_err_{path}']:.3e}"
            assert d[f"h_err_{path}"] <= F32_TOL, f"rank {d['rank']} path {path}: hT error {d[f'h_err_{path}']:.3e}"
        slowest = max(d[f"ms_{path}"] for d in res)
        assert all(d[f"slowest_{path}"] == pytest.approx(slowest) for d in res)
