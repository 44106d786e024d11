"""Host logic of the scan split across ranks, on CPU.

The split cuts one sequence into pieces, one per rank, every piece but the
last a whole number of segments (split_pieces); each rank writes its
segments' map records, the ranks all-gather them in rank order, and each
rank's second launch reads the records of the whole sequence.  These tests
check the piece arithmetic, and -- in two gloo ranks with the two launches
replaced by stand-ins that write and read marked bytes -- that the wrapper
scan_fwd_split passes each rank its own place in the sequence and hands the
second launch every rank's records in rank order.  The launches themselves
are covered on the GPU (test_scan_split_gpu.py).
"""
import os
import socket

import pytest

import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import build as mmbuild

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("total,world,S,expect", [
    (1024, 2, 64, [(0, 512), (512, 512)]),
    (1000, 3, 64, [(0, 384), (384, 384), (768, 232)]),
    (1600, 2, 128, [(0, 896), (896, 704)]),
    (100, 1, 32, [(0, 100)]),
    (131072, 8, 2048, [(r * 16384, 16384) for r in range(8)]),
])
def test_split_pieces(total, world, S, expect):
    pieces = mm.split_pieces(total, world, S)
    assert pieces == expect
    assert sum(n for _, n in pieces) == total
    for f, n in pieces[:-1]:
        assert f % S == 0 and n % S == 0            # inner pieces: whole segments at segment boundaries
    assert pieces[-1][0] % S == 0


def test_split_pieces_refuses_an_empty_rank():
    with pytest.raises(ValueError, match="without a piece"):
        mm.split_pieces(128, 3, 64)                # two segments, three ranks
    with pytest.raises(ValueError):
        mm.split_pieces(0, 1, 64)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        seen = {}

        def fake_maps(x, delta, A, B, C, beta, alpha, y, maps, seg_len, stream=None):
            # mark each record with (rank, segment within the piece)
            rec = mm.mm_scan_split_maps_size(x.shape[0], x.shape[2], x.shape[1], A.shape[1], 1)
            for k in range(maps.numel() // rec):
                maps[k * rec:(k + 1) * rec] = 16 * rank + k
            seen["maps_bytes"] = maps.numel()

        def fake_correct(delta, A, C, h0, v0, beta, alpha, y, hT, vT, maps_all, seg_len, seq_first,
                         seqlen_total, stream=None):
            seen.update(first=seq_first, total=seqlen_total, seg=seg_len,
                        gathered=maps_all.reshape(-1)[::mm.mm_scan_split_maps_size(1, 32, 8, 16, 1)].tolist())

        mm.mm_scan_fwd_split_maps = fake_maps
        mm.mm_scan_fwd_split_correct = fake_correct
        total, S = 1000, 64
        first, n = mm.split_pieces(total, world, S)[rank]
        x = torch.zeros((1, 8, n))
        A = torch.zeros((8, 16))
        B = torch.zeros((1, 16, n))
        mm.scan_fwd_split(x, x, A, B, B, S, total)
        dist.barrier()
        q.put((rank, first, n, seen))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_records_in_rank_order():
    mmbuild.build()                                # the record size comes from the library
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    rec = mm.mm_scan_split_maps_size(1, 32, 8, 16, 1)
    per = 8                                          # 16 segments of 64 steps over two ranks
    for rank, first, n, seen in res:
        assert (first, n) == mm.split_pieces(1000, world, 64)[rank]
        assert seen["first"] == first and seen["total"] == 1000 and seen["seg"] == 64
        assert seen["maps_bytes"] == per * rec         # every rank sends the same count: the last one pads
        # rank 0's eight records, then rank 1's (its last piece fills all eight: 488 steps -> 8 segments)
        assert seen["gathered"] == [k for k in range(8)] + [16 + k for k in range(8)]
