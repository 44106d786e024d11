"""GPU parity of the scan split across ranks, through the C ABI.

"Forward Pass: Two-Stage Parallel Scan" of "Momentum Mamba: Enhanced State
Space Models with Momentum" joins chunks of the sequence by their 2x2
affine carry maps.  The split form carries that join across devices: each
rank scans its piece of the sequence from a zero state and writes one map
record per segment (mm_scan_fwd_split_maps), the ranks exchange the records,
and each rank folds the records of every earlier segment into its piece's
carry-ins and adds their response to y (mm_scan_fwd_split_correct).

Here the ranks are emulated on the one GPU, one after another (nothing in
the split waits on another rank inside a kernel): every piece's first
launch, the records concatenated in rank order (what the all-gather
delivers), then every piece's second launch.  The result must equal, bit
for bit, one mm_scan_fwd over the whole sequence on the sequence-split path
with the same segment length, and match the fp64 oracle at the scan's
tolerances:
  * fp32 I/O: max |y - y_ref| <= 1e-4 * max |y_ref| (also hT, vT);
  * bf16 I/O: ||y - y_ref||_2 / ||y_ref||_2 <= 1e-2, states at fp32 bound.
The exchange can also be folded into the first launch
(mm_scan_fwd_split_maps_peers): each piece's records are stored straight
into every rank's buffer of the whole sequence's records.  That form is
emulated the same way, each emulated rank with a buffer of its own.  The
last tests run the wrappers scan_fwd_split (records gathered through host
memory) and scan_fwd_split_peers (records stored into the other process's
buffer through CUDA IPC) in two processes on this GPU joined by a gloo group,
each on its own piece.
"""
import os
import socket

import numpy as np
import pytest

import oracle
import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_TOL = 1e-2


def _inputs(batch, L, D, N, seed, io="f32"):
    law = wl.SCAN_MEDIUM if io == "f32" else wl.SCAN_BF16
    inp = wl.scan_inputs(law, batch=batch, seqlen=L, dim=D, dstate=N, seed=seed)
    if io == "bf16":
        for k in ("x", "delta", "B", "C"):
            inp[k] = wl.bf16_round(inp[k])
    return inp


def _dev(inp, io):
    dt = torch.float32 if io == "f32" else torch.bfloat16
    out = {k: torch.from_numpy(inp[k]).cuda().to(dt).contiguous() for k in ("x", "delta", "B", "C")}
    out["A"] = torch.from_numpy(inp["A"]).cuda().contiguous()
    return out


def _states(batch, D, N, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    h0 = (rng.standard_normal((batch, D, N)) * scale).astype(np.float32)
    v0 = (rng.standard_normal((batch, D, N)) * scale * 0.3).astype(np.float32)
    return h0, v0


def _emulate(dev, h0, v0, beta, alpha, S, world):
    """The split over `world` ranks, run rank after rank on this GPU."""
    batch, dim, L = dev["x"].shape
    N = dev["A"].shape[1]
    io = mm.MM_F32 if dev["x"].dtype == torch.float32 else mm.MM_BF16
    pieces = mm.split_pieces(L, world, S)
    per = pieces[0][1] // S if world > 1 else -(-L // S)
    rec = mm.mm_scan_split_maps_size(batch, L, dim, N, 1, io)
    sl = [{k: dev[k][..., f:f + n].contiguous() for k in ("x", "delta", "B", "C")} for f, n in pieces]
    ys, bufs = [], []
    for p in sl:
        local = torch.empty(per * rec, dtype=torch.uint8, device="cuda")
        y = torch.empty_like(p["x"])
        mm.mm_scan_fwd_split_maps(p["x"], p["delta"], dev["A"], p["B"], p["C"], beta, alpha, y, local, S)
        ys.append(y)
        bufs.append(local)
    gathered = torch.cat(bufs)          # the all-gather, in rank order
    states = []
    for (first, _), p, y in zip(pieces, sl, ys):
        hT = torch.empty((batch, dim, N), device="cuda")
        vT = torch.empty_like(hT)
        mm.mm_scan_fwd_split_correct(p["delta"], dev["A"], p["C"], h0, v0, beta, alpha, y, hT, vT, gathered, S,
                                     first, L)
        states.append((hT, vT))
    torch.cuda.synchronize()
    mm.mm_device_status()
    return torch.cat(ys, dim=-1), states


def _one_call(dev, h0, v0, beta, alpha, S):
    mm.mm_scan_set_path(2, S)
    try:
        y, hT, vT = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=h0, v0=v0,
                                beta=beta, alpha=alpha)
        torch.cuda.synchronize()
        mm.mm_device_status()
    finally:
        mm.mm_scan_set_path(0, 0)
    return y, hT, vT


def _check_oracle(io, inp, y, hT, vT, h0, v0, beta, alpha, what):
    L, N = inp["x"].shape[2], inp["A"].shape[1]
    h0r = None if h0 is None else h0.cpu().numpy().astype(np.float64)
    v0r = None if v0 is None else v0.cpu().numpy().astype(np.float64)
    yr, hr, vr = oracle.scan_seq(**inp, h0=h0r, v0=v0r, beta=beta, alpha=alpha)
    yg = y.float().cpu().numpy().reshape(-1, L)
    if io == "f32":
        assert np.abs(yg - yr).max() <= F32_TOL * np.abs(yr).max(), f"{what}: y"
    else:
        assert np.linalg.norm(yg - yr) <= BF16_TOL * np.linalg.norm(yr), f"{what}: y"
    for name, got, ref in (("hT", hT, hr), ("vT", vT, vr)):
        g = got.cpu().numpy().reshape(-1, N)
        assert np.abs(g - ref).max() <= F32_TOL * np.abs(ref).max(), f"{what}: {name}"


CASES = [
    # L, S, world, beta, alpha, io
    (1024, 64, 2, 0.9, 1.0, "f32"),
    (1000, 64, 3, 0.99, 0.5, "f32"),     # ragged last piece and last segment
    (4096, 32, 2, 0.3, 2.0, "f32"),      # 64 segments a piece: eight rounds of a cluster; the plain form
    (2048, 128, 4, 0.9, 1.0, "bf16"),
    (1024, 64, 1, 0.5, 1.0, "f32"),      # one rank: the two launches alone
    (640, 64, 5, 0.0, 1.0, "f32"),       # beta = 0: no velocity carried
    (768, 256, 3, 0.999, 1.0, "f32"),    # one segment a piece
]


@pytest.mark.parametrize("L,S,world,beta,alpha,io", CASES)
def test_split_equals_one_call_bit_for_bit(L, S, world, beta, alpha, io):
    batch, D, N = 2, 40, 16
    inp = _inputs(batch, L, D, N, seed=L + world, io=io)
    dev = _dev(inp, io)
    h0, v0 = (torch.from_numpy(a).cuda() for a in _states(batch, D, N, seed=world))
    y, states = _emulate(dev, h0, v0, beta, alpha, S, world)
    y1, h1, v1 = _one_call(dev, h0, v0, beta, alpha, S)
    assert torch.equal(y, y1), "y of the split differs from one call"
    for r, (hT, vT) in enumerate(states):
        assert torch.equal(hT, h1) and torch.equal(vT, v1), f"rank {r}: final states differ from one call"
    _check_oracle(io, inp, y, states[0][0], states[0][1], h0, v0, beta, alpha, f"L={L} S={S} world={world}")


def test_split_negative_delta_and_growing_modes():
    # delta < 0 somewhere and A > 0 on a lane: every correction runs to its segment's end
    batch, D, N, L, S = 1, 24, 12, 768, 64
    inp = _inputs(batch, L, D, N, seed=5)
    inp["delta"][0, 3, 100:110] *= -1.0
    inp["A"][:, 0] = 0.2
    inp["delta"] = (inp["delta"] * 0.1).astype(np.float32)
    dev = _dev(inp, "f32")
    y, states = _emulate(dev, None, None, 0.8, 1.0, S, 3)
    y1, h1, v1 = _one_call(dev, None, None, 0.8, 1.0, S)
    assert torch.equal(y, y1)
    assert all(torch.equal(h, h1) and torch.equal(v, v1) for h, v in states)
    _check_oracle("f32", inp, y, states[0][0], states[0][1], None, None, 0.8, 1.0, "negative delta, A > 0")


def test_split_records_are_what_the_first_launch_wrote():
    # the record layout: a piece's records are the same bytes whichever rank's buffer they sit in
    batch, D, N, L, S = 1, 32, 16, 512, 64
    inp = _inputs(batch, L, D, N, seed=9)
    dev = _dev(inp, "f32")
    rec = mm.mm_scan_split_maps_size(batch, L, D, N, 1)
    whole = torch.empty(8 * rec, dtype=torch.uint8, device="cuda")
    y = torch.empty_like(dev["x"])
    mm.mm_scan_fwd_split_maps(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], 0.9, 1.0, y, whole, S)
    half = torch.empty(4 * rec, dtype=torch.uint8, device="cuda")
    p = {k: dev[k][..., 256:].contiguous() for k in ("x", "delta", "B", "C")}
    y2 = torch.empty_like(p["x"])
    mm.mm_scan_fwd_split_maps(p["x"], p["delta"], dev["A"], p["B"], p["C"], 0.9, 1.0, y2, half, S)
    torch.cuda.synchronize()
    mm.mm_device_status()
    assert torch.equal(whole[4 * rec:], half)
    assert torch.equal(y[..., 256:], y2)           # the zero-start read-out of the same segments


def _emulate_peers(dev, h0, v0, beta, alpha, S, world):
    """The split with the exchange in the first launch: every emulated rank
    stores its records into every rank's own buffer, then corrects from its
    own buffer."""
    batch, dim, L = dev["x"].shape
    N = dev["A"].shape[1]
    io = mm.MM_F32 if dev["x"].dtype == torch.float32 else mm.MM_BF16
    pieces = mm.split_pieces(L, world, S)
    nbytes = mm.mm_scan_split_maps_size(batch, L, dim, N, -(-L // S), io)
    bufs = [torch.full((nbytes,), 0xff, dtype=torch.uint8, device="cuda") for _ in range(world)]
    dests = torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device="cuda")
    sl = [{k: dev[k][..., f:f + n].contiguous() for k in ("x", "delta", "B", "C")} for f, n in pieces]
    ys = []
    for (first, _), p in zip(pieces, sl):
        y = torch.empty_like(p["x"])
        mm.mm_scan_fwd_split_maps_peers(p["x"], p["delta"], dev["A"], p["B"], p["C"], beta, alpha, y, dests, S,
                                        first, L)
        ys.append(y)
    torch.cuda.synchronize()
    for b in bufs[1:]:
        assert torch.equal(b, bufs[0]), "the ranks' record buffers differ"
    states = []
    for r, ((first, _), p, y) in enumerate(zip(pieces, sl, ys)):
        hT = torch.empty((batch, dim, N), device="cuda")
        vT = torch.empty_like(hT)
        mm.mm_scan_fwd_split_correct(p["delta"], dev["A"], p["C"], h0, v0, beta, alpha, y, hT, vT, bufs[r], S,
                                     first, L)
        states.append((hT, vT))
    torch.cuda.synchronize()
    mm.mm_device_status()
    return torch.cat(ys, dim=-1), states


@pytest.mark.parametrize("L,S,world,io", [(1024, 64, 2, "f32"), (1000, 64, 3, "f32"), (2048, 128, 4, "bf16"),
                                          (768, 256, 1, "f32")])
def test_records_stored_into_every_rank_buffer(L, S, world, io):
    inp = _inputs(2, L, 40, 16, seed=L * 3 + world, io=io)
    dev = _dev(inp, io)
    h0, v0 = (torch.from_numpy(a).cuda() for a in _states(2, 40, 16, seed=world + 10))
    y, states = _emulate_peers(dev, h0, v0, 0.95, 1.0, S, world)
    y1, h1, v1 = _one_call(dev, h0, v0, 0.95, 1.0, S)
    assert torch.equal(y, y1), "y of the peer-exchange split differs from one call"
    for hT, vT in states:
        assert torch.equal(hT, h1) and torch.equal(vT, v1)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, exchange="gather"):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        L, S = 1600, 128
        inp = _inputs(2, L, 48, 16, seed=77)      # every rank draws the whole sequence, keeps its piece
        dev = _dev(inp, "f32")
        h0, v0 = (torch.from_numpy(a).cuda() for a in _states(2, 48, 16, seed=78))
        first, n = mm.split_pieces(L, world, S)[rank]
        p = {k: dev[k][..., first:first + n].contiguous() for k in ("x", "delta", "B", "C")}
        if exchange == "peers":
            peers = mm.SplitPeers(2, 48, 16, L, S)
            runs = [mm.scan_fwd_split_peers(p["x"], p["delta"], dev["A"], p["B"], p["C"], S, L, peers, h0=h0,
                                            v0=v0, beta=0.95, alpha=1.0) for _ in range(3)]   # both buffer sets
            torch.cuda.synchronize()
            dist.barrier()            # the other rank has read its records before the mapping goes
            peers.close()
            y, hT, vT = runs[-1]
            assert all(torch.equal(a, b) for r in runs[:-1] for a, b in zip(r, runs[-1]))
        else:
            y, hT, vT = mm.scan_fwd_split(p["x"], p["delta"], dev["A"], p["B"], p["C"], S, L, h0=h0, v0=v0,
                                          beta=0.95, alpha=1.0)
        torch.cuda.synchronize()
        mm.mm_device_status()
        y1, h1, v1 = _one_call(dev, h0, v0, 0.95, 1.0, S)
        yr, hr, _ = oracle.scan_seq(**inp, h0=h0.cpu().numpy().astype(np.float64),
                                    v0=v0.cpu().numpy().astype(np.float64), beta=0.95, alpha=1.0)
        yp = y.cpu().numpy().reshape(-1, n)
        out = {"rank": rank, "piece": (first, n),
               "same_y": bool(torch.equal(y, y1[..., first:first + n])),
               "same_states": bool(torch.equal(hT, h1) and torch.equal(vT, v1)),
               "y_err": float(np.abs(yp - yr[:, first:first + n]).max() / np.abs(yr).max()),
               "h_err": float(np.abs(hT.cpu().numpy().reshape(-1, 16) - hr).max() / np.abs(hr).max())}
        dist.barrier()
        q.put(out)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("exchange", ["gather", "peers"])
def test_two_gloo_ranks_split_one_sequence(exchange):
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, exchange)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
    res = sorted((q.get(timeout=10) for _ in range(2)), key=lambda d: d["rank"])
    assert [d["piece"] for d in res] == [(0, 896), (896, 704)]
    for d in res:
        assert d["same_y"] and d["same_states"], d
        assert d["y_err"] <= F32_TOL and d["h_err"] <= F32_TOL, d


def test_long_workload_over_eight_emulated_ranks():
    # the long streaming workload (B1 L131072 D2048 N16, beta 0.99) cut over eight ranks
    # with 2048-step segments, as bench.py --split-l at eight GPUs cuts it: bit-identical
    # to one call with the same segments, and a channel sample within the oracle's tolerance
    w = wl.SCAN_LONG
    inp = wl.scan_inputs(w, seed=wl.seed_of(w.seed_index))
    dev = {k: torch.from_numpy(inp[k]).cuda().contiguous() for k in ("x", "delta", "B", "C", "A")}
    y, states = _emulate(dev, None, None, 0.99, 1.0, 2048, 8)
    y1, h1, v1 = _one_call(dev, None, None, 0.99, 1.0, 2048)
    assert torch.equal(y, y1), "y of the eight-rank split differs from one call"
    assert all(torch.equal(h, h1) and torch.equal(v, v1) for h, v in states)
    rng = np.random.default_rng(8)
    chan = np.sort(rng.choice(w.dim, 24, replace=False))
    yr, hr, vr = oracle.scan_seq(**inp, beta=0.99, alpha=1.0, chan=chan)
    yg = y.cpu().numpy().reshape(-1, w.seqlen)[chan]
    assert np.abs(yg - yr).max() <= F32_TOL * np.abs(yr).max()
    hg = states[0][0].cpu().numpy().reshape(-1, w.dstate)[chan]
    assert np.abs(hg - hr).max() <= F32_TOL * np.abs(hr).max()
