"""GPU parity of the sequence-split scan path against the fp64 oracle.

The sequence-split kernel cuts the sequence into segments of a power-of-two
length S that run side by side from a zero state and are joined by folding
each segment's 2x2 affine carry map ("Momentum Mamba: Enhanced State Space
Models with Momentum", "Forward Pass: Two-Stage Parallel Scan").  These tests
force that path (mm_scan_set_path) with short segments so that small inputs
cross many segments, several rounds of a cluster and ragged ends, and compare
the whole output with the oracle at the scan's tolerances.  The path runs as
two launches (segment maps passed through stream-ordered records) or, forced
with path 3 and for in-place streaming, as one fused launch (maps through
distributed shared memory); the two forms must agree bit for bit.
  * fp32 I/O: max |y - y_ref| <= 1e-4 * max |y_ref| (also hT, vT);
  * bf16 I/O: ||y - y_ref||_2 / ||y_ref||_2 <= 1e-2;
  * streaming: hT, vT bit-identical between one call and two calls split at
    a multiple of S.
"""
import numpy as np
import pytest

import oracle
import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_TOL = 1e-2


@pytest.fixture
def seg_path():
    """Force the sequence-split path (2: two launches, 3: one fused launch)
    with a given segment length; restore after."""
    def force(seg_len, path=2):
        mm.mm_scan_set_path(path, seg_len)
    yield force
    mm.mm_scan_set_path(0, 0)


def _inputs(batch, L, D, N, seed, io="f32", law=wl.SCAN_MEDIUM):
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


def _states(rng, batch, D, N, scale):
    h0 = (rng.standard_normal((batch, D, N)) * scale).astype(np.float32)
    v0 = (rng.standard_normal((batch, D, N)) * scale * 0.3).astype(np.float32)
    return h0, v0


def _run(dev, beta, alpha, h0=None, v0=None):
    th0 = None if h0 is None else torch.from_numpy(h0).cuda()
    tv0 = None if v0 is None else torch.from_numpy(v0).cuda()
    y, hT, vT = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=th0, v0=tv0,
                            beta=beta, alpha=alpha)
    torch.cuda.synchronize()
    mm.mm_device_status()
    return y.float().cpu().numpy(), hT.cpu().numpy(), vT.cpu().numpy()


def _check(io, got, inp, beta, alpha, h0=None, v0=None, what=""):
    y, hT, vT = got
    L = inp["x"].shape[2]
    N = inp["A"].shape[1]
    h0r = None if h0 is None else h0.astype(np.float64)
    v0r = None if v0 is None else v0.astype(np.float64)
    yr, hr, vr = oracle.scan_seq(**inp, h0=h0r, v0=v0r, beta=beta, alpha=alpha)
    y = y.reshape(-1, L)
    if io == "f32":
        err = np.abs(y - yr).max()
        assert err <= F32_TOL * np.abs(yr).max(), f"{what}: y max abs err {err:.3e} vs {np.abs(yr).max():.3e}"
    else:
        r = np.linalg.norm(y - yr) / np.linalg.norm(yr)
        assert r <= BF16_TOL, f"{what}: y relative L2 {r:.3e}"
    for got_s, ref_s, name in ((hT.reshape(-1, N), hr, "hT"), (vT.reshape(-1, N), vr, "vT")):
        err = np.abs(got_s - ref_s).max()
        scale = np.abs(ref_s).max()
        assert err <= F32_TOL * scale, f"{what}: {name} max abs err {err:.3e} vs {scale:.3e}"


@pytest.mark.parametrize("path", [2, 3], ids=["two-launch", "fused"])
@pytest.mark.parametrize("L,seg", [(256, 32), (1000, 64), (4096, 128), (4133 // 4 * 4, 256), (96, 128), (2000, 160)])
@pytest.mark.parametrize("beta,alpha", [(0.9, 1.0), (0.0, 1.0), (0.99, 0.5), (0.3, 2.0), (0.5, 1.0)])
def test_segments_rounds_and_ragged_ends(seg_path, L, seg, beta, alpha, path):
    # beta >= 1/2 runs the scaled form of the recurrence, smaller beta the plain one
    # up to 32 segments: rounds of an 8-CTA cluster (fused) or of a plain grid
    # (two launches), a ragged last chunk, a forced length that is not a power of
    # two (13 segments of 160 steps, the last of 80)
    seg_path(seg, path)
    inp = _inputs(2, L, 40, 16, seed=7 + L)
    _check("f32", _run(_dev(inp, "f32"), beta, alpha), inp, beta, alpha, what=f"L={L} S={seg}")


@pytest.mark.parametrize("N", [9, 12, 16])
def test_state_counts_and_initial_state(seg_path, N):
    seg_path(64)
    rng = np.random.default_rng(N)
    inp = _inputs(1, 640, 33, N, seed=100 + N)
    h0, v0 = _states(rng, 1, 33, N, 2.0)
    _check("f32", _run(_dev(inp, "f32"), 0.9, 1.0, h0, v0), inp, 0.9, 1.0, h0, v0, what=f"N={N} with h0, v0")


def test_bf16_io(seg_path):
    seg_path(128)
    inp = _inputs(2, 1024, 48, 16, seed=5, io="bf16", law=wl.SCAN_BF16)
    rng = np.random.default_rng(3)
    h0, v0 = _states(rng, 2, 48, 16, 1.0)
    _check("bf16", _run(_dev(inp, "bf16"), 0.9, 1.0, h0, v0), inp, 0.9, 1.0, h0, v0, what="bf16")


def test_slow_decay_runs_the_whole_correction(seg_path):
    # beta = 0.999 and tiny steps: the carry's response outlives every segment
    seg_path(64)
    inp = _inputs(1, 512, 16, 16, seed=11)
    inp["delta"] = (inp["delta"] * 1e-2).astype(np.float32)
    rng = np.random.default_rng(1)
    h0, v0 = _states(rng, 1, 16, 16, 1.0)
    _check("f32", _run(_dev(inp, "f32"), 0.999, 1.0, h0, v0), inp, 0.999, 1.0, h0, v0, what="slow decay")


def test_growing_modes_are_not_cut_short(seg_path):
    # A > 0 on some lanes: the response grows, so the correction must run to each segment's end
    seg_path(64)
    inp = _inputs(1, 384, 16, 16, seed=12)
    inp["A"][:, 0] = 0.5
    inp["delta"] = (inp["delta"] * 0.1).astype(np.float32)
    _check("f32", _run(_dev(inp, "f32"), 0.5, 1.0), inp, 0.5, 1.0, what="A > 0")


@pytest.mark.parametrize("seg", [64, 256, 160])
def test_streaming_split_at_segment_multiples_is_bit_identical(seg_path, seg):
    seg_path(seg)
    L, L1 = 2048, 4 * seg
    inp = _inputs(2, L, 48, 16, seed=21)
    dev = _dev(inp, "f32")
    rng = np.random.default_rng(2)
    h0, v0 = _states(rng, 2, 48, 16, 1.0)
    th0, tv0 = torch.from_numpy(h0).cuda(), torch.from_numpy(v0).cuda()
    y, hT, vT = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=th0, v0=tv0, beta=0.99)
    parts = []
    h, v = th0, tv0
    for lo, hi in ((0, L1), (L1, L)):
        sl = {k: dev[k][..., lo:hi].contiguous() for k in ("x", "delta", "B", "C")}
        yp, h, v = mm.scan_fwd(sl["x"], sl["delta"], dev["A"], sl["B"], sl["C"], h0=h, v0=v, beta=0.99)
        parts.append(yp)
    torch.cuda.synchronize()
    assert torch.equal(h, hT) and torch.equal(v, vT), "final states differ between one call and two"
    y2 = torch.cat(parts, dim=-1)
    assert torch.equal(y2, y), "y differs between one call and two calls split at a segment multiple"


def test_segmented_and_register_paths_agree(seg_path):
    inp = _inputs(1, 2048, 64, 16, seed=31)
    dev = _dev(inp, "f32")
    mm.mm_scan_set_path(1, 0)
    y1, h1, v1 = _run(dev, 0.9, 1.0)
    seg_path(256)
    y2, h2, v2 = _run(dev, 0.9, 1.0)
    scale = np.abs(y1).max()
    assert np.abs(y1 - y2).max() <= 2 * F32_TOL * scale
    assert np.abs(h1 - h2).max() <= 2 * F32_TOL * np.abs(h1).max()


def test_in_place_streaming_state(seg_path):
    # hT may be h0 and vT may be v0
    seg_path(64)
    inp = _inputs(1, 512, 32, 16, seed=41)
    dev = _dev(inp, "f32")
    rng = np.random.default_rng(4)
    h0, v0 = _states(rng, 1, 32, 16, 1.0)
    h = torch.from_numpy(h0).cuda()
    v = torch.from_numpy(v0).cuda()
    y = torch.empty_like(dev["x"])
    mm.mm_scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h, v, 0.9, 1.0, y, h, v)
    torch.cuda.synchronize()
    _check("f32", (y.cpu().numpy(), h.cpu().numpy(), v.cpu().numpy()), inp, 0.9, 1.0, h0, v0, what="in place")


def test_segment_length_query():
    # the automatic choice: the long workload's 2048 channels get 16384-step segments
    assert mm.mm_scan_segment_len(1, 131072, 2048, 16) == 16384
    assert mm.mm_scan_segment_len(1, 131072, 1024, 16) == 32768
    assert mm.mm_scan_segment_len(4, 2048, 1536, 16) == 0          # register-resident path
    assert mm.mm_scan_segment_len(1, 131072, 2048, 8) == 0          # dstate <= 8
    assert mm.mm_scan_segment_len(1, 256, 64, 16) == 0              # one segment: nothing to split
    assert mm.mm_scan_segment_len(1, 16384, 2048, 16) == 0


@pytest.mark.parametrize("L,seg,beta,io", [(4096, 128, 0.99, "f32"), (1000, 64, 0.3, "f32"),
                                           (2048, 256, 0.9, "bf16"), (8192, 64, 0.999, "f32"),
                                           (2000, 160, 0.99, "f32"), (4096, 448, 0.9, "bf16")])
def test_two_launch_and_fused_forms_are_bit_identical(seg_path, L, seg, beta, io):
    law = wl.SCAN_MEDIUM if io == "f32" else wl.SCAN_BF16
    inp = _inputs(2, L, 40, 16, seed=L + seg, io=io, law=law)
    dev = _dev(inp, io)
    rng = np.random.default_rng(L)
    h0, v0 = (torch.from_numpy(a).cuda() for a in _states(rng, 2, 40, 16, 1.0))
    out = {}
    for path in (2, 3):
        seg_path(seg, path)
        out[path] = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=h0, v0=v0, beta=beta)
        torch.cuda.synchronize()
        mm.mm_device_status()
    for a, b, name in zip(out[2], out[3], ("y", "hT", "vT")):
        assert torch.equal(a, b), f"{name} differs between the two-launch and the fused form"


def test_graph_capture_runs_the_fused_launch_and_replays(seg_path):
    # a call captured into a CUDA graph allocates nothing: it records the fused launch,
    # whose replay gives what the eager two-launch call gave
    seg_path(128)
    inp = _inputs(1, 2048, 32, 16, seed=61)
    dev = _dev(inp, "f32")
    rng = np.random.default_rng(6)
    h0, v0 = (torch.from_numpy(a).cuda() for a in _states(rng, 1, 32, 16, 1.0))
    y_ref, h_ref, v_ref = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=h0, v0=v0, beta=0.95)
    torch.cuda.synchronize()
    y, hT, vT = torch.empty_like(y_ref), torch.empty_like(h_ref), torch.empty_like(v_ref)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        mm.mm_scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0, v0, 0.95, 1.0, y, hT, vT)
    for _ in range(2):
        y.zero_()
        hT.zero_()
        g.replay()
        torch.cuda.synchronize()
        mm.mm_device_status()
        assert torch.equal(y, y_ref) and torch.equal(hT, h_ref) and torch.equal(vT, v_ref)
    del g


def test_record_memory_refused_runs_the_fused_launch(seg_path, monkeypatch):
    # the request for record memory fails (test hook): the call runs the fused launch,
    # bit-identical to it, and leaves no CUDA error behind for the next call to find
    inp = _inputs(2, 3000, 40, 16, seed=71)
    dev = _dev(inp, "f32")
    seg_path(256, 3)
    fused = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.97)
    seg_path(256, 2)
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "records")
    got = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.97)
    monkeypatch.delenv("MMSCAN_FAULT_INJECT")
    torch.cuda.synchronize()
    mm.mm_device_status()
    assert all(torch.equal(a, b) for a, b in zip(got, fused))
    again = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.97)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(again, fused))
    _check("f32", tuple(t.cpu().numpy() for t in got), inp, 0.97, 1.0, what="fallback")


def test_concurrent_calls_on_two_streams_keep_their_own_records(seg_path):
    # the two-launch form's records come from stream-ordered memory: calls on two
    # streams at once each get their own, and give what they give one at a time
    seg_path(128)
    a = _dev(_inputs(1, 4096, 48, 16, seed=81), "f32")
    b = _dev(_inputs(1, 4096, 48, 16, seed=82), "f32")
    ref_a = mm.scan_fwd(a["x"], a["delta"], a["A"], a["B"], a["C"], beta=0.97)
    ref_b = mm.scan_fwd(b["x"], b["delta"], b["A"], b["B"], b["C"], beta=0.97)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    outs = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            ga = mm.scan_fwd(a["x"], a["delta"], a["A"], a["B"], a["C"], beta=0.97, stream=s1)
        with torch.cuda.stream(s2):
            gb = mm.scan_fwd(b["x"], b["delta"], b["A"], b["B"], b["C"], beta=0.97, stream=s2)
        outs.append((ga, gb))
    torch.cuda.synchronize()
    mm.mm_device_status()
    for ga, gb in outs:
        assert all(torch.equal(p, q) for p, q in zip(ga, ref_a))
        assert all(torch.equal(p, q) for p, q in zip(gb, ref_b))
