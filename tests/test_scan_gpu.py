"""GPU parity of mm_scan_fwd against the fp64 oracle (through the C ABI).

Tolerances are those the task fixes for the scan:
  * fp32 I/O: max |y - y_ref| <= 1e-4 * max |y_ref| (the same test is
    applied to hT and vT against their own scale);
  * bf16 I/O with fp32 state: ||y - y_ref||_2 / ||y_ref||_2 <= 1e-2;
  * streaming: hT, vT bit-identical between one call and two calls.
Small sizes are compared element by element over the whole output;
full-size workloads are compared on a seeded sample of channels, each of
which the oracle computes on its own.
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


def _dev(inp, io):
    dt = torch.float32 if io == "f32" else torch.bfloat16
    out = {}
    for k in ("x", "delta", "B", "C"):
        out[k] = torch.from_numpy(inp[k]).to("cuda").to(dt).contiguous()
    out["A"] = torch.from_numpy(inp["A"]).to("cuda").contiguous()
    return out


def _run(dev, beta, alpha, h0=None, v0=None):
    y, hT, vT = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=h0, v0=v0,
                            beta=beta, alpha=alpha)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), hT.cpu().numpy(), vT.cpu().numpy()


def _max_abs_ok(got, ref, what):
    err = float(np.abs(got - ref).max())
    scale = float(np.abs(ref).max())
    assert err <= F32_TOL * scale, f"{what}: max abs err {err:.3e} > {F32_TOL} * {scale:.3e}"
    return err / scale if scale else 0.0


def _rel_l2_ok(got, ref, what):
    r = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert r <= BF16_TOL, f"{what}: relative L2 {r:.3e} > {BF16_TOL}"
    return r


def _compare(io, got, ref, what):
    y, hT, vT = got
    yr, hr, vr = ref
    if io == "f32":
        _max_abs_ok(y, yr, what + " y")
    else:
        _rel_l2_ok(y, yr, what + " y")
    _max_abs_ok(hT, hr, what + " hT")
    _max_abs_ok(vT, vr, what + " vT")


def _full_compare(inp, io, beta, alpha, h0=None, v0=None, what=""):
    dev = _dev(inp, io)
    th0 = None if h0 is None else torch.from_numpy(h0.astype(np.float32)).cuda()
    tv0 = None if v0 is None else torch.from_numpy(v0.astype(np.float32)).cuda()
    y, hT, vT = _run(dev, beta, alpha, th0, tv0)
    Bsz, D, L = inp["x"].shape
    N = inp["A"].shape[1]
    h0r = None if h0 is None else h0.astype(np.float32).astype(np.float64)
    v0r = None if v0 is None else v0.astype(np.float32).astype(np.float64)
    yr, hr, vr = oracle.scan_seq(**inp, h0=h0r, v0=v0r, beta=beta, alpha=alpha)
    _compare(io, (y.reshape(-1, L), hT.reshape(-1, N), vT.reshape(-1, N)), (yr, hr, vr), what)
    return y, hT, vT


def _sample_channels(nch, k, seed=0):
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(nch, size=min(k, nch), replace=False).tolist())
    pick.update({0, nch - 1})
    return np.array(sorted(pick), dtype=np.int64)


def _sampled_compare(inp, io, beta, alpha, dev=None, got=None, k=48, what=""):
    if got is None:
        got = _run(dev or _dev(inp, io), beta, alpha)
    y, hT, vT = got
    Bsz, D, L = inp["x"].shape
    N = inp["A"].shape[1]
    chan = _sample_channels(Bsz * D, k)
    yr, hr, vr = oracle.scan_seq(**inp, beta=beta, alpha=alpha, chan=chan)
    _compare(io, (y.reshape(-1, L)[chan], hT.reshape(-1, N)[chan], vT.reshape(-1, N)[chan]),
             (yr, hr, vr), what)


# --------------------------------------------------------- workloads -----
@pytest.mark.parametrize("beta,alpha", wl.SCAN_SMALL.runs)
def test_small_workload_full_output(beta, alpha):
    inp = wl.scan_inputs(wl.SCAN_SMALL)
    _full_compare(inp, "f32", beta, alpha, what=f"small b={beta} a={alpha}")


def test_medium_workload_all_runs_reduced_size():
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=2, seqlen=512, dim=96)
    for beta, alpha in wl.SCAN_MEDIUM.runs:
        _full_compare(inp, "f32", beta, alpha, what=f"medium-reduced b={beta} a={alpha}")


def test_medium_workload_full_size_sampled():
    w = wl.SCAN_MEDIUM
    inp = wl.scan_inputs(w)
    dev = _dev(inp, "f32")
    for beta, alpha in ((0.9, 1.0), (0.5, 2.0), (0.0, 0.5)):
        _sampled_compare(inp, "f32", beta, alpha, dev=dev, what=f"medium b={beta} a={alpha}")


def test_bf16_workload_reduced_size_full_output():
    inp = wl.scan_inputs(wl.SCAN_BF16, batch=2, seqlen=1024, dim=256)
    _full_compare(inp, "bf16", 0.9, 1.0, what="bf16-reduced")


def test_bf16_workload_full_size_sampled():
    inp = wl.scan_inputs(wl.SCAN_BF16)
    _sampled_compare(inp, "bf16", 0.9, 1.0, what="bf16 full")


def test_long_workload_streaming_split_bit_identical():
    w = wl.SCAN_LONG
    inp = wl.scan_inputs(w)
    beta, alpha = w.runs[0]
    dev = _dev(inp, "f32")
    one = _run(dev, beta, alpha)
    half = w.split
    d1 = {k: (v[..., :half].contiguous() if k in ("x", "delta", "B", "C") else v) for k, v in dev.items()}
    d2 = {k: (v[..., half:].contiguous() if k in ("x", "delta", "B", "C") else v) for k, v in dev.items()}
    y1, h1, v1 = mm.scan_fwd(d1["x"], d1["delta"], d1["A"], d1["B"], d1["C"], beta=beta, alpha=alpha)
    y2, h2, v2 = mm.scan_fwd(d2["x"], d2["delta"], d2["A"], d2["B"], d2["C"], h0=h1, v0=v1,
                             beta=beta, alpha=alpha)
    torch.cuda.synchronize()
    assert np.array_equal(h2.cpu().numpy(), one[1]), "hT differs between one call and two calls"
    assert np.array_equal(v2.cpu().numpy(), one[2]), "vT differs between one call and two calls"
    ysplit = torch.cat([y1, y2], dim=-1).cpu().numpy()
    scale = np.abs(one[0]).max()
    assert np.abs(ysplit - one[0]).max() <= F32_TOL * scale
    # 64 sampled channels (the first and the last included) against the oracle
    _sampled_compare(inp, "f32", beta, alpha, got=one, k=64, what="long one-shot")
    # and the state handed over at the split point
    N = inp["A"].shape[1]
    chan = _sample_channels(inp["x"].shape[0] * inp["x"].shape[1], 64)
    inp1 = {k: (np.ascontiguousarray(v[..., :half]) if k in ("x", "delta", "B", "C") else v)
            for k, v in inp.items()}
    _, hr1, vr1 = oracle.scan_seq(**inp1, beta=beta, alpha=alpha, chan=chan)
    _max_abs_ok(h1.cpu().numpy().reshape(-1, N)[chan], hr1, "long split-point hT")
    _max_abs_ok(v1.cpu().numpy().reshape(-1, N)[chan], vr1, "long split-point vT")


# -------------------------------------------------------- edge cases -----
EDGE = [
    # batch, L, dim, N, io, beta, alpha, with_state
    (1, 1, 8, 16, "f32", 0.9, 1.0, True),        # single-step sequence
    (2, 3, 5, 3, "f32", 0.5, 1.0, True),         # ragged L, rows not 16-byte multiples
    (1, 33, 7, 16, "f32", 0.9, 2.0, False),      # one full chunk plus one step
    (3, 36, 9, 8, "bf16", 0.9, 1.0, True),       # bf16, L*2 not a multiple of 16
    (1, 37, 16, 16, "bf16", 0.3, 1.0, False),    # bf16 rows with odd length
    (2, 100, 33, 1, "f32", 0.9, 1.0, True),      # one state
    (1, 64, 17, 2, "f32", 0.0, 1.0, True),       # two states
    (1, 64, 19, 4, "bf16", 0.9, 1.0, False),
    (32, 64, 4, 16, "f32", 0.9, 1.0, False),     # batch = 32 (README edge list)
    (2, 256, 24, 16, "f32", 1e-6, 1.0, True),    # beta = 1e-6
    (2, 256, 24, 16, "f32", 0.999, 1.0, True),   # beta = 0.999
    (2, 256, 24, 16, "f32", 0.9, 10.0, True),    # alpha = 10
    (1, 4096, 3, 16, "bf16", 0.99, 0.5, True),
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "-".join(map(str, c)))
def test_edge_cases(case):
    bsz, L, D, N, io, beta, alpha, with_state = case
    w = wl.SCAN_BF16 if io == "bf16" else wl.SCAN_SMALL
    inp = wl.scan_inputs(w, batch=bsz, seqlen=L, dim=D, dstate=N)
    h0 = v0 = None
    if with_state:
        rng = np.random.default_rng(L * 7 + D)
        h0 = rng.standard_normal((bsz, D, N)).astype(np.float32)
        v0 = rng.standard_normal((bsz, D, N)).astype(np.float32)
    _full_compare(inp, io, beta, alpha, h0=h0, v0=v0, what=str(case))


def test_alpha_zero_is_exactly_zero():
    inp = wl.scan_inputs(wl.SCAN_SMALL, dim=32)
    y, hT, vT = _run(_dev(inp, "f32"), 0.9, 0.0)
    assert not y.any() and not hT.any() and not vT.any()


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_every_tile_variant_matches(io):
    w = wl.SCAN_BF16 if io == "bf16" else wl.SCAN_MEDIUM
    inp = wl.scan_inputs(w, batch=2, seqlen=200, dim=70)
    dev = _dev(inp, io)
    mm.mm_scan_set_path(1, 0)          # the tiles are those of the register-resident kernel
    yr, hr, vr = oracle.scan_seq(**inp, beta=0.9, alpha=1.0)
    try:
        base = _run(dev, 0.9, 1.0)
        for spt, warps in ((2, 2), (2, 4), (2, 8), (4, 1), (4, 2), (4, 4)):
                mm.mm_scan_set_tile(spt, warps, 1)
                got = _run(dev, 0.9, 1.0)
                _compare(io, (got[0].reshape(-1, 200), got[1].reshape(-1, 16), got[2].reshape(-1, 16)),
                         (yr, hr, vr), f"tile spt={spt} warps={warps}")
                # the per-state arithmetic is the same in every variant
                assert np.array_equal(got[1], base[1]) and np.array_equal(got[2], base[2])
    finally:
        mm.mm_scan_set_tile(0, 0, 1)
        mm.mm_scan_set_path(0, 0)


TIME_SPLIT_TILES = ((4, 2), (4, 4), (2, 4), (2, 8))


def test_time_split_variants_match_and_agree_on_state():
    """fp32 variants with two lanes along time per state group: each matches
    the oracle (ragged last chunk, carried initial state), and all give the
    same final states, since the per-state arithmetic does not depend on
    how states are spread over lanes."""
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=2, seqlen=200, dim=70)
    dev = _dev(inp, "f32")
    rng = np.random.default_rng(4)
    h0 = rng.standard_normal((2, 70, 16)).astype(np.float32)
    v0 = rng.standard_normal((2, 70, 16)).astype(np.float32)
    th0, tv0 = torch.from_numpy(h0).cuda(), torch.from_numpy(v0).cuda()
    yr, hr, vr = oracle.scan_seq(**inp, h0=h0.astype(np.float64), v0=v0.astype(np.float64),
                                 beta=0.9, alpha=1.0)
    first = None
    mm.mm_scan_set_path(1, 0)
    try:
        for spt, warps in TIME_SPLIT_TILES:
            mm.mm_scan_set_tile(spt, warps, 2)
            got = _run(dev, 0.9, 1.0, th0, tv0)
            _compare("f32", (got[0].reshape(-1, 200), got[1].reshape(-1, 16), got[2].reshape(-1, 16)),
                     (yr, hr, vr), f"time split spt={spt} warps={warps}")
            if first is None:
                first = got
            assert np.array_equal(got[1], first[1]) and np.array_equal(got[2], first[2])
    finally:
        mm.mm_scan_set_tile(0, 0, 1)
        mm.mm_scan_set_path(0, 0)


@pytest.mark.parametrize("L", [1, 31, 32, 33, 64, 65, 130])
@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_time_split_lengths(L, beta):
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=1, seqlen=L, dim=24)
    mm.mm_scan_set_path(1, 0)
    try:
        mm.mm_scan_set_tile(4, 2, 2)
        _full_compare(inp, "f32", beta, 1.0, what=f"time split L={L} beta={beta}")
    finally:
        mm.mm_scan_set_tile(0, 0, 1)
        mm.mm_scan_set_path(0, 0)


def _split_streaming_bit_identical(halves):
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=2, seqlen=448, dim=40)
    dev = _dev(inp, "f32")
    one = _run(dev, 0.99, 1.0)
    for half in halves:
        d1 = {k: (v[..., :half].contiguous() if k in ("x", "delta", "B", "C") else v) for k, v in dev.items()}
        d2 = {k: (v[..., half:].contiguous() if k in ("x", "delta", "B", "C") else v) for k, v in dev.items()}
        y1, h1, v1 = mm.scan_fwd(d1["x"], d1["delta"], d1["A"], d1["B"], d1["C"], beta=0.99, alpha=1.0)
        y2, h2, v2 = mm.scan_fwd(d2["x"], d2["delta"], d2["A"], d2["B"], d2["C"], h0=h1, v0=v1,
                                 beta=0.99, alpha=1.0)
        torch.cuda.synchronize()
        assert np.array_equal(h2.cpu().numpy(), one[1]), f"hT differs (split at {half})"
        assert np.array_equal(v2.cpu().numpy(), one[2]), f"vT differs (split at {half})"


def test_register_path_streaming_any_split_bit_identical():
    # one time lane per state group applies the steps in order: any split point
    mm.mm_scan_set_path(1, 0)
    try:
        _split_streaming_bit_identical((100, 1, 257, 444))
    finally:
        mm.mm_scan_set_path(0, 0)


def test_time_split_streaming_bit_identical():
    # the time split carries its state across 32-step chunks: splits at multiples of 32
    mm.mm_scan_set_path(1, 0)
    try:
        mm.mm_scan_set_tile(4, 2, 2)
        _split_streaming_bit_identical((64, 192, 384, 32, 416))
    finally:
        mm.mm_scan_set_tile(0, 0, 1)
        mm.mm_scan_set_path(0, 0)


def test_in_place_streaming_state_and_optional_outputs():
    inp = wl.scan_inputs(wl.SCAN_SMALL, batch=2, seqlen=128, dim=24)
    dev = _dev(inp, "f32")
    rng = np.random.default_rng(2)
    h0 = rng.standard_normal((2, 24, 16)).astype(np.float32)
    v0 = rng.standard_normal((2, 24, 16)).astype(np.float32)
    yr, hr, vr = oracle.scan_seq(**inp, h0=h0.astype(np.float64), v0=v0.astype(np.float64),
                                 beta=0.9, alpha=1.0)
    hs = torch.from_numpy(h0).cuda()
    vs = torch.from_numpy(v0).cuda()
    y = torch.empty_like(dev["x"])
    mm.mm_scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], hs, vs, 0.9, 1.0, y, hs, vs)
    torch.cuda.synchronize()
    _compare("f32", (y.cpu().numpy().reshape(-1, 128), hs.cpu().numpy().reshape(-1, 16),
                     vs.cpu().numpy().reshape(-1, 16)), (yr, hr, vr), "in-place")
    y2 = torch.empty_like(dev["x"])
    mm.mm_scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], None, None, 0.9, 1.0,
                   y2, None, None)
    torch.cuda.synchronize()
    yr0, _, _ = oracle.scan_seq(**inp, beta=0.9, alpha=1.0)
    _max_abs_ok(y2.cpu().numpy().reshape(-1, 128), yr0, "no final state")


def test_causality_and_determinism():
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=1, seqlen=300, dim=40)
    dev = _dev(inp, "f32")
    a = _run(dev, 0.9, 1.0)
    b = _run(dev, 0.9, 1.0)
    assert all(np.array_equal(p, q) for p, q in zip(a, b)), "two runs differ"
    k = 150
    dev["x"][:, :, k] += 1.0
    c = _run(dev, 0.9, 1.0)
    assert np.array_equal(c[0][:, :, :k], a[0][:, :, :k])
    assert not np.array_equal(c[0][:, :, k], a[0][:, :, k])


def test_errors_on_device_buffers():
    inp = wl.scan_inputs(wl.SCAN_SMALL, dim=16)
    dev = _dev(inp, "f32")
    y = torch.empty_like(dev["x"])
    with pytest.raises(mm.MMError) as e:
        mm.mm_scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], None, None, 0.9, 1.0,
                       dev["x"], None, None)
    assert e.value.name == "MM_ERR_ALIAS"
    flat = torch.empty(dev["x"].numel() + 1, device="cuda")
    bad = flat[1:].view_as(dev["x"])
    with pytest.raises(mm.MMError) as e:
        mm.mm_scan_fwd(bad, dev["delta"], dev["A"], dev["B"], dev["C"], None, None, 0.9, 1.0,
                       y, None, None)
    assert e.value.name == "MM_ERR_ALIGN"
