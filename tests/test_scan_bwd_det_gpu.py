"""The deterministic backward (mm_scan_set_deterministic(1)).

Its parameter gradients -- dA, dB, dC and, through the extras, dD and
ddelta_bias -- are sums over CTAs that the default form adds atomically in
no fixed order.  Switched on, each CTA writes its channel tile's partials to
a workspace and a second kernel adds them in a fixed order, so two runs on
the same inputs give the same bits.  Each case runs the deterministic form
twice (L2 flushed between) and compares every output bit for bit, checks it
against the fp64 oracle ("Momentum Mamba: Enhanced State Space Models with
Momentum", sections "Gradient Flow" and "Backward Pass: Reconstructed
Forward + Reverse Scans") at the same tolerance as the default form, and
against the default form within that tolerance -- on every tile variant of
the backward (dstate 16 with four- and two-warp CTAs, 8, 4, 2), ragged rows,
both element types and the gated extras.
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
def det():
    mm.mm_scan_set_deterministic(True)
    yield
    mm.mm_scan_set_deterministic(False)


def _t(a, dt=torch.float32):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().to(dt).contiguous()


def _flush():
    torch.empty(256 << 20, dtype=torch.uint8, device="cuda").fill_(1)


def _problem(io, batch, L, dim, dstate, extras, seed):
    w = wl.SCAN_BF16 if io == "bf16" else wl.SCAN_MEDIUM
    inp = wl.scan_inputs(w, batch=batch, seqlen=L, dim=dim, dstate=dstate, seed=seed)
    rng = np.random.default_rng(seed)
    if io == "bf16":
        for k in ("x", "delta", "B", "C"):
            inp[k] = wl.bf16_round(inp[k])
    g = {"dy": rng.standard_normal((batch, dim, L)).astype(np.float32),
         "dhT": rng.standard_normal((batch, dim, dstate)).astype(np.float32),
         "dvT": rng.standard_normal((batch, dim, dstate)).astype(np.float32)}
    if io == "bf16":
        g["dy"] = wl.bf16_round(g["dy"])
    inp["h0"] = rng.standard_normal((batch, dim, dstate)).astype(np.float32)
    inp["v0"] = rng.standard_normal((batch, dim, dstate)).astype(np.float32)
    kw = {}
    if extras:
        ex = wl.scan_extras(w, batch=batch, seqlen=L, dim=dim, seed=seed)
        inp["delta"] = ex["delta_raw"] if io == "f32" else wl.bf16_round(ex["delta_raw"])
        kw = dict(D=ex["D"], z=ex["z"] if io == "f32" else wl.bf16_round(ex["z"]),
                  delta_bias=ex["delta_bias"], delta_softplus=True)
    return inp, g, kw


def _run(io, inp, g, kw, beta=0.9, alpha=1.0):
    dt = torch.float32 if io == "f32" else torch.bfloat16
    dev = {k: _t(inp[k], dt) for k in ("x", "delta", "B", "C")}
    A, h0, v0 = _t(inp["A"]), _t(inp["h0"]), _t(inp["v0"])
    dkw = {}
    if kw:
        dkw = dict(D=_t(kw["D"]), z=_t(kw["z"], dt), delta_bias=_t(kw["delta_bias"]),
                   delta_softplus=kw["delta_softplus"])
    _, _, _, ckpt = mm.scan_fwd_train(dev["x"], dev["delta"], A, dev["B"], dev["C"], h0=h0, v0=v0,
                                      beta=beta, alpha=alpha, **dkw)
    _flush()
    gr = mm.scan_bwd(dev["x"], dev["delta"], A, dev["B"], dev["C"], ckpt, _t(g["dy"], dt), h0=h0, v0=v0,
                     dhT=_t(g["dhT"]), dvT=_t(g["dvT"]), beta=beta, alpha=alpha, **dkw)
    torch.cuda.synchronize()
    mm.mm_device_status()
    return {k: v.float().cpu().numpy() for k, v in gr.items() if v is not None}


def _oracle(inp, g, kw, beta=0.9, alpha=1.0):
    f64 = lambda a: None if a is None else np.asarray(a, np.float64)
    return oracle.scan_bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], g["dy"],
                           h0=f64(inp["h0"]), v0=f64(inp["v0"]), dhT=f64(g["dhT"]), dvT=f64(g["dvT"]),
                           beta=beta, alpha=alpha, **kw)


def _close(io, got, ref, what):
    for k, r in ref.items():
        if k not in got:
            continue
        a = got[k].reshape(r.shape)
        if io == "f32":
            err = np.abs(a - r).max()
            assert err <= F32_TOL * np.abs(r).max(), f"{what} {k}: {err:.3g} vs max {np.abs(r).max():.3g}"
        else:
            rel = np.linalg.norm(a - r) / np.linalg.norm(r)
            assert rel <= BF16_TOL, f"{what} {k}: rel L2 {rel:.3g}"


CASES = [
    # io, batch, L, dim, dstate, extras: the tile each picks
    ("f32", 2, 200, 1040, 16, False),     # four-warp CTAs (batch * dim >= 2048), 16 channels
    ("f32", 2, 200, 70, 16, False),       # two-warp CTAs, a partial channel tile
    ("f32", 1, 37, 24, 16, False),        # rows not whole 16-byte pieces: element-wise staging
    ("f32", 2, 150, 20, 8, False),
    ("f32", 2, 150, 40, 4, False),
    ("f32", 2, 150, 70, 2, False),
    ("bf16", 2, 256, 1040, 16, False),
    ("f32", 2, 200, 1040, 16, True),      # the gated extras, four-warp CTAs
    ("f32", 2, 200, 70, 16, True),
    ("bf16", 2, 256, 70, 16, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-B{c[1]}-L{c[2]}-D{c[3]}-N{c[4]}" +
                         ("-gated" if c[5] else ""))
def test_deterministic_backward(det, case):
    io, batch, L, dim, dstate, extras = case
    inp, g, kw = _problem(io, batch, L, dim, dstate, extras, seed=L + dim + dstate)
    first = _run(io, inp, g, kw)
    second = _run(io, inp, g, kw)
    for k in first:
        assert np.array_equal(first[k], second[k]), f"{k} differs between two deterministic runs"
    _close(io, first, _oracle(inp, g, kw), f"deterministic {case}")
    mm.mm_scan_set_deterministic(False)
    atomic = _run(io, inp, g, kw)
    ref = {k: v for k, v in atomic.items()}
    _close(io, first, {k: np.asarray(v, np.float64) for k, v in ref.items() if np.any(v)},
           f"deterministic vs atomic {case}")


def test_deterministic_backward_full_size_medium(det):
    # the medium workload (4 x 1536 channels, 2048 steps): 101 MB of workspace
    w = wl.SCAN_MEDIUM
    inp = wl.scan_inputs(w)
    rng = np.random.default_rng(5)
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    dev = {k: _t(inp[k]) for k in ("x", "delta", "B", "C")}
    A = _t(inp["A"])
    _, _, _, ckpt = mm.scan_fwd_train(dev["x"], dev["delta"], A, dev["B"], dev["C"], beta=0.9)
    outs = []
    for _ in range(2):
        _flush()
        gr = mm.scan_bwd(dev["x"], dev["delta"], A, dev["B"], dev["C"], ckpt, _t(dy), beta=0.9)
        torch.cuda.synchronize()
        mm.mm_device_status()
        outs.append({k: v.clone() for k, v in gr.items() if v is not None})
    for k in outs[0]:
        assert torch.equal(outs[0][k], outs[1][k]), f"{k} differs between two deterministic runs"
    mm.mm_scan_set_deterministic(False)
    gr = mm.scan_bwd(dev["x"], dev["delta"], A, dev["B"], dev["C"], ckpt, _t(dy), beta=0.9)
    torch.cuda.synchronize()
    for k in ("dA", "dB", "dC"):
        a, r = outs[0][k].cpu().numpy(), gr[k].cpu().numpy()
        assert np.abs(a - r).max() <= F32_TOL * np.abs(r).max(), k


def test_deterministic_backward_refuses_graph_capture(det):
    inp, g, _ = _problem("f32", 1, 64, 16, 16, False, seed=3)
    dev = {k: _t(inp[k]) for k in ("x", "delta", "B", "C")}
    A = _t(inp["A"])
    _, _, _, ckpt = mm.scan_fwd_train(dev["x"], dev["delta"], A, dev["B"], dev["C"], beta=0.9)
    dy = _t(g["dy"])
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with pytest.raises(mm.MMError) as err:
        with torch.cuda.graph(graph, stream=s):
            mm.scan_bwd(dev["x"], dev["delta"], A, dev["B"], dev["C"], ckpt, dy, beta=0.9, stream=s)
    assert "captured" in str(err.value)
    torch.cuda.synchronize()
