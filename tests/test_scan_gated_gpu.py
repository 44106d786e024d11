"""GPU parity of mm_scan_fwd_gated (delta bias and softplus, D skip, SiLU
gate) against the fp64 oracle's scan_gated, through the C ABI.

Tolerances as for the plain scan: fp32 I/O max |out - ref| <= 1e-4 max |ref|
(and the same for hT, vT); bf16 I/O relative L2 <= 1e-2.
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


def _t(a, dt=torch.float32):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().to(dt).contiguous()


def _case(w, batch, L, dim, use_D, use_z, use_bias, softplus, beta=0.9, alpha=1.0, h0v0=False,
          chan=None):
    inp = wl.scan_inputs(w, batch=batch, seqlen=L, dim=dim)
    ex = wl.scan_extras(w, batch=batch, seqlen=L, dim=dim)
    D = ex["D"] if use_D else None
    z = ex["z"] if use_z else None
    if softplus:        # raw delta and an inverse-softplus bias, as a Mamba layer feeds them
        delta = ex["delta_raw"]
        bias = ex["delta_bias"] if use_bias else None
    else:               # without softplus the step must stay positive: a small positive bias
        delta = inp["delta"]
        bias = np.linspace(1e-3, 5e-2, dim, dtype=np.float32) if use_bias else None
    h0 = v0 = None
    if h0v0:
        rng = np.random.default_rng(L + dim)
        h0 = rng.standard_normal((batch, dim, 16)).astype(np.float32)
        v0 = rng.standard_normal((batch, dim, 16)).astype(np.float32)
    io = torch.float32 if w.io == "f32" else torch.bfloat16
    y, hT, vT = mm.scan_fwd(_t(inp["x"], io), _t(delta, io), _t(inp["A"]), _t(inp["B"], io),
                            _t(inp["C"], io), h0=_t(h0), v0=_t(v0), beta=beta, alpha=alpha,
                            D=_t(D), z=_t(z, io), delta_bias=_t(bias), delta_softplus=softplus)
    torch.cuda.synchronize()
    mm.mm_device_status()
    yr, hr, vr = oracle.scan_gated(inp["x"], delta, inp["A"], inp["B"], inp["C"], D=D, z=z,
                                   delta_bias=bias, delta_softplus=softplus,
                                   h0=None if h0 is None else h0.astype(np.float64),
                                   v0=None if v0 is None else v0.astype(np.float64),
                                   beta=beta, alpha=alpha, chan=chan)
    y = y.float().cpu().numpy().reshape(-1, L)
    hT = hT.cpu().numpy().reshape(-1, 16)
    vT = vT.cpu().numpy().reshape(-1, 16)
    if chan is not None:
        y, hT, vT = y[chan], hT[chan], vT[chan]
    what = f"{w.io} L={L} D={use_D} z={use_z} bias={use_bias} softplus={softplus}"
    if w.io == "f32":
        assert np.abs(y - yr).max() <= F32_TOL * np.abs(yr).max(), what + " out"
    else:
        assert np.linalg.norm(y - yr) / np.linalg.norm(yr) <= BF16_TOL, what + " out"
    for got, ref, nm in ((hT, hr, "hT"), (vT, vr, "vT")):
        assert np.abs(got - ref).max() <= F32_TOL * np.abs(ref).max(), f"{what} {nm}"
    return y, hT, vT


COMBOS = [
    # D, z, bias, softplus
    (True, False, False, False),
    (False, True, False, False),
    (False, False, True, False),
    (False, False, False, True),
    (False, False, True, True),
    (True, True, True, True),
]


@pytest.mark.parametrize("combo", COMBOS, ids=lambda c: "".join("DzbS"[i] if f else "-" for i, f in enumerate(c)))
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_extras_each_and_all(io, combo):
    w = wl.SCAN_BF16 if io == "bf16" else wl.SCAN_MEDIUM
    _case(w, 2, 200, 70, *combo, h0v0=True)      # ragged last chunk, a partial channel tile


@pytest.mark.parametrize("L", [1, 37, 64, 129])
def test_extras_lengths_and_row_fallback(L):
    # L = 37 fp32 rows are not whole 16-byte pieces: element-wise staging
    _case(wl.SCAN_MEDIUM, 1, L, 24, True, True, True, True, beta=0.5, alpha=2.0)


@pytest.mark.parametrize("dstate", [1, 4, 8])
def test_extras_small_state_counts(dstate):
    w = wl.SCAN_MEDIUM
    inp = wl.scan_inputs(w, batch=1, seqlen=96, dim=20, dstate=dstate)
    ex = wl.scan_extras(w, batch=1, seqlen=96, dim=20)
    t = lambda a: _t(a)
    y, hT, vT = mm.scan_fwd(t(inp["x"]), t(ex["delta_raw"]), t(inp["A"]), t(inp["B"]), t(inp["C"]),
                            beta=0.9, alpha=1.0, D=t(ex["D"]), z=t(ex["z"]),
                            delta_bias=t(ex["delta_bias"]), delta_softplus=True)
    torch.cuda.synchronize()
    yr, hr, vr = oracle.scan_gated(inp["x"], ex["delta_raw"], inp["A"], inp["B"], inp["C"], D=ex["D"],
                                   z=ex["z"], delta_bias=ex["delta_bias"], delta_softplus=True,
                                   beta=0.9, alpha=1.0)
    y = y.cpu().numpy().reshape(-1, 96)
    assert np.abs(y - yr).max() <= F32_TOL * np.abs(yr).max()
    assert np.abs(hT.cpu().numpy().reshape(-1, dstate) - hr).max() <= F32_TOL * np.abs(hr).max()


def test_extras_full_size_medium_sampled():
    w = wl.SCAN_MEDIUM
    nch = w.batch * w.dim
    rng = np.random.default_rng(0)
    chan = np.unique(np.concatenate([rng.choice(nch, 24, replace=False), [0, nch - 1]])).astype(np.int64)
    _case(w, w.batch, w.seqlen, w.dim, True, True, True, True, chan=chan)


def test_extras_streaming_split_bit_identical():
    w = wl.SCAN_MEDIUM
    L, dim = 512, 40
    inp = wl.scan_inputs(w, batch=2, seqlen=L, dim=dim)
    ex = wl.scan_extras(w, batch=2, seqlen=L, dim=dim)
    dev = {k: _t(v) for k, v in inp.items()}
    d = _t(ex["delta_raw"]); z = _t(ex["z"]); D = _t(ex["D"]); bias = _t(ex["delta_bias"])
    kw = dict(beta=0.99, alpha=1.0, D=D, delta_bias=bias, delta_softplus=True)
    y, h, v = mm.scan_fwd(dev["x"], d, dev["A"], dev["B"], dev["C"], z=z, **kw)
    half = 192
    sl = lambda a, lo, hi: a[..., lo:hi].contiguous()
    y1, h1, v1 = mm.scan_fwd(sl(dev["x"], 0, half), sl(d, 0, half), dev["A"], sl(dev["B"], 0, half),
                             sl(dev["C"], 0, half), z=sl(z, 0, half), **kw)
    y2, h2, v2 = mm.scan_fwd(sl(dev["x"], half, L), sl(d, half, L), dev["A"], sl(dev["B"], half, L),
                             sl(dev["C"], half, L), z=sl(z, half, L), h0=h1, v0=v1, **kw)
    torch.cuda.synchronize()
    assert torch.equal(h2, h) and torch.equal(v2, v)
    assert torch.allclose(torch.cat([y1, y2], dim=-1), y, rtol=0, atol=F32_TOL * float(y.abs().max()))


def test_gated_rejects_bad_extras():
    inp = wl.scan_inputs(wl.SCAN_SMALL, batch=1, seqlen=64, dim=8)
    dev = {k: _t(v) for k, v in inp.items()}
    y = torch.empty_like(dev["x"])
    with pytest.raises(mm.MMError) as e:          # y on top of z
        mm.mm_scan_fwd_gated(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], None, y, None, 0,
                             None, None, 0.9, 1.0, y, None, None)
    assert e.value.name == "MM_ERR_ALIAS"
