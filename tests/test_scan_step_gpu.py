"""GPU parity of the decode step (mm_scan_step) against the fp64 oracle's
one-step scan (oracle.scan_gated with L = 1 and the cached states as h0,
v0), through the C ABI, and its agreement with the scan kernel.

Tolerances as for the scan: fp32 I/O max |y - ref| <= 1e-4 max |ref| (and
the same for the updated states); bf16 I/O relative L2 <= 1e-2 for y, the
fp32 states to 1e-4 of their largest value.
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


def _run(inp, io, use_D, use_z, use_bias, softplus, beta=0.9, alpha=1.0, chan=None):
    dt = torch.float32 if io == "f32" else torch.bfloat16
    dev = {k: _t(inp[k], dt) for k in ("x", "delta", "B", "C", "z")}
    h, v = _t(inp["h"]), _t(inp["v"])
    y = torch.empty_like(dev["x"])
    mm.mm_scan_step(dev["x"], dev["delta"], _t(inp["A"]), dev["B"], dev["C"],
                    _t(inp["D"]) if use_D else None, dev["z"] if use_z else None,
                    _t(inp["delta_bias"]) if use_bias else None, softplus, h, v, beta, alpha, y)
    torch.cuda.synchronize()
    mm.mm_device_status()
    batch, dim = inp["x"].shape
    N = inp["A"].shape[1]
    col = lambda a: a[..., None]
    yr, hr, vr = oracle.scan_gated(col(inp["x"]), col(inp["delta"]), inp["A"], col(inp["B"]), col(inp["C"]),
                                   D=inp["D"] if use_D else None, z=col(inp["z"]) if use_z else None,
                                   delta_bias=inp["delta_bias"] if use_bias else None,
                                   delta_softplus=softplus, h0=inp["h"].astype(np.float64),
                                   v0=inp["v"].astype(np.float64), beta=beta, alpha=alpha, chan=chan)
    got = (y.float().cpu().numpy().reshape(-1), h.cpu().numpy().reshape(-1, N), v.cpu().numpy().reshape(-1, N))
    if chan is not None:
        got = (got[0][chan], got[1][chan], got[2][chan])
    what = f"{io} D={use_D} z={use_z} bias={use_bias} softplus={softplus}"
    yr = yr.reshape(-1)
    if io == "f32":
        assert np.abs(got[0] - yr).max() <= F32_TOL * np.abs(yr).max(), what + " y"
    else:
        assert np.linalg.norm(got[0] - yr) / np.linalg.norm(yr) <= BF16_TOL, what + " y"
    for a, r, nm in ((got[1], hr, "h"), (got[2], vr, "v")):
        assert np.abs(a - r).max() <= F32_TOL * np.abs(r).max(), f"{what} {nm}"


COMBOS = [(False, False, False, False), (True, True, True, True), (True, False, False, False),
          (False, True, False, False), (False, False, True, False), (False, False, False, True)]


@pytest.mark.parametrize("combo", COMBOS, ids=lambda c: "".join("DzbS"[i] if f else "-" for i, f in enumerate(c)))
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_step_matches_oracle(io, combo):
    w = wl.DecodeWorkload("t", 7, 37, 16, io=io)          # ragged warp tail
    inp = wl.decode_inputs(w)
    if not combo[3]:                                       # without softplus the step must stay positive
        delta = np.abs(inp["delta"]) * np.float32(0.05)
        inp["delta"] = wl.bf16_round(delta) if io == "bf16" else delta
        inp["delta_bias"] = np.full_like(inp["delta_bias"], 0.01)
    _run(inp, io, *combo)


@pytest.mark.parametrize("dstate", [1, 3, 4, 5, 8, 12, 13, 16])
def test_step_state_counts(dstate):
    # multiples of 4 take the 16-byte state path, others the element path
    inp = wl.decode_inputs(wl.DecodeWorkload("t", 3, 50, dstate, io="f32"))
    _run(inp, "f32", True, True, True, True, beta=0.5, alpha=2.0)


def test_step_full_size_sampled():
    w = wl.DECODE
    inp = wl.decode_inputs(w)
    rng = np.random.default_rng(3)
    chan = np.unique(np.concatenate([rng.choice(w.batch * w.dim, 200, replace=False),
                                     [0, w.batch * w.dim - 1]])).astype(np.int64)
    _run(inp, w.io, True, True, True, True, beta=w.beta, alpha=w.alpha, chan=chan)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_steps_equal_one_scan(io):
    """L decode steps leave the states bit-identical to one gated scan over
    the L steps; the outputs agree within rounding of the read-out."""
    dt = torch.float32 if io == "f32" else torch.bfloat16
    w = wl.SCAN_MEDIUM if io == "f32" else wl.SCAN_BF16
    L, batch, dim = 24, 3, 40
    inp = wl.scan_inputs(w, batch=batch, seqlen=L, dim=dim)
    ex = wl.scan_extras(w, batch=batch, seqlen=L, dim=dim)
    rng = np.random.default_rng(8)
    h0 = _t(rng.standard_normal((batch, dim, 16)).astype(np.float32))
    v0 = _t(rng.standard_normal((batch, dim, 16)).astype(np.float32))
    x, d, B, C, z = (_t(a, dt) for a in (inp["x"], ex["delta_raw"], inp["B"], inp["C"], ex["z"]))
    A, D, bias = _t(inp["A"]), _t(ex["D"]), _t(ex["delta_bias"])
    y, hT, vT = mm.scan_fwd(x, d, A, B, C, h0=h0, v0=v0, beta=0.9, alpha=1.0, D=D, z=z,
                            delta_bias=bias, delta_softplus=True)
    h, v = h0.clone(), v0.clone()
    ys = []
    for t in range(L):
        yt = torch.empty((batch, dim), device="cuda", dtype=dt)
        mm.mm_scan_step(x[..., t].contiguous(), d[..., t].contiguous(), A, B[..., t].contiguous(),
                        C[..., t].contiguous(), D, z[..., t].contiguous(), bias, True, h, v, 0.9, 1.0, yt)
        ys.append(yt)
    torch.cuda.synchronize()
    assert torch.equal(h, hT) and torch.equal(v, vT)
    ystep = torch.stack(ys, dim=-1).float()
    tol = F32_TOL if io == "f32" else 1e-2
    assert float((ystep - y.float()).abs().max()) <= tol * float(y.float().abs().max())


def test_step_rejects_overlaps():
    inp = wl.decode_inputs(wl.DecodeWorkload("t", 2, 16, 16, io="f32"))
    dev = {k: _t(v) for k, v in inp.items()}
    y = torch.empty_like(dev["x"])
    with pytest.raises(mm.MMError) as e:
        mm.mm_scan_step(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], None, None, None, False,
                        dev["h"], dev["h"], 0.9, 1.0, y)
    assert e.value.name == "MM_ERR_ALIAS"
