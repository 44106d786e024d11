"""GPU parity of the backward (mm_scan_bwd) and of the forward's checkpoints
against the fp64 oracle, through the C ABI.

Tolerances: fp32 I/O max |g - ref| <= 1e-4 max |ref| for every gradient
(dx, ddelta, dA, dB, dC, dh0, dv0); bf16 I/O relative L2 <= 1e-2 for dx and
ddelta (stored in bf16) and the fp32 gradients alike.  Checkpoints: 1e-4 of
the largest state, like hT and vT.
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
GRADS = ("dx", "ddelta", "dA", "dB", "dC", "dh0", "dv0")


def _t(a, dt=torch.float32):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().to(dt).contiguous()


def _round(a, io):
    """The values a bf16 tensor of `a` holds, as fp32 (what the oracle reads)."""
    if io == "f32":
        return np.asarray(a, np.float32)
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def _problem(w, batch, L, dim, dstate=16, h0v0=True, seed=0):
    inp = wl.scan_inputs(w, batch=batch, seqlen=L, dim=dim, dstate=dstate)
    rng = np.random.default_rng(seed + L + 7 * dim)
    g = {"dy": _round(rng.standard_normal((batch, dim, L)), w.io)}
    if h0v0:
        inp["h0"] = rng.standard_normal((batch, dim, dstate)).astype(np.float32)
        inp["v0"] = rng.standard_normal((batch, dim, dstate)).astype(np.float32)
        g["dhT"] = rng.standard_normal((batch, dim, dstate)).astype(np.float32)
        g["dvT"] = rng.standard_normal((batch, dim, dstate)).astype(np.float32)
    return inp, g


def _gpu(w, inp, g, beta, alpha):
    io = torch.float32 if w.io == "f32" else torch.bfloat16
    dev = {k: _t(inp[k], io) for k in ("x", "delta", "B", "C")}
    A, h0, v0 = _t(inp["A"]), _t(inp.get("h0")), _t(inp.get("v0"))
    y, hT, vT, ckpt = mm.scan_fwd_train(dev["x"], dev["delta"], A, dev["B"], dev["C"], h0=h0, v0=v0,
                                        beta=beta, alpha=alpha)
    gr = mm.scan_bwd(dev["x"], dev["delta"], A, dev["B"], dev["C"], ckpt, _t(g["dy"], io), h0=h0, v0=v0,
                     dhT=_t(g.get("dhT")), dvT=_t(g.get("dvT")), beta=beta, alpha=alpha)
    torch.cuda.synchronize()
    mm.mm_device_status()
    return {k: v.float().cpu().numpy() for k, v in gr.items()}, (y, hT, vT, ckpt)


def _ref(inp, g, beta, alpha, chan=None, bn=None):
    f64 = lambda a: None if a is None else np.asarray(a, np.float64)
    return oracle.scan_bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], g["dy"],
                           h0=f64(inp.get("h0")), v0=f64(inp.get("v0")), dhT=f64(g.get("dhT")),
                           dvT=f64(g.get("dvT")), beta=beta, alpha=alpha, chan=chan, bn=bn)


def _compare(got, ref, io, what, keys=GRADS):
    for k in keys:
        a = got[k].reshape(ref[k].shape)
        r = ref[k]
        if not np.any(r):                      # e.g. dv0 = beta P_0 with beta = 0
            assert not np.any(a), f"{what} {k}: expected exact zeros"
            continue
        if io == "f32":
            err = np.abs(a - r).max()
            assert err <= F32_TOL * np.abs(r).max(), f"{what} {k}: {err:.3g} vs max {np.abs(r).max():.3g}"
        else:
            rel = np.linalg.norm(a - r) / np.linalg.norm(r)
            assert rel <= BF16_TOL, f"{what} {k}: rel L2 {rel:.3g}"


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("beta,alpha", [(0.9, 1.0), (0.0, 1.0), (0.5, 2.0)])
def test_bwd_matches_oracle(io, beta, alpha):
    w = wl.SCAN_BF16 if io == "bf16" else wl.SCAN_MEDIUM
    inp, g = _problem(w, 2, 200, 70)            # ragged last chunk, a partial channel tile
    got, _ = _gpu(w, inp, g, beta, alpha)
    _compare(got, _ref(inp, g, beta, alpha), io, f"{io} beta={beta} alpha={alpha}")


@pytest.mark.parametrize("L", [1, 37, 64, 65, 129])
def test_bwd_lengths_and_row_fallback(L):
    # L = 37 fp32 rows are not whole 16-byte pieces: element-wise staging;
    # L = 1 needs no checkpoint; 65 has a one-step last chunk and block
    w = wl.SCAN_MEDIUM
    inp, g = _problem(w, 1, L, 24)
    got, _ = _gpu(w, inp, g, 0.8, 1.5)
    _compare(got, _ref(inp, g, 0.8, 1.5), "f32", f"L={L}")


@pytest.mark.parametrize("dstate", [1, 4, 8, 13])
def test_bwd_small_state_counts(dstate):
    w = wl.SCAN_MEDIUM
    inp, g = _problem(w, 2, 150, 20, dstate=dstate)
    got, _ = _gpu(w, inp, g, 0.9, 1.0)
    _compare(got, _ref(inp, g, 0.9, 1.0), "f32", f"N={dstate}")


def test_bwd_without_initial_state_or_final_gradients():
    w = wl.SCAN_MEDIUM
    inp, g = _problem(w, 2, 300, 40, h0v0=False)
    got, _ = _gpu(w, inp, g, 0.95, 1.0)
    _compare(got, _ref(inp, g, 0.95, 1.0), "f32", "no h0/v0/dhT/dvT")


def test_checkpoints_are_the_states_after_each_chunk():
    w = wl.SCAN_MEDIUM
    inp, g = _problem(w, 2, 200, 24)
    _, (y, hT, vT, ckpt) = _gpu(w, inp, g, 0.9, 1.0)
    ck = ckpt.cpu().numpy()                     # (batch, dim, 13, 2, N)
    assert ck.shape == (2, 24, 13, 2, 16)
    for k, end in enumerate(list(range(16, 200, 16)) + [200]):
        sub = {key: inp[key][..., :end] for key in ("x", "delta", "B", "C")}
        _, hr, vr = oracle.scan_seq(sub["x"], sub["delta"], inp["A"], sub["B"], sub["C"],
                                    h0=inp["h0"].astype(np.float64), v0=inp["v0"].astype(np.float64),
                                    beta=0.9, alpha=1.0)
        h = ck[:, :, k, 0, :].reshape(hr.shape)
        v = ck[:, :, k, 1, :].reshape(vr.shape)
        assert np.abs(h - hr).max() <= F32_TOL * np.abs(hr).max(), f"h after chunk {k}"
        assert np.abs(v - vr).max() <= F32_TOL * np.abs(vr).max(), f"v after chunk {k}"
    # the last checkpoint is the final state itself, and keeping checkpoints changes nothing
    assert np.array_equal(ck[:, :, -1, 0, :], hT.cpu().numpy())
    assert np.array_equal(ck[:, :, -1, 1, :], vT.cpu().numpy())
    # (the forward that keeps checkpoints is the register-resident kernel; compare with that path)
    dev = {k: _t(inp[k]) for k in ("x", "delta", "A", "B", "C", "h0", "v0")}
    mm.mm_scan_set_path(1, 0)
    try:
        y2, h2, v2 = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=dev["h0"],
                                 v0=dev["v0"], beta=0.9, alpha=1.0)
    finally:
        mm.mm_scan_set_path(0, 0)
    assert torch.equal(y2, y) and torch.equal(h2, hT) and torch.equal(v2, vT)


def test_bwd_split_sequence_chain_rule():
    """Backward of the second half, then of the first half fed with the second's
    dh0, dv0: dx, ddelta, dh0, dv0 bit-identical to one call; sums close."""
    w = wl.SCAN_MEDIUM
    L, half = 384, 192
    inp, g = _problem(w, 2, L, 40)
    dev = {k: _t(inp[k]) for k in ("x", "delta", "A", "B", "C", "h0", "v0")}
    dy, dhT, dvT = _t(g["dy"]), _t(g["dhT"]), _t(g["dvT"])
    kw = dict(beta=0.97, alpha=1.0)
    _, _, _, ck = mm.scan_fwd_train(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=dev["h0"],
                                    v0=dev["v0"], **kw)
    whole = mm.scan_bwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], ck, dy, h0=dev["h0"],
                        v0=dev["v0"], dhT=dhT, dvT=dvT, **kw)
    sl = lambda a, lo, hi: a[..., lo:hi].contiguous()
    parts = [{k: sl(dev[k], lo, hi) for k in ("x", "delta", "B", "C")} for lo, hi in ((0, half), (half, L))]
    _, h1, v1, ck1 = mm.scan_fwd_train(parts[0]["x"], parts[0]["delta"], dev["A"], parts[0]["B"],
                                       parts[0]["C"], h0=dev["h0"], v0=dev["v0"], **kw)
    _, _, _, ck2 = mm.scan_fwd_train(parts[1]["x"], parts[1]["delta"], dev["A"], parts[1]["B"],
                                     parts[1]["C"], h0=h1, v0=v1, **kw)
    g2 = mm.scan_bwd(parts[1]["x"], parts[1]["delta"], dev["A"], parts[1]["B"], parts[1]["C"], ck2,
                     sl(dy, half, L), h0=h1, v0=v1, dhT=dhT, dvT=dvT, **kw)
    g1 = mm.scan_bwd(parts[0]["x"], parts[0]["delta"], dev["A"], parts[0]["B"], parts[0]["C"], ck1,
                     sl(dy, 0, half), h0=dev["h0"], v0=dev["v0"], dhT=g2["dh0"], dvT=g2["dv0"], **kw)
    torch.cuda.synchronize()
    for k in ("dx", "ddelta"):
        assert torch.equal(torch.cat([g1[k], g2[k]], dim=-1), whole[k]), k
    assert torch.equal(g1["dh0"], whole["dh0"]) and torch.equal(g1["dv0"], whole["dv0"])
    for k in ("dB", "dC"):
        joined = torch.cat([g1[k], g2[k]], dim=-1)
        assert torch.allclose(joined, whole[k], rtol=0, atol=1e-5 * float(whole[k].abs().max())), k
    assert torch.allclose(g1["dA"] + g2["dA"], whole["dA"], rtol=0, atol=1e-5 * float(whole["dA"].abs().max()))


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_bwd_full_size_sampled(io):
    """The bench workloads at full size, in the launch the bench times;
    sampled channels (all batch rows of the sampled d, for dA) and (b, n) rows."""
    w = wl.SCAN_BF16 if io == "bf16" else wl.SCAN_MEDIUM
    inp, g = _problem(w, w.batch, w.seqlen, w.dim, h0v0=False)
    got, _ = _gpu(w, inp, g, 0.9, 1.0)
    rng = np.random.default_rng(1)
    ds = np.unique(np.concatenate([rng.choice(w.dim, 6, replace=False), [0, w.dim - 1]]))
    chan = np.array([b * w.dim + d for b in range(w.batch) for d in ds], np.int64)
    bn = np.array([0, 5, 16 * (w.batch - 1) + 15], np.int64)
    ref = _ref(inp, g, 0.9, 1.0, chan=chan, bn=bn)
    sub = {"dx": got["dx"].reshape(-1, w.seqlen)[chan], "ddelta": got["ddelta"].reshape(-1, w.seqlen)[chan],
           "dh0": got["dh0"].reshape(-1, 16)[chan], "dv0": got["dv0"].reshape(-1, 16)[chan],
           "dA": got["dA"][ds], "dB": got["dB"].reshape(-1, w.seqlen)[bn],
           "dC": got["dC"].reshape(-1, w.seqlen)[bn]}
    ref = dict(ref, dA=ref["dA"][ds])
    _compare(sub, ref, io, f"full {io}")


GATED = [  # D, z, bias, softplus
    (True, False, False, False), (False, True, False, False), (False, False, True, False),
    (False, False, False, True), (False, False, True, True), (True, True, True, True),
]


def _gated(w, batch, L, dim, use_D, use_z, use_bias, softplus, beta=0.9, alpha=1.0, dstate=16):
    inp, g = _problem(w, batch, L, dim, dstate=dstate)
    ex = wl.scan_extras(w, batch=batch, seqlen=L, dim=dim)
    if softplus:
        inp["delta"] = ex["delta_raw"]
        bias = ex["delta_bias"] if use_bias else None
    else:
        bias = np.linspace(1e-3, 5e-2, dim, dtype=np.float32) if use_bias else None
    D = ex["D"] if use_D else None
    z = ex["z"] if use_z else None
    io = torch.float32 if w.io == "f32" else torch.bfloat16
    dev = {k: _t(inp[k], io) for k in ("x", "delta", "B", "C")}
    A, h0, v0 = _t(inp["A"]), _t(inp["h0"]), _t(inp["v0"])
    kw = dict(D=_t(D), z=_t(z, io), delta_bias=_t(bias), delta_softplus=softplus)
    _, _, _, ckpt = mm.scan_fwd_train(dev["x"], dev["delta"], A, dev["B"], dev["C"], h0=h0, v0=v0,
                                      beta=beta, alpha=alpha, **kw)
    gr = mm.scan_bwd(dev["x"], dev["delta"], A, dev["B"], dev["C"], ckpt, _t(g["dy"], io), h0=h0, v0=v0,
                     dhT=_t(g["dhT"]), dvT=_t(g["dvT"]), beta=beta, alpha=alpha, **kw)
    torch.cuda.synchronize()
    mm.mm_device_status()
    got = {k: v.float().cpu().numpy() for k, v in gr.items() if v is not None}
    f64 = lambda a: np.asarray(a, np.float64)
    ref = oracle.scan_bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], g["dy"], D=D, z=z,
                          delta_bias=bias, delta_softplus=softplus, h0=f64(inp["h0"]), v0=f64(inp["v0"]),
                          dhT=f64(g["dhT"]), dvT=f64(g["dvT"]), beta=beta, alpha=alpha)
    keys = GRADS + ("dD", "ddelta_bias") + (("dz",) if use_z else ())
    _compare(got, ref, w.io, f"{w.io} D={use_D} z={use_z} bias={use_bias} softplus={softplus}", keys)


@pytest.mark.parametrize("combo", GATED, ids=lambda c: "".join("DzbS"[i] if f else "-" for i, f in enumerate(c)))
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_gated_bwd_matches_oracle(io, combo):
    w = wl.SCAN_BF16 if io == "bf16" else wl.SCAN_MEDIUM
    _gated(w, 2, 200, 70, *combo)


@pytest.mark.parametrize("L", [1, 37, 65])
def test_gated_bwd_lengths_and_row_fallback(L):
    _gated(wl.SCAN_MEDIUM, 1, L, 24, True, True, True, True, beta=0.5, alpha=2.0)


@pytest.mark.parametrize("dstate", [4, 13])
def test_gated_bwd_state_counts(dstate):
    _gated(wl.SCAN_MEDIUM, 2, 100, 20, True, True, True, True, dstate=dstate)
