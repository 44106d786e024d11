"""Pins of the oracle's backward (oracle.scan_bwd) against its forward.

The pages print gradient formulas for the momentum scan ("Gradient Flow" and
"Backward Pass: Reconstructed Forward + Reverse Scans" in the Momentum Mamba
README) but use one symbol for both state gradients and leave a term out of
the velocity's recursion; the oracle derives the recursions from the forward
recurrence.  Nothing here retypes them.  What pins them:

* central finite differences of the pinned forward (oracle.scan_gated), in
  fp64, for every entry of every input: x, delta, A, B, C, D, z, delta_bias,
  h0, v0 (the loss is sum(dout*out) + sum(dhT*hT) + sum(dvT*vT));
* exact directional identities where the forward is affine in an input
  (x, B, C, D, h0, v0): J(u + s) - J(u) = <grad, s> to fp64 rounding;
* causality: a gradient arriving only at step s leaves every step after s
  with exactly zero gradient;
* the chain rule across a split sequence: the second half's dh0, dv0 fed as
  dhT, dvT to the first half reproduce the whole sequence's gradients;
* channel and (b, n) selection return the same rows as the full call.
"""
import numpy as np
import pytest

import oracle


def _problem(seed, batch=2, dim=3, L=10, N=4, gated=False, softplus=False, bias=False,
             h0v0=True):
    rng = np.random.default_rng(seed)
    p = {
        "x": rng.standard_normal((batch, dim, L)).astype(np.float32),
        "A": (-rng.uniform(0.5, 4.0, (dim, N))).astype(np.float32),
        "B": rng.standard_normal((batch, N, L)).astype(np.float32),
        "C": rng.standard_normal((batch, N, L)).astype(np.float32),
    }
    if softplus:
        p["delta"] = rng.normal(-1.0, 1.0, (batch, dim, L)).astype(np.float32)
    else:
        p["delta"] = np.exp(rng.uniform(np.log(0.02), np.log(0.4), (batch, dim, L))).astype(np.float32)
    if gated:
        p["D"] = rng.uniform(0.5, 1.5, dim).astype(np.float32)
        p["z"] = rng.standard_normal((batch, dim, L)).astype(np.float32)
    if bias:
        p["delta_bias"] = (rng.normal(0.0, 0.5, dim) if softplus
                           else rng.uniform(0.01, 0.1, dim)).astype(np.float32)
    if h0v0:
        p["h0"] = rng.standard_normal((batch, dim, N))
        p["v0"] = rng.standard_normal((batch, dim, N))
    seeds = {
        "dout": rng.standard_normal((batch, dim, L)).astype(np.float32),
        "dhT": rng.standard_normal((batch, dim, N)),
        "dvT": rng.standard_normal((batch, dim, N)),
    }
    return p, seeds


def _loss(p, g, beta, alpha, softplus):
    out, hT, vT = oracle.scan_gated(p["x"], p["delta"], p["A"], p["B"], p["C"], D=p.get("D"),
                                    z=p.get("z"), delta_bias=p.get("delta_bias"),
                                    delta_softplus=softplus, h0=p.get("h0"), v0=p.get("v0"),
                                    beta=beta, alpha=alpha)
    batch, dim, _ = p["x"].shape
    return (float(np.sum(g["dout"].astype(np.float64).reshape(out.shape) * out))
            + float(np.sum(g["dhT"].reshape(hT.shape) * hT))
            + float(np.sum(g["dvT"].reshape(vT.shape) * vT)))


def _grads(p, g, beta, alpha, softplus):
    return oracle.scan_bwd(p["x"], p["delta"], p["A"], p["B"], p["C"], g["dout"], D=p.get("D"),
                           z=p.get("z"), delta_bias=p.get("delta_bias"), delta_softplus=softplus,
                           h0=p.get("h0"), v0=p.get("v0"), dhT=g["dhT"], dvT=g["dvT"],
                           beta=beta, alpha=alpha)


# gradient name for each input; its array is reshaped to the input's shape
GRAD_OF = {"x": "dx", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
           "z": "dz", "delta_bias": "ddelta_bias", "h0": "dh0", "v0": "dv0"}
# relative central-difference step per input (third derivatives in delta,
# bias are ~|A|^3, so their step is small)
STEP = {"x": 1e-2, "delta": 2e-4, "A": 1e-3, "B": 1e-2, "C": 1e-2, "D": 1e-2, "z": 1e-3,
        "delta_bias": 2e-4, "h0": 1e-3, "v0": 1e-3}

CONFIGS = {
    "momentum_h0v0":  dict(kw=dict(), beta=0.9, alpha=1.3, softplus=False),
    "mamba_beta0":    dict(kw=dict(h0v0=False), beta=0.0, alpha=1.0, softplus=False),
    "gated_softplus": dict(kw=dict(gated=True, softplus=True, bias=True), beta=0.8, alpha=0.7,
                           softplus=True),
    "gated_bias":     dict(kw=dict(gated=True, bias=True), beta=0.5, alpha=2.0, softplus=False),
}


def fd_failures(cfg_name, lib=None, seed=3):
    """Inputs whose finite-difference gradient disagrees with scan_bwd."""
    cfg = CONFIGS[cfg_name]
    p, g = _problem(seed, **cfg["kw"])
    beta, alpha, sp = cfg["beta"], cfg["alpha"], cfg["softplus"]

    def loss(q):
        out, hT, vT = oracle.scan_gated(q["x"], q["delta"], q["A"], q["B"], q["C"], D=q.get("D"),
                                        z=q.get("z"), delta_bias=q.get("delta_bias"),
                                        delta_softplus=sp, h0=q.get("h0"), v0=q.get("v0"),
                                        beta=beta, alpha=alpha, lib=lib)
        return (float(np.sum(g["dout"].astype(np.float64).reshape(out.shape) * out))
                + float(np.sum(g["dhT"].reshape(hT.shape) * hT))
                + float(np.sum(g["dvT"].reshape(vT.shape) * vT)))

    gr = oracle.scan_bwd(p["x"], p["delta"], p["A"], p["B"], p["C"], g["dout"], D=p.get("D"),
                         z=p.get("z"), delta_bias=p.get("delta_bias"), delta_softplus=sp,
                         h0=p.get("h0"), v0=p.get("v0"), dhT=g["dhT"], dvT=g["dvT"],
                         beta=beta, alpha=alpha, lib=lib)
    bad = []
    for name, arr in p.items():
        ana = gr[GRAD_OF[name]].reshape(arr.shape)
        fd = np.empty(arr.shape)
        for i in np.ndindex(arr.shape):
            val = float(arr[i])
            e = STEP[name] * max(1.0, abs(val))
            q = dict(p)
            up, dn = arr.copy(), arr.copy()
            up[i] = val + e
            dn[i] = val - e
            step = float(up[i]) - float(dn[i])       # the step the dtype actually took
            q[name] = up
            jp = loss(q)
            q[name] = dn
            jm = loss(q)
            fd[i] = (jp - jm) / step
        scale = max(float(np.abs(fd).max()), 1e-12)
        if not np.abs(fd - ana).max() <= 1e-5 * scale:
            bad.append(name)
    return bad


@pytest.mark.parametrize("cfg", sorted(CONFIGS))
def test_finite_differences_every_input(cfg):
    assert fd_failures(cfg) == []


@pytest.mark.parametrize("name", ["x", "B", "C", "D", "h0", "v0"])
def test_affine_inputs_exact_directional(name):
    """out, hT, vT are affine in each of these: the difference is exact."""
    cfg = CONFIGS["gated_softplus"] if name == "D" else CONFIGS["momentum_h0v0"]
    p, g = _problem(11, **cfg["kw"])
    if name in ("h0", "v0") and name not in p:
        pytest.skip("no initial state in this configuration")
    beta, alpha, sp = cfg["beta"], cfg["alpha"], cfg["softplus"]
    gr = _grads(p, g, beta, alpha, sp)
    rng = np.random.default_rng(5)
    arr = p[name]
    moved = (arr + 0.3 * rng.standard_normal(arr.shape)).astype(arr.dtype)
    s = moved.astype(np.float64) - arr.astype(np.float64)
    j0 = _loss(p, g, beta, alpha, sp)
    q = dict(p)
    q[name] = moved
    j1 = _loss(q, g, beta, alpha, sp)
    pred = float(np.sum(gr[GRAD_OF[name]].reshape(arr.shape) * s))
    assert abs((j1 - j0) - pred) <= 1e-11 * (abs(j0) + abs(j1) + 1.0)


def test_causality_exact_zeros():
    p, g = _problem(7, gated=True, softplus=True, bias=True, L=16)
    s = 9
    g["dout"][:, :, s + 1:] = 0.0
    g["dhT"][:] = 0.0
    g["dvT"][:] = 0.0
    gr = _grads(p, g, 0.9, 1.0, True)
    for k in ("dx", "ddelta", "dz", "dB", "dC"):
        assert np.all(gr[k][:, s + 1:] == 0.0), k
        assert np.any(gr[k][:, s] != 0.0), k


def test_chain_rule_across_a_split():
    p, g = _problem(9, L=24)
    beta, alpha = 0.95, 1.1
    whole = _grads(p, g, beta, alpha, False)
    h = 13
    first = {k: (v[..., :h] if k in ("x", "delta", "B", "C") else v) for k, v in p.items()}
    first.pop("h0"), first.pop("v0")
    first["h0"], first["v0"] = p["h0"], p["v0"]
    _, h1, v1 = oracle.scan_gated(first["x"], first["delta"], p["A"], first["B"], first["C"],
                                  h0=p["h0"], v0=p["v0"], beta=beta, alpha=alpha)
    second = {k: (v[..., h:] if k in ("x", "delta", "B", "C") else v) for k, v in p.items()}
    second["h0"], second["v0"] = h1.reshape(p["h0"].shape), v1.reshape(p["v0"].shape)
    g2 = {"dout": g["dout"][..., h:], "dhT": g["dhT"], "dvT": g["dvT"]}
    gr2 = _grads(second, g2, beta, alpha, False)
    g1 = {"dout": g["dout"][..., :h], "dhT": gr2["dh0"].reshape(p["h0"].shape),
          "dvT": gr2["dv0"].reshape(p["v0"].shape)}
    gr1 = _grads(first, g1, beta, alpha, False)
    for k in ("dx", "ddelta", "dB", "dC"):
        joined = np.concatenate([gr1[k], gr2[k]], axis=1)
        np.testing.assert_allclose(joined, whole[k], rtol=1e-12, atol=1e-12 * np.abs(whole[k]).max())
    np.testing.assert_allclose(gr1["dA"] + gr2["dA"], whole["dA"], rtol=1e-11)
    for k in ("dh0", "dv0"):
        np.testing.assert_allclose(gr1[k], whole[k], rtol=1e-12, atol=1e-14)


def test_selection_rows_match_the_full_call():
    p, g = _problem(13, gated=True, softplus=True, bias=True, batch=3, dim=4)
    full = _grads(p, g, 0.9, 1.0, True)
    chan = np.array([0, 5, 11], np.int64)
    bn = np.array([1, 6, 11], np.int64)
    sub = oracle.scan_bwd(p["x"], p["delta"], p["A"], p["B"], p["C"], g["dout"], D=p["D"], z=p["z"],
                          delta_bias=p["delta_bias"], delta_softplus=True, h0=p["h0"], v0=p["v0"],
                          dhT=g["dhT"], dvT=g["dvT"], beta=0.9, alpha=1.0, chan=chan, bn=bn)
    for k in ("dx", "ddelta", "dz", "dh0", "dv0"):
        assert np.array_equal(sub[k], full[k][chan]), k
    for k in ("dB", "dC"):
        assert np.array_equal(sub[k], full[k][bn]), k
