"""Pins of the oracle's full selective_scan_fn forward (oracle.scan_gated):
delta bias and softplus, the D skip and the SiLU gate.

The pages give these arguments ("selective_scan_fn" in the Momentum Mamba
README) and the gate's place after the scan ("Mamba: Choosing What to
Remember Based on the Input", "Where the state computation sits in a Mamba
block") but no formulas; the readings are delta' = softplus(delta + bias),
out = (y + D x) * silu(z).  What pins them, independently of that formula:

* with no extra argument the result is the plain scan, bit for bit;
* the pages' worked examples (Figures 2 and 5) reached through the bias and
  the softplus: bias = ln(e^Delta - 1) turns a stored delta of 0 into Delta;
* softplus(0) = ln 2, so with A = -1 a state of 2 is retained as exactly 1;
* delta + bias against numpy's logaddexp on random values;
* C = 0 leaves out = D x exactly; z = 0 gives out = 0 exactly; z = 1 scales
  by sigma(1) = e / (1 + e) and z = 2 by 2 e^2 / (1 + e^2); the skip enters
  before the gate.
"""
import math

import numpy as np
import pytest

import oracle
from selective_state_space_momentum_b200 import workloads as wl
from tests.test_oracle_pins import _golden, _num

SIGMA1 = math.e / (1.0 + math.e)
SILU2 = 2.0 * math.exp(2.0) / (1.0 + math.exp(2.0))


def _one_step_gated(h_prev, A, delta, B, u, C, delta_bias=None, softplus=False, D=None, z=None,
                    beta=0.0, alpha=1.0, lib=None):
    N = len(A)
    x = np.array([[[u]]], np.float32)
    d = np.array([[[delta]]], np.float32)
    Am = np.array([A], np.float32)
    Bm = np.array(B, np.float32).reshape(1, N, 1)
    Cm = np.array(C, np.float32).reshape(1, N, 1)
    h0 = np.array(h_prev, np.float64).reshape(1, 1, N)
    bias = None if delta_bias is None else np.array([delta_bias], np.float32)
    Dv = None if D is None else np.array([D], np.float32)
    zz = None if z is None else np.array([[[z]]], np.float32)
    y, hT, vT = oracle.scan_gated(x, d, Am, Bm, Cm, D=Dv, z=zz, delta_bias=bias,
                                  delta_softplus=softplus, h0=h0, beta=beta, alpha=alpha, lib=lib)
    return y[0, 0], hT[0], vT[0]


def test_no_extras_is_the_plain_scan_bit_for_bit():
    inp = wl.scan_inputs(wl.SCAN_SMALL, dim=12, seqlen=70)
    rng = np.random.default_rng(1)
    h0 = rng.standard_normal((1, 12, 16))
    a = oracle.scan_seq(**inp, h0=h0, beta=0.7, alpha=1.3)
    b = oracle.scan_gated(**inp, h0=h0, beta=0.7, alpha=1.3)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


@pytest.mark.parametrize("softplus", [False, True])
def test_fig2_through_the_bias(softplus):
    """Figure 2 with the step size supplied as stored delta + bias."""
    g = _golden()["selective_fig2"]
    A = _num(g["A"])
    for case in g["cases"]:
        Delta = case["delta"]
        if softplus:
            delta, bias = 0.0, math.log(math.expm1(Delta))     # softplus(bias) = Delta
        else:
            delta, bias = 0.25 * Delta, 0.75 * Delta           # exact in fp32
        y, h, _ = _one_step_gated([g["h_prev"]], [A], delta, [g["B"]], g["u"], [g["C"]],
                                  delta_bias=bias, softplus=softplus)
        assert h[0] == pytest.approx(case["new_state_derived"], rel=1e-6)
        assert y == pytest.approx(case["new_state_derived"], rel=1e-6)


def test_fig5_through_softplus():
    g = _golden()["selective_fig5"]
    A = [_num(a) for a in g["A"]]
    for case in g["cases"]:
        bias = math.log(math.expm1(case["delta"]))
        y, h, _ = _one_step_gated(g["h_prev"], A, 0.0, case["B"], g["u"], case["C"],
                                  delta_bias=bias, softplus=True)
        np.testing.assert_allclose(h, case["new_state"], rtol=1e-6)
        assert y == pytest.approx(case["y"], rel=1e-6)


def test_softplus_of_zero_is_ln2():
    # delta' = ln 2, A = -1: the state 2 is retained as 2 * exp(-ln 2) = 1
    _, h, _ = _one_step_gated([2.0], [-1.0], 0.0, [1.0], 0.0, [1.0], softplus=True)
    assert h[0] == pytest.approx(1.0, rel=1e-15)


def test_softplus_with_bias_matches_logaddexp():
    inp = wl.scan_inputs(wl.SCAN_SMALL, dim=6, seqlen=40)
    rng = np.random.default_rng(2)
    raw = rng.normal(-2.0, 2.0, inp["delta"].shape).astype(np.float32)   # any sign
    bias = rng.normal(0.0, 1.0, 6).astype(np.float32)
    got = oracle.scan_gated(inp["x"], raw, inp["A"], inp["B"], inp["C"], delta_bias=bias,
                            delta_softplus=True, beta=0.8, alpha=1.0)
    dprime = np.logaddexp(0.0, raw.astype(np.float64) + bias.astype(np.float64)[None, :, None])
    ref = oracle.scan_seq(inp["x"], dprime.astype(np.float32), inp["A"], inp["B"], inp["C"],
                          beta=0.8, alpha=1.0)
    for u, v in zip(got, ref):       # only the fp32 rounding of delta' separates them
        np.testing.assert_allclose(u, v, rtol=2e-6, atol=2e-6 * float(np.abs(v).max()))


def test_skip_is_D_times_x_when_C_is_zero():
    inp = wl.scan_inputs(wl.SCAN_SMALL, dim=5, seqlen=33)
    inp["C"] = np.zeros_like(inp["C"])
    D = np.array([0.5, -1.25, 2.0, 0.0, 3.0], np.float32)
    y, _, _ = oracle.scan_gated(**inp, D=D, beta=0.9, alpha=1.0)
    ref = (D.astype(np.float64)[None, :, None] * inp["x"].astype(np.float64)).reshape(-1, 33)
    assert np.array_equal(y, ref)


def test_gate_zero_one_and_order():
    inp = wl.scan_inputs(wl.SCAN_SMALL, dim=4, seqlen=25)
    D = np.array([0.3, -0.7, 1.1, 2.0], np.float32)
    base, _, _ = oracle.scan_gated(**inp, D=D, beta=0.5, alpha=1.0)
    zeros = np.zeros_like(inp["x"])
    y0, _, _ = oracle.scan_gated(**inp, D=D, z=zeros, beta=0.5, alpha=1.0)
    assert np.array_equal(y0, np.zeros_like(y0))                 # silu(0) = 0
    y1, h1, _ = oracle.scan_gated(**inp, D=D, z=np.ones_like(inp["x"]), beta=0.5, alpha=1.0)
    np.testing.assert_allclose(y1, base * SIGMA1, rtol=1e-13)     # silu(1) = sigma(1)
    # the skip enters before the gate: C = 0, D = 2, x = 3, z = 1 gives 6 sigma(1)
    y, _, _ = _one_step_gated([0.0], [-1.0], 0.1, [1.0], 3.0, [0.0], D=2.0, z=1.0)
    assert y == pytest.approx(6.0 * SIGMA1, rel=1e-14)
    # silu, not a plain sigmoid: z = 2 scales by 2 e^2 / (1 + e^2)
    y, _, _ = _one_step_gated([0.0], [-1.0], 0.1, [1.0], 3.0, [0.0], D=2.0, z=2.0)
    assert y == pytest.approx(6.0 * SILU2, rel=1e-14)
    # the gate leaves the states alone
    _, hr, vr = oracle.scan_seq(**inp, beta=0.5, alpha=1.0)
    assert np.array_equal(h1, hr)
