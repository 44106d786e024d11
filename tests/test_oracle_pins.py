"""Pins for the fp64 oracle: values and identities fixed outside the oracle.

Each test checks the oracle against something other than itself: numbers the
pages print for a worked example (tests/golden/worked_examples.json), closed
forms of the recurrence, an FFT convolution (numpy), brute force through the
materialised lower-triangular matrix on tiny inputs, exact invariants of
linear recurrences, and the agreement of two independent routes (sequential
and chunked).  A plausible mistake in the oracle -- a dropped momentum term, a
read-out of the pre-update state, a wrong sign in the exponent, B and C
swapped, an off-by-one in a product -- fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from selective_state_space_momentum_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _num(v):
    if isinstance(v, str):
        if v.startswith("ln(") and v.endswith(")"):
            return math.log(float(v[3:-1]))
        raise ValueError(v)
    return float(v)


def _one_step(h_prev, A, delta, B, u, C, beta=0.0, alpha=1.0, v_prev=None):
    """Run the oracle for one time step of one channel with N = len(A)."""
    N = len(A)
    x = np.array([[[u]]], np.float32)
    d = np.array([[[delta]]], np.float32)
    Am = np.array([A], np.float32)
    Bm = np.array(B, np.float32).reshape(1, N, 1)
    Cm = np.array(C, np.float32).reshape(1, N, 1)
    h0 = np.array(h_prev, np.float64).reshape(1, 1, N)
    v0 = None if v_prev is None else np.array(v_prev, np.float64).reshape(1, 1, N)
    y, hT, vT = oracle.scan_seq(x, d, Am, Bm, Cm, h0=h0, v0=v0, beta=beta, alpha=alpha)
    return y[0, 0], hT[0], vT[0]


# ----------------------------------------------------- worked examples -----
@pytest.mark.parametrize("beta", [0.0, 0.5, 0.9])
def test_selective_fig2_retained_and_written(beta):
    """Figure 2 of 'Mamba: Choosing What to Remember Based on the Input'.

    With a zero initial velocity the first step writes alpha*delta*B*x
    whatever beta is, so the example pins every beta.
    """
    g = _golden()["selective_fig2"]
    A = _num(g["A"])
    for case in g["cases"]:
        # retained part alone: no input
        _, h, _ = _one_step([g["h_prev"]], [A], case["delta"], [g["B"]], 0.0, [g["C"]], beta)
        assert h[0] == pytest.approx(case["retained"], rel=1e-6)
        # written part alone: empty state
        _, h, _ = _one_step([0.0], [A], case["delta"], [g["B"]], g["u"], [g["C"]], beta)
        assert h[0] == pytest.approx(case["write"], rel=1e-6)
        # both, and the read-out of the updated state (C = 1)
        y, h, _ = _one_step([g["h_prev"]], [A], case["delta"], [g["B"]], g["u"], [g["C"]], beta)
        assert h[0] == pytest.approx(case["new_state_derived"], rel=1e-6)
        assert y == pytest.approx(case["new_state_derived"], rel=1e-6)


def test_selective_fig5_two_updates():
    """Figure 5: N = 2, the read-out C . h of the updated state."""
    g = _golden()["selective_fig5"]
    A = [_num(a) for a in g["A"]]
    for case in g["cases"]:
        _, h, _ = _one_step(g["h_prev"], A, case["delta"], case["B"], 0.0, case["C"])
        np.testing.assert_allclose(h, case["retained"], rtol=1e-6)
        _, h, _ = _one_step([0.0, 0.0], A, case["delta"], case["B"], g["u"], case["C"])
        np.testing.assert_allclose(h, case["write"], rtol=1e-6)
        y, h, _ = _one_step(g["h_prev"], A, case["delta"], case["B"], g["u"], case["C"])
        np.testing.assert_allclose(h, case["new_state"], rtol=1e-6)
        assert y == pytest.approx(case["y"], rel=1e-6)


def test_glossary_retention_table_via_prescaled_B():
    """SelfMadeQuant glossary table (zero-order hold of dh/dtau = -h + x).

    Pre-scaling B to (1 - exp(-delta)) / delta makes the first-order write
    delta*B*x equal to the zero-order-hold write, so the table's new states
    must come out of the oracle.
    """
    g = _golden()["glossary_retention_table"]
    for case in g["cases"]:
        delta = np.float32(_num(case["delta"]))
        Bpre = (1.0 - math.exp(-float(delta))) / float(delta)
        y, h, _ = _one_step([g["h_prev"]], [g["A"]], float(delta), [Bpre], g["x"], [1.0])
        assert h[0] == pytest.approx(case["new_state"], rel=1e-6)
        _, hr, _ = _one_step([g["h_prev"]], [g["A"]], float(delta), [Bpre], 0.0, [1.0])
        assert hr[0] == pytest.approx(case["old_weight"], rel=1e-6)


# -------------------------------------------------------- closed forms -----
def _constant_run(L, delta, A, B, C, xval, beta, alpha):
    N = len(A)
    x = np.full((1, 1, L), xval, np.float32)
    d = np.full((1, 1, L), delta, np.float32)
    Am = np.array([A], np.float32)
    Bm = np.repeat(np.array(B, np.float32).reshape(1, N, 1), L, axis=2)
    Cm = np.repeat(np.array(C, np.float32).reshape(1, N, 1), L, axis=2)
    return oracle.scan_seq(x, d, Am, Bm, Cm, beta=beta, alpha=alpha)


@pytest.mark.parametrize("beta", [0.0, 0.3, 0.9, 0.99])
def test_closed_form_geometric_sum(beta):
    """Constant delta, B, x from a zero state: a sum of two geometric series.

    v_t = w (1 - beta^t) / (1 - beta) and
    h_t = w/(1-beta) * [(1 - a^t)/(1 - a) - beta (a^t - beta^t)/(a - beta)].
    """
    L = 300
    delta, A, B, C, xval, alpha = 0.05, [-1.0, -3.0], [0.7, -1.3], [1.5, 0.25], 0.8, 1.7
    y, hT, vT = _constant_run(L, delta, A, B, C, xval, beta, alpha)
    d32 = float(np.float32(delta))
    t = np.arange(1, L + 1, dtype=np.float64)
    yref = np.zeros(L)
    for n in range(2):
        a = math.exp(d32 * float(np.float32(A[n])))
        w = alpha * d32 * float(np.float32(B[n])) * float(np.float32(xval))
        geo_a = (1.0 - a ** t) / (1.0 - a)
        cross = beta * (a ** t - beta ** t) / (a - beta)
        h = w / (1.0 - beta) * (geo_a - cross)
        yref += float(np.float32(C[n])) * h
        if n == 0:
            np.testing.assert_allclose(vT[0, 0], w * (1 - beta ** L) / (1 - beta), rtol=1e-12)
            # special cases: h_1 = w, h_2 = w (1 + a + beta)
            assert h[0] == pytest.approx(w, rel=1e-14)
            assert h[1] == pytest.approx(w * (1 + a + beta), rel=1e-13)
    np.testing.assert_allclose(y[0], yref, rtol=1e-10, atol=1e-12)


def test_closed_form_steady_state():
    """Long constant drive: h tends to w / ((1 - beta)(1 - a))."""
    beta, delta, A, B, xval = 0.9, 0.1, [-2.0], [1.0], 1.0
    y, hT, _ = _constant_run(4000, delta, A, B, [1.0], xval, beta, 1.0)
    a = math.exp(float(np.float32(delta)) * -2.0)
    w = float(np.float32(delta))
    assert hT[0, 0] == pytest.approx(w / ((1 - beta) * (1 - a)), rel=1e-12)


@pytest.mark.parametrize("beta", [0.0, 0.6])
def test_lti_convolution_by_fft(beta):
    """Time-invariant coefficients: the scan is a causal convolution.

    complextorch 'State-space models', 'The diagonal SSM': with fixed
    coefficients the recurrence equals a convolution with the kernel
    K_l = sum_n C_n * Abar_n^l * Bbar_n.  With momentum the impulse response
    becomes K_l = sum_n C_n * alpha*delta*B_n * (a_n^(l+1) - beta^(l+1)) /
    (a_n - beta).  The convolution is done with numpy's FFT.
    """
    rng = np.random.default_rng(7)
    L, N, alpha = 512, 4, 1.3
    delta = np.float32(0.03)
    A = (-(np.arange(N) + 1.0)).astype(np.float32)
    B = rng.standard_normal(N).astype(np.float32)
    C = rng.standard_normal(N).astype(np.float32)
    x = rng.standard_normal((1, 1, L)).astype(np.float32)
    y, _, _ = oracle.scan_seq(x, np.full((1, 1, L), delta, np.float32), A[None, :],
                              np.repeat(B.reshape(1, N, 1), L, 2), np.repeat(C.reshape(1, N, 1), L, 2),
                              beta=beta, alpha=alpha)
    ell = np.arange(L, dtype=np.float64)
    K = np.zeros(L)
    for n in range(N):
        a = math.exp(float(delta) * float(A[n]))
        K += float(C[n]) * alpha * float(delta) * float(B[n]) * (a ** (ell + 1) - beta ** (ell + 1)) / (a - beta)
    nfft = 2 * L
    conv = np.fft.irfft(np.fft.rfft(x[0, 0].astype(np.float64), nfft) * np.fft.rfft(K, nfft), nfft)[:L]
    np.testing.assert_allclose(y[0], conv, rtol=1e-9, atol=1e-11)


# ------------------------------------------------ brute-force matrices -----
def _brute_force_scan(x, delta, A, B, C, h0, v0, beta, alpha):
    """y through the materialised lower-triangular operator, explicit products.

    For beta = 0 the weight of input j in output i is the Mamba-2 page's
    L_ij = C_i . (Abar_i ... Abar_{j+1}) . Bbar_j.  With momentum, input j
    enters the velocity at step j and reaches the state at step k >= j with
    weight beta^(k-j), then decays by Abar_{k+1} ... Abar_i.
    """
    Bsz, D, L = x.shape
    N = A.shape[1]
    y = np.zeros((Bsz, D, L))
    for b in range(Bsz):
        for d in range(D):
            a = np.exp(delta[b, d].astype(np.float64)[None, :] * A[d].astype(np.float64)[:, None])  # (N, L)
            w = alpha * delta[b, d].astype(np.float64)[None, :] * B[b].astype(np.float64) * x[b, d].astype(np.float64)[None, :]
            for i in range(L):
                for n in range(N):
                    tot = 0.0
                    for j in range(i + 1):
                        m = 0.0
                        for k in range(j, i + 1):
                            m += np.prod(a[n, k + 1:i + 1]) * beta ** (k - j)
                        tot += m * w[n, j]
                    # initial state: h0 decays through every step, v0 enters as beta^(k+1)
                    tot += np.prod(a[n, 0:i + 1]) * h0[b, d, n]
                    vin = 0.0
                    for k in range(0, i + 1):
                        vin += np.prod(a[n, k + 1:i + 1]) * beta ** (k + 1)
                    tot += vin * v0[b, d, n]
                    y[b, d, i] += float(C[b, n, i]) * tot
    return y


@pytest.mark.parametrize("beta,alpha", [(0.0, 1.0), (0.7, 1.0), (0.45, 2.5)])
def test_brute_force_lower_triangular_matrix(beta, alpha):
    rng = np.random.default_rng(11)
    Bsz, D, L, N = 2, 2, 13, 3
    x = rng.standard_normal((Bsz, D, L)).astype(np.float32)
    delta = np.exp(rng.uniform(np.log(1e-2), np.log(0.5), (Bsz, D, L))).astype(np.float32)
    A = (-rng.uniform(0.5, 3.0, (D, N))).astype(np.float32)
    B = rng.standard_normal((Bsz, N, L)).astype(np.float32)
    C = rng.standard_normal((Bsz, N, L)).astype(np.float32)
    h0 = rng.standard_normal((Bsz, D, N))
    v0 = rng.standard_normal((Bsz, D, N))
    y, _, _ = oracle.scan_seq(x, delta, A, B, C, h0=h0, v0=v0, beta=beta, alpha=alpha)
    yref = _brute_force_scan(x, delta, A, B, C, h0, v0, beta, alpha)
    np.testing.assert_allclose(y.reshape(Bsz, D, L), yref, rtol=1e-11, atol=1e-12)


# ---------------------------------------------- two independent routes -----
@pytest.mark.parametrize("chunk", [1, 7, 64, 100, 1000])
def test_chunked_equals_sequential(chunk):
    w = wl.SCAN_SMALL
    inp = wl.scan_inputs(w, batch=2, seqlen=300, dim=5, dstate=16)
    rng = np.random.default_rng(3)
    h0 = rng.standard_normal((2, 5, 16))
    v0 = rng.standard_normal((2, 5, 16))
    for beta, alpha in [(0.0, 1.0), (0.9, 1.0), (0.99, 0.5)]:
        ys, hs, vs = oracle.scan_seq(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha)
        yc, hc, vc = oracle.scan_chunked(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha, chunk=chunk)
        scale = np.abs(ys).max()
        np.testing.assert_allclose(yc, ys, rtol=0, atol=1e-12 * scale)
        np.testing.assert_allclose(hc, hs, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(vc, vs, rtol=1e-12, atol=1e-14)


def test_streaming_split_is_bitwise_identical():
    """One call over L equals two calls carrying (hT, vT) into (h0, v0)."""
    inp = wl.scan_inputs(wl.SCAN_LONG, seqlen=1024, dim=6)
    y, hT, vT = oracle.scan_seq(**inp, beta=0.99, alpha=1.0)
    half = {k: (np.ascontiguousarray(v[..., :512]) if k in ("x", "delta", "B", "C") else v)
            for k, v in inp.items()}
    rest = {k: (np.ascontiguousarray(v[..., 512:]) if k in ("x", "delta", "B", "C") else v)
            for k, v in inp.items()}
    y1, h1, v1 = oracle.scan_seq(**half, beta=0.99, alpha=1.0)
    y2, h2, v2 = oracle.scan_seq(**rest, h0=h1.reshape(1, 6, 16), v0=v1.reshape(1, 6, 16),
                                 beta=0.99, alpha=1.0)
    assert np.array_equal(np.concatenate([y1, y2], axis=1), y)
    assert np.array_equal(h2, hT) and np.array_equal(v2, vT)


# ------------------------------------------------------------ invariants -----
def _rand_inputs(seed=5, Bsz=2, D=3, L=64, N=8):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((Bsz, D, L)).astype(np.float32),
        delta=np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), (Bsz, D, L))).astype(np.float32),
        A=(-(np.arange(N) + 1.0) * rng.uniform(0.5, 2.0, (D, 1))).astype(np.float32),
        B=rng.standard_normal((Bsz, N, L)).astype(np.float32),
        C=rng.standard_normal((Bsz, N, L)).astype(np.float32)), rng


def test_alpha_zero_gives_zero_output():
    inp, _ = _rand_inputs()
    y, hT, vT = oracle.scan_seq(**inp, beta=0.9, alpha=0.0)
    assert not y.any() and not hT.any() and not vT.any()


def test_power_of_two_scaling_is_exact():
    inp, rng = _rand_inputs()
    h0 = rng.standard_normal((2, 3, 8))
    v0 = rng.standard_normal((2, 3, 8))
    y, hT, vT = oracle.scan_seq(**inp, h0=h0, v0=v0, beta=0.8, alpha=1.5)
    inp2 = dict(inp, x=inp["x"] * np.float32(4.0))
    y2, hT2, vT2 = oracle.scan_seq(**inp2, h0=4 * h0, v0=4 * v0, beta=0.8, alpha=1.5)
    assert np.array_equal(y2, 4 * y) and np.array_equal(hT2, 4 * hT) and np.array_equal(vT2, 4 * vT)


def test_superposition_of_input_and_initial_state():
    inp, rng = _rand_inputs()
    h0 = rng.standard_normal((2, 3, 8))
    v0 = rng.standard_normal((2, 3, 8))
    y, _, _ = oracle.scan_seq(**inp, h0=h0, v0=v0, beta=0.7, alpha=1.0)
    y_in, _, _ = oracle.scan_seq(**inp, beta=0.7, alpha=1.0)
    y_st, _, _ = oracle.scan_seq(**dict(inp, x=np.zeros_like(inp["x"])), h0=h0, v0=v0,
                                 beta=0.7, alpha=1.0)
    np.testing.assert_allclose(y, y_in + y_st, rtol=1e-12, atol=1e-13)


def test_causality():
    inp, _ = _rand_inputs()
    y, _, _ = oracle.scan_seq(**inp, beta=0.9, alpha=1.0)
    k = 40
    x2 = inp["x"].copy()
    x2[:, :, k] += 3.0
    y2, _, _ = oracle.scan_seq(**dict(inp, x=x2), beta=0.9, alpha=1.0)
    assert np.array_equal(y2[:, :k], y[:, :k])
    assert not np.array_equal(y2[:, k], y[:, k])


def test_additivity_over_states():
    inp, _ = _rand_inputs()
    y, _, _ = oracle.scan_seq(**inp, beta=0.5, alpha=1.0)
    acc = np.zeros_like(y)
    for n in range(8):
        sub = dict(inp, A=np.ascontiguousarray(inp["A"][:, n:n + 1]),
                   B=np.ascontiguousarray(inp["B"][:, n:n + 1]),
                   C=np.ascontiguousarray(inp["C"][:, n:n + 1]))
        yn, _, _ = oracle.scan_seq(**sub, beta=0.5, alpha=1.0)
        acc += yn
    np.testing.assert_allclose(acc, y, rtol=1e-12, atol=1e-13)


def test_channel_selection_matches_full_run():
    inp, _ = _rand_inputs()
    y, hT, vT = oracle.scan_seq(**inp, beta=0.9, alpha=1.0)
    sel = np.array([5, 0, 3])
    ys, hs, vs = oracle.scan_seq(**inp, beta=0.9, alpha=1.0, chan=sel)
    assert np.array_equal(ys, y[sel]) and np.array_equal(hs, hT[sel]) and np.array_equal(vs, vT[sel])


# ----------------------------------- the README's edge-case list -----------
def test_edge_tiny_beta_close_to_plain_mamba():
    inp, _ = _rand_inputs()
    y0, _, _ = oracle.scan_seq(**inp, beta=0.0, alpha=1.0)
    y1, _, _ = oracle.scan_seq(**inp, beta=1e-6, alpha=1.0)
    assert 0 < np.abs(y1 - y0).max() <= 1e-4 * np.abs(y0).max()


def test_edge_large_beta_and_alpha_linear():
    inp, _ = _rand_inputs()
    y1, _, _ = oracle.scan_seq(**inp, beta=0.999, alpha=1.0)
    y10, _, _ = oracle.scan_seq(**inp, beta=0.999, alpha=10.0)
    assert np.isfinite(y1).all()
    np.testing.assert_allclose(y10, 10.0 * y1, rtol=1e-12, atol=1e-12)


def test_edge_single_step_sequence_and_large_batch():
    inp, _ = _rand_inputs(Bsz=32, D=2, L=1, N=4)
    y, hT, vT = oracle.scan_seq(**inp, beta=0.9, alpha=1.0)
    # one step from a zero state: h = v = alpha*delta*B*x, y = C . h
    w = (inp["delta"][:, :, 0].astype(np.float64)[:, :, None] * inp["B"][:, None, :, 0]
         * inp["x"][:, :, 0].astype(np.float64)[:, :, None])
    np.testing.assert_allclose(hT.reshape(32, 2, 4), w, rtol=1e-15)
    # every batch row on its own gives the same numbers
    for b in (0, 17, 31):
        sub = {k: (np.ascontiguousarray(v[b:b + 1]) if k != "A" else v) for k, v in inp.items()}
        yb, _, _ = oracle.scan_seq(**sub, beta=0.9, alpha=1.0)
        assert np.array_equal(yb, y[2 * b:2 * b + 2])


# --------------------------------------------------------------- SSD -------
def _ssd_small(seed=9, Bsz=2, L=50, H=4, P=3, N=5, G=2):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((Bsz, L, H, P)).astype(np.float32),
        delta=np.exp(rng.uniform(np.log(1e-2), np.log(0.3), (Bsz, L, H))).astype(np.float32),
        A=(-rng.uniform(1.0, 16.0, H)).astype(np.float32),
        B=rng.standard_normal((Bsz, L, G, N)).astype(np.float32),
        C=rng.standard_normal((Bsz, L, G, N)).astype(np.float32)), rng


def test_ssd_reduces_to_the_mamba1_scan():
    """Each (head, head-channel) lane is a Mamba-1 channel with A[., n] = A_h."""
    inp, rng = _ssd_small()
    Bsz, L, H, P = inp["x"].shape
    G, N = inp["B"].shape[2:]
    h0 = rng.standard_normal((Bsz, H, P, N))
    v0 = rng.standard_normal((Bsz, H, P, N))
    y, hT, vT = oracle.ssd_seq(**inp, h0=h0, v0=v0, beta=0.6, alpha=1.2)
    for b in range(Bsz):
        for h in range(H):
            g = h // (H // G)
            x1 = np.ascontiguousarray(inp["x"][b, :, h, :].T[None])                # (1, P, L)
            d1 = np.ascontiguousarray(np.repeat(inp["delta"][b, :, h][None, None], P, 1))
            A1 = np.full((P, N), inp["A"][h], np.float32)
            B1 = np.ascontiguousarray(inp["B"][b, :, g, :].T[None])                # (1, N, L)
            C1 = np.ascontiguousarray(inp["C"][b, :, g, :].T[None])
            ys, hs, vs = oracle.scan_seq(x1, d1, A1, B1, C1, h0=h0[b, h][None], v0=v0[b, h][None],
                                         beta=0.6, alpha=1.2)
            rows = (b * H + h) * P + np.arange(P)
            assert np.array_equal(y[rows], ys)
            assert np.array_equal(hT[rows], hs) and np.array_equal(vT[rows], vs)


@pytest.mark.parametrize("chunk", [1, 8, 16, 50, 64])
def test_ssd_chunked_equals_sequential(chunk):
    inp, rng = _ssd_small()
    Bsz, L, H, P = inp["x"].shape
    N = inp["B"].shape[3]
    h0 = rng.standard_normal((Bsz, H, P, N))
    ys, hs, _ = oracle.ssd_seq(**inp, h0=h0, beta=0.0, alpha=0.7)
    yc, hc = oracle.ssd_chunked(**inp, h0=h0, alpha=0.7, chunk=chunk)
    yc_rows = yc.transpose(0, 2, 3, 1).reshape(Bsz * H * P, L)
    np.testing.assert_allclose(yc_rows, ys, rtol=1e-11, atol=1e-12 * np.abs(ys).max())
    np.testing.assert_allclose(hc.reshape(-1, N), hs, rtol=1e-11, atol=1e-13)


def test_ssd_brute_force_Lij():
    """Mamba-2 page: y_i = sum_{j<=i} C_i . A_i ... A_{j+1} . B_j x_j (scalar A)."""
    inp, rng = _ssd_small(L=12, H=2, P=2, N=3, G=1)
    Bsz, L, H, P = inp["x"].shape
    N = inp["B"].shape[3]
    h0 = rng.standard_normal((Bsz, H, P, N))
    yc, _ = oracle.ssd_chunked(**inp, h0=h0, alpha=1.0, chunk=5)
    yref = np.zeros((Bsz, L, H, P))
    for b in range(Bsz):
        for h in range(H):
            a = np.exp(inp["delta"][b, :, h].astype(np.float64) * float(inp["A"][h]))
            for i in range(L):
                Ci = inp["C"][b, i, 0].astype(np.float64)
                for j in range(i + 1):
                    Lij = Ci @ inp["B"][b, j, 0].astype(np.float64) * np.prod(a[j + 1:i + 1])
                    yref[b, i, h] += Lij * float(inp["delta"][b, j, h]) * inp["x"][b, j, h].astype(np.float64)
                yref[b, i, h] += np.prod(a[:i + 1]) * (h0[b, h] @ Ci)
    np.testing.assert_allclose(yc, yref, rtol=1e-11, atol=1e-12)


def test_ssd_chunked_rejects_momentum(oracle_lib):
    inp, _ = _ssd_small()
    f = oracle_lib.oracle_ssd_chunked
    import ctypes
    y = np.empty(inp["x"].shape, np.float64)
    fp = ctypes.POINTER(ctypes.c_float)
    dp = ctypes.POINTER(ctypes.c_double)
    arr = {k: np.ascontiguousarray(v, np.float32) for k, v in inp.items()}
    rc = f(*(arr[k].ctypes.data_as(fp) for k in ("x", "delta", "A", "B", "C")), None, 0.5, 1.0,
           2, 50, 4, 3, 5, 2, 16, y.ctypes.data_as(dp), None)
    assert rc != 0


# ------------------------------------------------------------ inputs -------
def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    a = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 100,
                        np.array([0.0, -0.0, 1.0, 3.4e38, -3.4e38, 1e-40, np.inf, -np.inf], np.float32)])
    ours = wl.bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_workload_draws_are_seeded_and_independent():
    a = wl.scan_inputs(wl.SCAN_SMALL)
    b = wl.scan_inputs(wl.SCAN_SMALL)
    assert all(np.array_equal(a[k], b[k]) for k in a)
    assert a["delta"].min() >= 1e-3 * (1 - 1e-6) and a["delta"].max() <= 1e-1 * (1 + 1e-6)
    assert np.array_equal(a["A"][0], -(np.arange(16) + 1.0).astype(np.float32))
    c = wl.scan_inputs(wl.SCAN_BF16, batch=1, seqlen=64, dim=8)
    assert np.array_equal(c["x"], wl.bf16_round(c["x"]))
    assert (c["delta"] > 0).all()
