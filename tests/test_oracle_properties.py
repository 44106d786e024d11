"""Property-based checks of the oracle over random shapes and scalars.

The seeded pins elsewhere fix the oracle's values on chosen cases; these
draw the shapes (batch, dim, L, N, heads, groups, chunk lengths), beta and
alpha at random and check relations the recurrence of "Momentum Mamba:
Enhanced State Space Models with Momentum" ("Momentum Mamba Recurrence")
implies whatever the inputs:

* the chunked forms (per-chunk affine maps and a carry fold; the SSD
  "4-Step Algorithm" with and without momentum) agree with the sequential
  definition for any chunk length;
* a sequence scanned in two calls, the second starting from the first's
  final states, gives the one-call result exactly (the streaming use of
  (h0, v0) -> (hT, vT));
* the map (x, h0, v0) -> (y, hT, vT) is linear (exact under a power-of-two
  scale) and causal (y before a changed input is unchanged, bit for bit);
* the states are independent, so y is the sum over n of single-state scans;
* the multi-head scalar-A layout is the Mamba-1 scan of its channels.
"""
import numpy as np
import pytest

hyp = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

import oracle  # noqa: E402

SETTINGS = settings(max_examples=60, deadline=None, database=None, derandomize=True)


def _scan_inputs(seed, batch, dim, L, N):
    rng = np.random.default_rng(seed)
    return {
        "x": rng.standard_normal((batch, dim, L)).astype(np.float32),
        "delta": np.exp(rng.uniform(np.log(1e-3), np.log(0.5), (batch, dim, L))).astype(np.float32),
        "A": (-rng.uniform(0.05, 4.0, (dim, N))).astype(np.float32),
        "B": rng.standard_normal((batch, N, L)).astype(np.float32),
        "C": rng.standard_normal((batch, N, L)).astype(np.float32),
    }


def _states(seed, batch, dim, N):
    rng = np.random.default_rng(seed + 1)
    return rng.standard_normal((batch, dim, N)), rng.standard_normal((batch, dim, N))


scan_shapes = st.tuples(st.integers(0, 2**31 - 1), st.integers(1, 2), st.integers(1, 5),
                        st.integers(1, 70), st.integers(1, 16))
betas = st.floats(0.0, 0.999)
alphas = st.one_of(st.just(0.0), st.floats(1e-3, 3.0))    # no subnormal products: scaling stays exact


def _close(a, b, rel=1e-11):
    scale = max(np.abs(b).max(), 1e-300)
    return np.abs(a - b).max() <= rel * scale


@SETTINGS
@given(scan_shapes, betas, alphas, st.integers(1, 80))
def test_chunked_equals_sequential_for_any_chunk(shape, beta, alpha, chunk):
    seed, batch, dim, L, N = shape
    inp = _scan_inputs(seed, batch, dim, L, N)
    h0, v0 = _states(seed, batch, dim, N)
    ys, hs, vs = oracle.scan_seq(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha)
    yc, hc, vc = oracle.scan_chunked(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha, chunk=chunk)
    assert _close(yc, ys) and _close(hc, hs) and _close(vc, vs)


@SETTINGS
@given(scan_shapes, betas, alphas, st.data())
def test_two_calls_carrying_the_state_equal_one_call_exactly(shape, beta, alpha, data):
    seed, batch, dim, L, N = shape
    if L < 2:
        L = 2
    inp = _scan_inputs(seed, batch, dim, L, N)
    h0, v0 = _states(seed, batch, dim, N)
    cut = data.draw(st.integers(1, L - 1))
    y, hT, vT = oracle.scan_seq(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha)
    first = {k: (v[..., :cut] if k in ("x", "delta", "B", "C") else v) for k, v in inp.items()}
    rest = {k: (v[..., cut:] if k in ("x", "delta", "B", "C") else v) for k, v in inp.items()}
    y1, h1, v1 = oracle.scan_seq(**first, h0=h0, v0=v0, beta=beta, alpha=alpha)
    y2, h2, v2 = oracle.scan_seq(**rest, h0=h1.reshape(batch, dim, N), v0=v1.reshape(batch, dim, N),
                                 beta=beta, alpha=alpha)
    assert np.array_equal(np.concatenate([y1, y2], axis=1), y)
    assert np.array_equal(h2, hT) and np.array_equal(v2, vT)


@SETTINGS
@given(scan_shapes, betas, alphas, st.sampled_from([0.5, 2.0, 4.0, 0.25]))
def test_linear_in_input_and_initial_states(shape, beta, alpha, s):
    seed, batch, dim, L, N = shape
    inp = _scan_inputs(seed, batch, dim, L, N)
    h0, v0 = _states(seed, batch, dim, N)
    y, hT, vT = oracle.scan_seq(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha)
    scaled = dict(inp, x=(inp["x"] * np.float32(s)).astype(np.float32))
    ys, hs, vs = oracle.scan_seq(**scaled, h0=h0 * s, v0=v0 * s, beta=beta, alpha=alpha)
    # a power-of-two scale commutes with every rounding: exact
    assert np.array_equal(ys, y * s) and np.array_equal(hs, hT * s) and np.array_equal(vs, vT * s)
    # superposition of the input part and the initial-state part
    y_in, h_in, v_in = oracle.scan_seq(**inp, beta=beta, alpha=alpha)
    zero_x = dict(inp, x=np.zeros_like(inp["x"]))
    y_st, h_st, v_st = oracle.scan_seq(**zero_x, h0=h0, v0=v0, beta=beta, alpha=alpha)
    assert _close(y_in + y_st, y, 1e-12) and _close(h_in + h_st, hT, 1e-12) and _close(v_in + v_st, vT, 1e-12)


@SETTINGS
@given(scan_shapes, betas, alphas, st.data())
def test_causal_bit_for_bit(shape, beta, alpha, data):
    seed, batch, dim, L, N = shape
    inp = _scan_inputs(seed, batch, dim, L, N)
    k = data.draw(st.integers(0, L - 1))
    y, _, _ = oracle.scan_seq(**inp, beta=beta, alpha=alpha)
    for name in ("x", "delta", "B", "C"):
        changed = {kk: v.copy() for kk, v in inp.items()}
        changed[name][..., k] += np.float32(0.75)
        y2, _, _ = oracle.scan_seq(**changed, beta=beta, alpha=alpha)
        assert np.array_equal(y2[:, :k], y[:, :k]), name


@SETTINGS
@given(scan_shapes, betas, alphas)
def test_output_is_the_sum_of_single_state_scans(shape, beta, alpha):
    seed, batch, dim, L, N = shape
    inp = _scan_inputs(seed, batch, dim, L, N)
    y, hT, _ = oracle.scan_seq(**inp, beta=beta, alpha=alpha)
    total = np.zeros_like(y)
    for n in range(N):
        one = dict(inp, A=np.ascontiguousarray(inp["A"][:, n:n + 1]),
                   B=np.ascontiguousarray(inp["B"][:, n:n + 1]), C=np.ascontiguousarray(inp["C"][:, n:n + 1]))
        yn, hn, _ = oracle.scan_seq(**one, beta=beta, alpha=alpha)
        total += yn
        assert np.array_equal(hn[:, 0], hT[:, n])      # a state sees only its own column
    assert _close(total, y, 1e-12)


def _ssd_inputs(seed, batch, L, H, P, N, G):
    rng = np.random.default_rng(seed)
    return {
        "x": rng.standard_normal((batch, L, H, P)).astype(np.float32),
        "delta": np.exp(rng.uniform(np.log(1e-3), np.log(0.5), (batch, L, H))).astype(np.float32),
        "A": (-rng.uniform(0.05, 4.0, H)).astype(np.float32),
        "B": rng.standard_normal((batch, L, G, N)).astype(np.float32),
        "C": rng.standard_normal((batch, L, G, N)).astype(np.float32),
    }


ssd_shapes = st.tuples(st.integers(0, 2**31 - 1), st.integers(1, 2), st.integers(1, 70),
                       st.sampled_from([(1, 1), (2, 1), (2, 2), (4, 2)]), st.integers(1, 4),
                       st.integers(1, 8))


@SETTINGS
@given(ssd_shapes, betas, alphas)
def test_multi_head_layout_is_the_channel_scan(shape, beta, alpha):
    seed, batch, L, (H, G), P, N = shape
    inp = _ssd_inputs(seed, batch, L, H, P, N, G)
    y, hT, vT = oracle.ssd_seq(**inp, beta=beta, alpha=alpha)
    # the same lanes as Mamba-1 channels: d = (h, p), A[d, n] = A_h,
    # B/C of the head's group, x and delta of (t, h, p) / (t, h)
    D = H * P
    hp = np.arange(D)
    head = hp // P
    grp = head // (H // G)
    x1 = np.ascontiguousarray(inp["x"].reshape(batch, L, D).transpose(0, 2, 1))
    d1 = np.ascontiguousarray(inp["delta"][:, :, head].transpose(0, 2, 1))
    A1 = np.ascontiguousarray(np.repeat(inp["A"][head][:, None], N, axis=1))
    for gg in range(G):
        sel = np.nonzero(grp == gg)[0]
        B1 = np.ascontiguousarray(inp["B"][:, :, gg, :].transpose(0, 2, 1))
        C1 = np.ascontiguousarray(inp["C"][:, :, gg, :].transpose(0, 2, 1))
        ym, hm, vm = oracle.scan_seq(np.ascontiguousarray(x1[:, sel]), np.ascontiguousarray(d1[:, sel]),
                                     np.ascontiguousarray(A1[sel]), B1, C1, beta=beta, alpha=alpha)
        lanes = (np.arange(batch)[:, None] * D + sel[None, :]).reshape(-1)
        assert _close(ym, y[lanes], 1e-13) and _close(hm, hT[lanes], 1e-13) and _close(vm, vT[lanes], 1e-13)


@SETTINGS
@given(ssd_shapes, alphas, st.sampled_from([1, 2, 4, 8, 16, 32, 64]))
def test_ssd_chunked_equals_sequential(shape, alpha, chunk):
    seed, batch, L, (H, G), P, N = shape
    inp = _ssd_inputs(seed, batch, L, H, P, N, G)
    rng = np.random.default_rng(seed + 7)
    h0 = rng.standard_normal((batch, H, P, N))
    yc, hc = oracle.ssd_chunked(**inp, h0=h0, alpha=alpha, chunk=chunk)
    ys, hs, _ = oracle.ssd_seq(**inp, h0=h0, alpha=alpha)
    assert _close(yc.transpose(0, 2, 3, 1).reshape(-1, L), ys, 1e-10)
    assert _close(hc.reshape(-1, N), hs, 1e-10)


@SETTINGS
@given(ssd_shapes, betas, alphas, st.integers(1, 40))
def test_ssd_momentum_chunked_equals_sequential(shape, beta, alpha, chunk):
    seed, batch, L, (H, G), P, N = shape
    inp = _ssd_inputs(seed, batch, L, H, P, N, G)
    rng = np.random.default_rng(seed + 9)
    h0 = rng.standard_normal((batch, H, P, N))
    v0 = rng.standard_normal((batch, H, P, N))
    yc, hc, vc = oracle.ssd_chunked_momentum(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha, chunk=chunk)
    ys, hs, vs = oracle.ssd_seq(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha)
    assert _close(yc.transpose(0, 2, 3, 1).reshape(-1, L), ys, 1e-10)
    assert _close(hc.reshape(-1, N), hs, 1e-10) and _close(vc.reshape(-1, N), vs, 1e-10)


bwd_shapes = st.tuples(st.integers(0, 2**31 - 1), st.integers(1, 2), st.integers(1, 3), st.integers(1, 20),
                       st.integers(1, 6))


@SETTINGS
@given(bwd_shapes, st.floats(0.0, 0.95), st.floats(0.1, 2.0), st.booleans(), st.booleans())
def test_backward_matches_directional_differences(shape, beta, alpha, extras, states):
    """The backward oracle's gradient of a random linear functional of
    (out, hT, vT) against a central difference of the forward along a random
    direction, one input array at a time, for random shapes and scalars
    (with and without D, z, delta_bias + softplus, h0 and v0)."""
    seed, batch, dim, L, N = shape
    rng = np.random.default_rng(seed)
    f32 = np.float32
    p = {"x": rng.standard_normal((batch, dim, L)).astype(f32),
         "delta": (rng.uniform(0.02, 0.3, (batch, dim, L)) if not extras
                   else rng.standard_normal((batch, dim, L)) * 0.5).astype(f32),
         "A": (-rng.uniform(0.2, 2.0, (dim, N))).astype(f32),
         "B": rng.standard_normal((batch, N, L)).astype(f32),
         "C": rng.standard_normal((batch, N, L)).astype(f32)}
    if extras:
        p.update(D=rng.uniform(0.5, 1.5, dim).astype(f32), z=rng.standard_normal((batch, dim, L)).astype(f32),
                 delta_bias=rng.uniform(-3.0, -1.0, dim).astype(f32))
    if states:
        p.update(h0=rng.standard_normal((batch, dim, N)), v0=rng.standard_normal((batch, dim, N)))
    dout = rng.standard_normal((batch, dim, L)).astype(f32)
    dhT = rng.standard_normal((batch, dim, N))
    dvT = rng.standard_normal((batch, dim, N))

    def loss(q):
        out, hT, vT = oracle.scan_gated(q["x"], q["delta"], q["A"], q["B"], q["C"], D=q.get("D"), z=q.get("z"),
                                        delta_bias=q.get("delta_bias"), delta_softplus=extras, h0=q.get("h0"),
                                        v0=q.get("v0"), beta=beta, alpha=alpha)
        return (float(np.sum(dout.astype(np.float64).reshape(out.shape) * out))
                + float(np.sum(dhT.reshape(hT.shape) * hT)) + float(np.sum(dvT.reshape(vT.shape) * vT)))

    gr = oracle.scan_bwd(p["x"], p["delta"], p["A"], p["B"], p["C"], dout, D=p.get("D"), z=p.get("z"),
                         delta_bias=p.get("delta_bias"), delta_softplus=extras, h0=p.get("h0"), v0=p.get("v0"),
                         dhT=dhT, dvT=dvT, beta=beta, alpha=alpha)
    grad_of = {"x": "dx", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "z": "dz",
               "delta_bias": "ddelta_bias", "h0": "dh0", "v0": "dv0"}
    for name, arr in p.items():
        r = rng.standard_normal(arr.shape)
        eps = 1e-4 if arr.dtype == f32 else 1e-6    # curvature error ~2e-5 of the difference at most
        up = (arr + eps * r).astype(arr.dtype)
        dn = (arr - eps * r).astype(arr.dtype)
        step = up.astype(np.float64) - dn.astype(np.float64)     # the move the dtype actually made
        lhs = loss(dict(p, **{name: up})) - loss(dict(p, **{name: dn}))
        rhs = float(np.sum(gr[grad_of[name]].reshape(arr.shape) * step))
        scale = max(abs(lhs), abs(rhs))
        assert abs(lhs - rhs) <= 2e-4 * scale + 1e-9, (name, lhs, rhs)
