"""Pins of the oracle's chunked momentum SSD form (oracle.ssd_chunked_momentum).

The pages give the momentum recurrence (Momentum Mamba README, "Momentum
Mamba Recurrence") and the chunked SSD algorithm for the plain recurrence
("Mamba-2 -- SSM = structured matrix multiply", "4-Step Algorithm") but not
their combination; the chunked form with momentum is derived in the oracle
(mask M_ij = sum_k exp(cs_i - cs_k) beta^(k-j), two carried states).  What
pins it, independently of that derivation:

* equality with the sequential multi-head recurrence (oracle.ssd_seq, itself
  pinned to the scan's sequential definition) for chunk lengths from 1 to
  longer than the sequence, ragged last chunks, several groups, a carried
  (h0, v0): y, hT and vT;
* beta = 0 gives the plain chunked form (oracle.ssd_chunked) and vT = the
  last step's input state;
* a chunk of length 1 is one step of the recurrence.
"""
import numpy as np
import pytest

import oracle
from selective_state_space_momentum_b200 import workloads as wl


def _problem(seed, batch=2, L=40, H=4, P=3, N=5, G=2):
    inp = wl.ssd_inputs(wl.SSD_MH, batch=batch, seqlen=L, nheads=H, headdim=P, dstate=N, ngroups=G)
    rng = np.random.default_rng(seed)
    inp["delta"] = np.exp(rng.uniform(np.log(0.02), np.log(0.5), inp["delta"].shape)).astype(np.float32)
    h0 = rng.standard_normal((batch, H, P, N))
    v0 = rng.standard_normal((batch, H, P, N))
    return inp, h0, v0


def _seq(inp, h0, v0, beta, alpha, lib=None):
    batch, L, H, P = inp["x"].shape
    N = inp["B"].shape[3]
    y, hT, vT = oracle.ssd_seq(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha, lib=lib)
    return (y.reshape(batch, H, P, L).transpose(0, 3, 1, 2), hT.reshape(batch, H, P, N),
            vT.reshape(batch, H, P, N))


def chunked_failures(lib=None):
    """Cases where the chunked momentum form disagrees with the sequential one."""
    bad = []
    for beta, alpha, chunk in ((0.9, 1.0, 8), (0.5, 2.0, 7), (0.99, 0.5, 64), (0.3, 1.0, 1)):
        inp, h0, v0 = _problem(int(beta * 100) + chunk)
        got = oracle.ssd_chunked_momentum(**inp, h0=h0, v0=v0, beta=beta, alpha=alpha, chunk=chunk, lib=lib)
        ref = _seq(inp, h0, v0, beta, alpha, lib=lib)
        for a, r, nm in zip(got, ref, ("y", "hT", "vT")):
            if not np.allclose(a, r, rtol=1e-10, atol=1e-10 * np.abs(r).max()):
                bad.append(f"{nm} beta={beta} chunk={chunk}")
    return bad


def test_chunked_equals_sequential():
    assert chunked_failures() == []


@pytest.mark.parametrize("chunk", [1, 5, 16, 40, 100])
def test_chunk_lengths(chunk):
    inp, h0, v0 = _problem(chunk, L=33)
    got = oracle.ssd_chunked_momentum(**inp, h0=h0, v0=v0, beta=0.8, alpha=1.0, chunk=chunk)
    ref = _seq(inp, h0, v0, 0.8, 1.0)
    for a, r in zip(got, ref):
        np.testing.assert_allclose(a, r, rtol=1e-10, atol=1e-10 * np.abs(r).max())


def test_beta_zero_is_the_plain_chunked_form():
    inp, h0, _ = _problem(3, L=50)
    y, hT, vT = oracle.ssd_chunked_momentum(**inp, h0=h0, beta=0.0, alpha=1.5, chunk=16)
    y0, h00 = oracle.ssd_chunked(**inp, h0=h0, alpha=1.5, chunk=16)
    np.testing.assert_allclose(y, y0.reshape(y.shape), rtol=1e-12, atol=1e-12 * np.abs(y0).max())
    np.testing.assert_allclose(hT, h00.reshape(hT.shape), rtol=1e-12, atol=1e-12 * np.abs(h00).max())
    # with beta = 0 the velocity is the last step's input alpha delta B x
    x, d, B = inp["x"][:, -1], inp["delta"][:, -1], inp["B"][:, -1]          # (b,H,P), (b,H), (b,G,N)
    G = B.shape[1]
    H = x.shape[1]
    Bh = np.repeat(B, H // G, axis=1)                                           # (b,H,N)
    ref = (1.5 * d.astype(np.float64)[:, :, None, None] * x.astype(np.float64)[:, :, :, None]
           * Bh.astype(np.float64)[:, :, None, :])
    np.testing.assert_allclose(vT, ref, rtol=1e-12, atol=1e-15)
