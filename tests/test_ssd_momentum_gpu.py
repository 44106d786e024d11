"""GPU parity of the momentum SSD path (mm_ssd_fwd_momentum, and mm_ssd_fwd
with beta != 0) against the fp64 oracle, through the C ABI.

Tolerances: y is bf16, relative L2 <= 1e-2 (the scan's bf16 bound).  The
states hT, vT (fp32): relative L2 <= 1e-2 on the tensor-core form (headdim 64,
dstate 128), whose state products take bf16 operands like mm_ssd_fwd's;
max |err| <= 1e-4 max |ref| on the CUDA-core form (other sizes), which keeps
every product in fp32.
"""
import numpy as np
import pytest

import oracle
import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

BF16_TOL = 1e-2
F32_TOL = 1e-4


def _dev(inp):
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(dt).contiguous()
    return {"x": t(inp["x"], torch.bfloat16), "delta": t(inp["delta"], torch.float32),
            "A": t(inp["A"], torch.float32), "B": t(inp["B"], torch.bfloat16),
            "C": t(inp["C"], torch.bfloat16)}


def _problem(batch=2, L=150, H=4, P=64, N=128, G=2, seed=0, states=True):
    inp = wl.ssd_inputs(wl.SSD_MH, batch=batch, seqlen=L, nheads=H, headdim=P, dstate=N, ngroups=G)
    rng = np.random.default_rng(seed)
    h0 = rng.standard_normal((batch, H, P, N)).astype(np.float32) if states else None
    v0 = (0.1 * rng.standard_normal((batch, H, P, N))).astype(np.float32) if states else None
    return inp, h0, v0


def _tensor_core(P, N):
    return P == 64 and N == 128


def _state_ok(got, ref, tc, what):
    ref = ref.reshape(got.shape)
    if tc:
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel <= BF16_TOL, f"{what}: relative L2 {rel:.3g}"
    else:
        err = np.abs(got - ref).max()
        assert err <= F32_TOL * np.abs(ref).max(), f"{what}: max abs err {err:.3g}"


def _check(got, ref, what):
    y, hT, vT = (a.float().cpu().numpy() for a in got)
    yr, hr, vr = ref
    rel = np.linalg.norm(y - yr.reshape(y.shape)) / np.linalg.norm(yr)
    assert rel <= BF16_TOL, f"{what} y rel L2 {rel:.3g}"
    tc = _tensor_core(hT.shape[2], hT.shape[3])
    for a, r, nm in ((hT, hr, "hT"), (vT, vr, "vT")):
        _state_ok(a, r, tc, f"{what} {nm}")


@pytest.mark.parametrize("beta,alpha", [(0.9, 1.0), (0.5, 2.0), (0.99, 0.5)])
def test_momentum_ssd_matches_oracle(beta, alpha):
    inp, h0, v0 = _problem(seed=int(beta * 100))
    d = _dev(inp)
    got = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=torch.from_numpy(h0).cuda(),
                              v0=torch.from_numpy(v0).cuda(), beta=beta, alpha=alpha)
    torch.cuda.synchronize()
    mm.mm_device_status()
    ref = oracle.ssd_chunked_momentum(**inp, h0=h0.astype(np.float64), v0=v0.astype(np.float64), beta=beta,
                                      alpha=alpha, chunk=64)
    _check(got, ref, f"beta={beta} alpha={alpha}")


@pytest.mark.parametrize("shape", [(1, 1, 2, 16, 32, 1), (2, 70, 3, 8, 5, 3), (1, 200, 2, 64, 128, 2)])
def test_momentum_ssd_shapes_and_lengths(shape):
    batch, L, H, P, N, G = shape
    inp, h0, v0 = _problem(batch, L, H, P, N, G, seed=L)
    d = _dev(inp)
    got = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=torch.from_numpy(h0).cuda(),
                              v0=torch.from_numpy(v0).cuda(), beta=0.8, alpha=1.0)
    torch.cuda.synchronize()
    ref = oracle.ssd_chunked_momentum(**inp, h0=h0.astype(np.float64), v0=v0.astype(np.float64), beta=0.8,
                                      alpha=1.0, chunk=64)
    _check(got, ref, f"shape {shape}")


def test_beta_zero_is_the_plain_recurrence():
    inp, h0, _ = _problem(L=130, seed=5)
    d = _dev(inp)
    y, hT, vT = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"],
                                    h0=torch.from_numpy(h0).cuda(), beta=0.0, alpha=1.0)
    torch.cuda.synchronize()
    yr, hr = oracle.ssd_chunked(**inp, h0=h0.astype(np.float64), alpha=1.0, chunk=64)
    rel = np.linalg.norm(y.float().cpu().numpy() - yr.reshape(y.shape)) / np.linalg.norm(yr)
    assert rel <= BF16_TOL
    _state_ok(hT.cpu().numpy(), hr, True, "beta = 0 hT")


def test_ssd_fwd_with_beta_routes_to_momentum():
    inp, h0, _ = _problem(batch=1, L=256, H=2, G=1, seed=6)
    d = _dev(inp)
    h0t = torch.from_numpy(h0).cuda()
    y, hT = mm.ssd_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=h0t, alpha=1.0, chunk=256)
    ym, hm, _ = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=h0t, beta=0.0)
    y2 = torch.empty_like(d["x"])
    h2 = torch.empty_like(hT)
    mm.mm_ssd_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], h0t, 0.7, 1.0, y2, h2, 256)
    torch.cuda.synchronize()
    ref = oracle.ssd_chunked_momentum(**inp, h0=h0.astype(np.float64), beta=0.7, alpha=1.0, chunk=64)
    rel = np.linalg.norm(y2.float().cpu().numpy() - ref[0].reshape(y2.shape)) / np.linalg.norm(ref[0])
    assert rel <= BF16_TOL
    _state_ok(h2.cpu().numpy(), ref[1], True, "routed hT")


def test_streaming_split_bit_identical():
    """Two calls split at a multiple of the kernel's block (128 steps on the
    tensor cores, 32 on the CUDA cores), carrying (hT, vT): the same blocks,
    so the same final states and y bit for bit."""
    inp, h0, v0 = _problem(batch=1, L=320, H=2, G=1, seed=7)
    d = _dev(inp)
    h0t, v0t = torch.from_numpy(h0).cuda(), torch.from_numpy(v0).cuda()
    y, hT, vT = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=h0t, v0=v0t, beta=0.95)
    sl = lambda a, lo, hi: a[:, lo:hi].contiguous()
    p1 = {k: (sl(v, 0, 128) if k != "A" else v) for k, v in d.items()}
    p2 = {k: (sl(v, 128, 320) if k != "A" else v) for k, v in d.items()}
    y1, h1, v1 = mm.ssd_fwd_momentum(p1["x"], p1["delta"], p1["A"], p1["B"], p1["C"], h0=h0t, v0=v0t, beta=0.95)
    y2, h2, v2 = mm.ssd_fwd_momentum(p2["x"], p2["delta"], p2["A"], p2["B"], p2["C"], h0=h1, v0=v1, beta=0.95)
    torch.cuda.synchronize()
    assert torch.equal(h2, hT) and torch.equal(v2, vT)
    assert torch.equal(torch.cat([y1, y2], dim=1), y)


def test_full_size_sampled():
    w = wl.SSD_MH
    inp = wl.ssd_inputs(w)
    d = _dev(inp)
    y, hT, vT = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"], beta=0.9, alpha=1.0)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    nl = w.batch * w.nheads * w.headdim
    lane = np.unique(np.concatenate([rng.choice(nl, 12, replace=False), [0, nl - 1]])).astype(np.int64)
    yr, hr, vr = oracle.ssd_seq(**inp, beta=0.9, alpha=1.0, lane=lane)
    b, hh, p = lane // (w.nheads * w.headdim), (lane // w.headdim) % w.nheads, lane % w.headdim
    yg = y.float().cpu().numpy()[b, :, hh, p]                  # (nlane, L)
    rel = np.linalg.norm(yg - yr) / np.linalg.norm(yr)
    assert rel <= BF16_TOL
    hg = hT.cpu().numpy()[b, hh, p]                            # (nlane, N)
    _state_ok(hg, hr, True, "full-size hT")
    vg = vT.cpu().numpy()[b, hh, p]
    _state_ok(vg, vr, True, "full-size vT")


@pytest.mark.parametrize("beta", [0.0, 0.5, 0.9, 0.99])
@pytest.mark.parametrize("L,G", [(1, 1), (129, 2), (300, 4), (513, 1)])
def test_tensor_core_form_lengths_groups_and_betas(beta, L, G):
    # headdim 64, dstate 128: the tcgen05 form, blocks of 128 steps with a ragged last block
    inp, h0, v0 = _problem(batch=2, L=L, H=4, G=G, seed=L + int(100 * beta))
    d = _dev(inp)
    got = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=torch.from_numpy(h0).cuda(),
                              v0=torch.from_numpy(v0).cuda(), beta=beta, alpha=0.7)
    torch.cuda.synchronize()
    mm.mm_device_status()
    ref = oracle.ssd_chunked_momentum(**inp, h0=h0.astype(np.float64), v0=v0.astype(np.float64), beta=beta,
                                      alpha=0.7, chunk=64)
    _check(got, ref, f"L={L} G={G} beta={beta}")


@pytest.mark.parametrize("scale,a_sign", [(20.0, -1.0), (1.0, 1.0)], ids=["strong-decay", "growing"])
def test_tensor_core_form_extreme_decays(scale, a_sign):
    # strong decay: a block's decay spans hundreds of powers of two; growing: A > 0
    inp, h0, v0 = _problem(batch=1, L=384, H=2, G=1, seed=9)
    inp["delta"] = (inp["delta"] * scale).astype(np.float32)
    if a_sign > 0:
        inp["A"] = (np.abs(inp["A"]) * 0.02).astype(np.float32)
    d = _dev(inp)
    got = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=torch.from_numpy(h0).cuda(),
                              v0=torch.from_numpy(v0).cuda(), beta=0.9, alpha=1.0)
    torch.cuda.synchronize()
    mm.mm_device_status()
    ref = oracle.ssd_chunked_momentum(**inp, h0=h0.astype(np.float64), v0=v0.astype(np.float64), beta=0.9,
                                      alpha=1.0, chunk=64)
    _check(got, ref, f"delta x{scale}, A sign {a_sign}")


def test_tensor_core_form_streaming_at_block_multiples():
    inp, h0, v0 = _problem(batch=1, L=700, H=2, G=1, seed=10)
    d = _dev(inp)
    h0t, v0t = torch.from_numpy(h0).cuda(), torch.from_numpy(v0).cuda()
    y, hT, vT = mm.ssd_fwd_momentum(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=h0t, v0=v0t, beta=0.9)
    sl = lambda a, lo, hi: a[:, lo:hi].contiguous()
    h, v, ys = h0t, v0t, []
    for lo, hi in ((0, 256), (256, 384), (384, 700)):
        part = {k: (sl(t, lo, hi) if k != "A" else t) for k, t in d.items()}
        yp, h, v = mm.ssd_fwd_momentum(part["x"], part["delta"], part["A"], part["B"], part["C"], h0=h, v0=v,
                                       beta=0.9)
        ys.append(yp)
    torch.cuda.synchronize()
    assert torch.equal(h, hT) and torch.equal(v, vT)
    assert torch.equal(torch.cat(ys, dim=1), y)
