"""GPU checks of the host-buffer entry points (mm_scan_fwd_host,
mm_ssd_fwd_host) through the C ABI.

The host entry streams the sequence through a device workspace in time
chunks, carrying the states on the device between chunks, so it must give
what the device entry gives for the same split (the streaming rule of
mm_scan_fwd: final states bit-identical, y within rounding), and match the
fp64 oracle at the device path's tolerances:
  * scan fp32: max |err| <= 1e-4 max |ref| (y, hT, vT); bf16 y relative L2
    <= 1e-2;
  * SSD and momentum SSD (tensor-core kernels at headdim 64, dstate 128:
    bf16 operands): y and the states relative L2 <= 1e-2.
"""
import ctypes

import numpy as np
import pytest

import oracle
import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_TOL = 1e-2


def _host(inp, io="f32", pin=True):
    dt = torch.float32 if io == "f32" else torch.bfloat16
    out = {}
    for k in ("x", "delta", "B", "C"):
        t = torch.from_numpy(np.ascontiguousarray(inp[k])).to(dt).contiguous()
        out[k] = t.pin_memory() if pin else t
    out["A"] = torch.from_numpy(np.ascontiguousarray(inp["A"])).contiguous()
    return out


def _max_ok(got, ref, what):
    err = np.abs(got - ref).max()
    assert err <= F32_TOL * np.abs(ref).max(), f"{what}: max abs err {err:.3e} vs {np.abs(ref).max():.3e}"


def _scan_oracle_check(out, inp, beta, alpha, io, h0=None, v0=None, what="", **extra):
    L, N = inp["x"].shape[2], inp["A"].shape[1]
    kw = dict(h0=None if h0 is None else h0.astype(np.float64), v0=None if v0 is None else v0.astype(np.float64))
    if extra:
        yr, hr, vr = oracle.scan_gated(**inp, **extra, **kw, beta=beta, alpha=alpha)
    else:
        yr, hr, vr = oracle.scan_seq(**inp, **kw, beta=beta, alpha=alpha)
    y = out["y"].float().numpy().reshape(-1, L)
    if io == "f32":
        _max_ok(y, yr, f"{what} y")
    else:
        rel = np.linalg.norm(y - yr) / np.linalg.norm(yr)
        assert rel <= BF16_TOL, f"{what}: y relative L2 {rel:.3e}"
    _max_ok(out["hT"].numpy().reshape(-1, N), hr, f"{what} hT")
    _max_ok(out["vT"].numpy().reshape(-1, N), vr, f"{what} vT")


@pytest.mark.parametrize("chunk_steps", [0, 96, 1000, 37])
def test_scan_host_matches_device_and_oracle(chunk_steps):
    # batch * dim > 4096: the register-resident path for every chunk and for the whole call
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=2, seqlen=1000, dim=2080)
    h = _host(inp)
    rng = np.random.default_rng(1)
    h0 = rng.standard_normal((2, 2080, 16)).astype(np.float32)
    v0 = (0.3 * rng.standard_normal((2, 2080, 16))).astype(np.float32)
    out = mm.scan_fwd_host(h["x"], h["delta"], h["A"], h["B"], h["C"], h0=torch.from_numpy(h0).pin_memory(),
                           v0=torch.from_numpy(v0).pin_memory(), beta=0.9, alpha=1.0, chunk_steps=chunk_steps)
    mm.mm_device_status()
    d = {k: v.cuda() for k, v in h.items()}
    y, hT, vT = mm.scan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], h0=torch.from_numpy(h0).cuda(),
                            v0=torch.from_numpy(v0).cuda(), beta=0.9, alpha=1.0)
    torch.cuda.synchronize()
    assert torch.equal(out["hT"], hT.cpu()) and torch.equal(out["vT"], vT.cpu()), \
        f"chunk_steps={chunk_steps}: final states differ from the device call"
    scale = y.abs().max().item()
    assert (out["y"] - y.cpu()).abs().max().item() <= F32_TOL * scale
    # 64 channels against the oracle
    chan = np.linspace(0, 2 * 2080 - 1, 64).astype(int)
    L = 1000
    yr, hr, vr = oracle.scan_seq(**inp, h0=h0.astype(np.float64), v0=v0.astype(np.float64), beta=0.9, alpha=1.0,
                                 chan=chan)
    _max_ok(out["y"].numpy().reshape(-1, L)[chan], yr, "y")
    _max_ok(out["hT"].numpy().reshape(-1, 16)[chan], hr, "hT")


@pytest.mark.parametrize("chunk_steps", [512, 1536])
def test_scan_host_on_the_sequence_split_path_is_identical(chunk_steps):
    # chunks at multiples of the segment length: the host call is the device call, bit for bit
    mm.mm_scan_set_path(2, 256)
    try:
        inp = wl.scan_inputs(wl.SCAN_LONG, batch=1, seqlen=4096, dim=64)
        h = _host(inp)
        out = mm.scan_fwd_host(h["x"], h["delta"], h["A"], h["B"], h["C"], beta=0.99, alpha=1.0,
                               chunk_steps=chunk_steps)
        d = {k: v.cuda() for k, v in h.items()}
        y, hT, vT = mm.scan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], beta=0.99, alpha=1.0)
        torch.cuda.synchronize()
        mm.mm_device_status()
    finally:
        mm.mm_scan_set_path(0, 0)
    assert torch.equal(out["hT"], hT.cpu()) and torch.equal(out["vT"], vT.cpu())
    assert torch.equal(out["y"], y.cpu())
    _scan_oracle_check(out, inp, 0.99, 1.0, "f32", what="sequence-split")


def test_scan_host_bf16_gated_with_states():
    inp = wl.scan_inputs(wl.SCAN_BF16, batch=2, seqlen=777, dim=96)
    for k in ("x", "delta", "B", "C"):
        inp[k] = wl.bf16_round(inp[k])
    rng = np.random.default_rng(2)
    z = wl.bf16_round(rng.standard_normal(inp["x"].shape).astype(np.float32))
    Dk = rng.standard_normal(96).astype(np.float32)
    bias = (0.1 * rng.standard_normal(96)).astype(np.float32)
    h0 = rng.standard_normal((2, 96, 16)).astype(np.float32)
    h = _host(inp, "bf16")
    out = mm.scan_fwd_host(h["x"], h["delta"], h["A"], h["B"], h["C"], h0=torch.from_numpy(h0), beta=0.9,
                           alpha=1.0, D=torch.from_numpy(Dk), z=torch.from_numpy(z).to(torch.bfloat16),
                           delta_bias=torch.from_numpy(bias), delta_softplus=True, chunk_steps=128)
    mm.mm_device_status()
    _scan_oracle_check(out, inp, 0.9, 1.0, "bf16", h0=h0, what="bf16 gated",
                       D=Dk, z=z, delta_bias=bias, delta_softplus=True)


def test_scan_host_in_place_states_and_pageable_memory():
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=1, seqlen=600, dim=40)
    h = _host(inp, pin=False)
    rng = np.random.default_rng(3)
    h0 = rng.standard_normal((1, 40, 16)).astype(np.float32)
    v0 = (0.2 * rng.standard_normal((1, 40, 16))).astype(np.float32)
    hs, vs = torch.from_numpy(h0.copy()), torch.from_numpy(v0.copy())
    y = torch.empty_like(h["x"])
    ws = torch.empty(mm.mm_scan_fwd_host_workspace_size(1, 600, 40, 16, chunk_steps=64), dtype=torch.uint8,
                     device="cuda")
    mm.mm_scan_fwd_host(h["x"], h["delta"], h["A"], h["B"], h["C"], None, None, None, False, hs, vs, 0.9, 1.0,
                        y, hs, vs, ws, chunk_steps=64)
    torch.cuda.synchronize()
    mm.mm_device_status()
    _scan_oracle_check({"y": y, "hT": hs, "vT": vs}, inp, 0.9, 1.0, "f32", h0=h0, v0=v0, what="in place")


def test_ssd_host_plain_and_momentum():
    inp = wl.ssd_inputs(wl.SSD_MH, batch=2, seqlen=1100, nheads=4, headdim=64, dstate=128, ngroups=1)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).contiguous().pin_memory()
    x, dl, A = t(inp["x"], torch.bfloat16), t(inp["delta"], torch.float32), t(inp["A"], torch.float32)
    B, C = t(inp["B"], torch.bfloat16), t(inp["C"], torch.bfloat16)
    rng = np.random.default_rng(4)
    h0 = rng.standard_normal((2, 4, 64, 128)).astype(np.float32)
    out = mm.ssd_fwd_host(x, dl, A, B, C, h0=torch.from_numpy(h0), chunk=256, chunk_steps=512)
    mm.mm_device_status()
    yr, hr = oracle.ssd_chunked(**inp, h0=h0.astype(np.float64), alpha=1.0, chunk=256)
    y = out["y"].float().numpy()
    rel = np.linalg.norm(y - yr.reshape(y.shape)) / np.linalg.norm(yr)
    assert rel <= BF16_TOL, f"SSD host y relative L2 {rel:.3e}"
    hg = out["hT"].numpy()
    rel = np.linalg.norm(hg - hr.reshape(hg.shape)) / np.linalg.norm(hr)
    assert rel <= BF16_TOL, f"SSD host hT relative L2 {rel:.3e}"
    v0 = (0.1 * rng.standard_normal((2, 4, 64, 128))).astype(np.float32)
    out = mm.ssd_fwd_host(x, dl, A, B, C, h0=torch.from_numpy(h0), v0=torch.from_numpy(v0), beta=0.9,
                          chunk=256, chunk_steps=256)
    mm.mm_device_status()
    yr, hr, vr = oracle.ssd_chunked_momentum(**inp, h0=h0.astype(np.float64), v0=v0.astype(np.float64),
                                             beta=0.9, alpha=1.0, chunk=64)
    y = out["y"].float().numpy()
    rel = np.linalg.norm(y - yr.reshape(y.shape)) / np.linalg.norm(yr)
    assert rel <= BF16_TOL, f"momentum SSD host y relative L2 {rel:.3e}"
    for name, ref in (("hT", hr), ("vT", vr)):      # tensor-core form: bf16 state products
        got = out[name].numpy()
        rel = np.linalg.norm(got - ref.reshape(got.shape)) / np.linalg.norm(ref)
        assert rel <= BF16_TOL, f"momentum SSD host {name} relative L2 {rel:.3e}"


def test_host_entry_rejects_device_tensors_and_small_workspaces():
    lib = mm.load_library()
    inp = wl.scan_inputs(wl.SCAN_SMALL, batch=1, seqlen=64, dim=8)
    h = _host(inp)
    d = {k: v.cuda() for k, v in h.items()}
    with pytest.raises(ValueError):
        mm.scan_fwd_host(d["x"], d["delta"], d["A"], d["B"], d["C"])
    need = mm.mm_scan_fwd_host_workspace_size(1, 64, 8, 16)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    y = torch.empty_like(h["x"])
    dims = mm.ScanDims(1, 64, 8, 16, mm.MM_F32)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # x in device memory, through the C ABI directly
    rc = lib.mm_scan_fwd_host(P(d["x"]), P(h["delta"]), P(h["A"]), P(h["B"]), P(h["C"]), None, None, None, 0, None,
                              None, 0.9, 1.0, P(y), None, None, P(ws), need, 0, ctypes.byref(dims), stream)
    assert rc == 6, mm.mm_last_error()
    rc = lib.mm_scan_fwd_host(P(h["x"]), P(h["delta"]), P(h["A"]), P(h["B"]), P(h["C"]), None, None, None, 0, None,
                              None, 0.9, 1.0, P(y), None, None, P(ws), need - 1, 0, ctypes.byref(dims), stream)
    assert rc == 2, mm.mm_last_error()
    hws = torch.empty(need, dtype=torch.uint8)
    rc = lib.mm_scan_fwd_host(P(h["x"]), P(h["delta"]), P(h["A"]), P(h["B"]), P(h["C"]), None, None, None, 0, None,
                              None, 0.9, 1.0, P(y), None, None, P(hws), need, 0, ctypes.byref(dims), stream)
    assert rc == 6, mm.mm_last_error()
    rc = lib.mm_scan_fwd_host(P(h["x"]), P(h["delta"]), P(h["A"]), P(h["B"]), P(h["C"]), None, None, None, 0, None,
                              None, 0.9, 1.0, P(y), None, None, P(ws), need, 0, ctypes.byref(dims), stream)
    assert rc == 0, mm.mm_last_error()
    torch.cuda.synchronize()
    mm.mm_device_status()
