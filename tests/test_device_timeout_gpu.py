"""Bounded device-side waits give up, report, and leave the context usable.

Every kernel that stages its inputs through mbarrier waits bounds each wait
(2 s of %globaltimer); a wait that runs out records the fact in the kernel
file's device error word, the whole CTA leaves together, and
mm_device_status() returns MM_ERR_DEVICE_TIMEOUT.  The test hook
MMSCAN_FAULT_INJECT=stall launches a kernel whose producer issues no copy at
all -- a flag that nothing sets, the allowed way to make a wait run out: no
copy is in flight, no GPU fault is provoked -- and each test then checks the
status and that a normal call right after still matches the fp64 oracle.
One test per kernel family: the register-resident scan, the sequence-split
scan (fused, and both launches of its split across ranks), the backward,
the SSD kernel, the tensor-core momentum SSD kernel.
"""
import numpy as np
import pytest

import oracle
import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

F32_TOL = 1e-4


def _expect_timeout():
    with pytest.raises(mm.MMError) as ei:
        mm.mm_device_status()
    assert ei.value.name == "MM_ERR_DEVICE_TIMEOUT", str(ei.value)
    mm.mm_device_status()                  # the record is cleared: the next check is clean


def _scan_dev(inp):
    out = {k: torch.from_numpy(inp[k]).cuda().contiguous() for k in ("x", "delta", "B", "C", "A")}
    return out


def _scan_check(dev, inp):
    y, hT, vT = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.9, alpha=1.0)
    torch.cuda.synchronize()
    mm.mm_device_status()
    L, N = inp["x"].shape[2], inp["A"].shape[1]
    yr, hr, vr = oracle.scan_seq(**inp, beta=0.9, alpha=1.0)
    assert np.abs(y.cpu().numpy().reshape(-1, L) - yr).max() <= F32_TOL * np.abs(yr).max()
    assert np.abs(hT.cpu().numpy().reshape(-1, N) - hr).max() <= F32_TOL * np.abs(hr).max()


@pytest.mark.parametrize("path,seg", [(1, 0), (2, 64)], ids=["register-resident", "sequence-split"])
def test_forward_scan_wait_runs_out(monkeypatch, path, seg):
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=2, seqlen=512, dim=48)
    dev = _scan_dev(inp)
    mm.mm_scan_set_path(path, seg)
    try:
        monkeypatch.setenv("MMSCAN_FAULT_INJECT", "stall")
        mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.9, alpha=1.0)
        monkeypatch.delenv("MMSCAN_FAULT_INJECT")
        _expect_timeout()
        _scan_check(dev, inp)
    finally:
        mm.mm_scan_set_path(0, 0)


def test_split_scan_waits_run_out(monkeypatch):
    # both launches of the scan split across ranks (one rank here)
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=2, seqlen=512, dim=48)
    dev = _scan_dev(inp)
    S, (batch, dim, L), N = 64, dev["x"].shape, dev["A"].shape[1]
    maps = torch.empty(mm.mm_scan_split_maps_size(batch, L, dim, N, L // S), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(dev["x"])
    h0 = torch.ones((batch, dim, N), device="cuda")
    hT, vT = torch.empty_like(h0), torch.empty_like(h0)
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "stall")
    mm.mm_scan_fwd_split_maps(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], 0.9, 1.0, y, maps, S)
    monkeypatch.delenv("MMSCAN_FAULT_INJECT")
    _expect_timeout()
    mm.mm_scan_fwd_split_maps(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], 0.9, 1.0, y, maps, S)
    mm.mm_device_status()
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "stall")
    mm.mm_scan_fwd_split_correct(dev["delta"], dev["A"], dev["C"], h0, None, 0.9, 1.0, y, hT, vT, maps, S, 0, L)
    monkeypatch.delenv("MMSCAN_FAULT_INJECT")
    _expect_timeout()
    _scan_check(dev, inp)


def test_backward_wait_runs_out(monkeypatch):
    inp = wl.scan_inputs(wl.SCAN_MEDIUM, batch=1, seqlen=256, dim=32)
    dev = _scan_dev(inp)
    y, hT, vT, ckpt = mm.scan_fwd_train(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.9)
    dy = torch.randn_like(dev["x"])
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "stall")
    mm.scan_bwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], ckpt, dy, beta=0.9)
    monkeypatch.delenv("MMSCAN_FAULT_INJECT")
    _expect_timeout()
    _scan_check(dev, inp)


def test_ssd_wait_runs_out(monkeypatch):
    inp = wl.ssd_inputs(wl.SSD_MH, batch=1, seqlen=256, nheads=2)
    dev = {"x": torch.from_numpy(inp["x"]).cuda().to(torch.bfloat16).contiguous(),
           "delta": torch.from_numpy(inp["delta"]).cuda().contiguous(),
           "A": torch.from_numpy(inp["A"]).cuda().contiguous(),
           "B": torch.from_numpy(inp["B"]).cuda().to(torch.bfloat16).contiguous(),
           "C": torch.from_numpy(inp["C"]).cuda().to(torch.bfloat16).contiguous()}
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "stall")
    mm.ssd_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], chunk=256)
    monkeypatch.delenv("MMSCAN_FAULT_INJECT")
    _expect_timeout()
    y, hT = mm.ssd_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], chunk=256)
    torch.cuda.synchronize()
    mm.mm_device_status()
    yr, hr, _ = oracle.ssd_seq(**inp, beta=0.0, alpha=1.0)
    yg = y.float().cpu().numpy()
    # oracle rows are lanes ((b * H + h) * P + p) over time
    Bsz, L, H, P = inp["x"].shape
    yg = yg.transpose(0, 2, 3, 1).reshape(Bsz * H * P, L)
    rel = np.linalg.norm(yg - yr) / np.linalg.norm(yr)
    assert rel <= 1e-2, f"SSD after a timeout: relative L2 {rel:.3e}"


def test_momentum_ssd_wait_runs_out(monkeypatch):
    inp = wl.ssd_inputs(wl.SSD_MH, batch=1, seqlen=256, nheads=2)
    dev = {"x": torch.from_numpy(inp["x"]).cuda().to(torch.bfloat16).contiguous(),
           "delta": torch.from_numpy(inp["delta"]).cuda().contiguous(),
           "A": torch.from_numpy(inp["A"]).cuda().contiguous(),
           "B": torch.from_numpy(inp["B"]).cuda().to(torch.bfloat16).contiguous(),
           "C": torch.from_numpy(inp["C"]).cuda().to(torch.bfloat16).contiguous()}
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "stall")
    mm.ssd_fwd_momentum(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.9)
    monkeypatch.delenv("MMSCAN_FAULT_INJECT")
    _expect_timeout()
    y, hT, vT = mm.ssd_fwd_momentum(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], beta=0.9)
    torch.cuda.synchronize()
    mm.mm_device_status()
    yr, hr, _ = oracle.ssd_seq(**inp, beta=0.9, alpha=1.0)
    yg = y.float().cpu().numpy()
    Bsz, L, H, P = inp["x"].shape
    yg = yg.transpose(0, 2, 3, 1).reshape(Bsz * H * P, L)
    rel = np.linalg.norm(yg - yr) / np.linalg.norm(yr)
    assert rel <= 1e-2, f"momentum SSD after a timeout: relative L2 {rel:.3e}"
