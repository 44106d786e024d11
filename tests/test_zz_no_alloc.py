"""mm_scan_fwd_noalloc: the forward scan for callers that cannot allocate.

Some callers cannot call cudaMalloc -- code inside a host framework that
owns every device allocation, a process whose device memory was reserved
once at start-up, a path that must not take cudaMalloc's device-wide
synchronisation.  mm_scan_fwd_noalloc gives them the scan with its
between-launch segment records in a fixed array inside the library.

The GPU test calls it through the C ABI twice in a row, on different inputs
(the second call finds the first call's records still in the shared array),
and compares each result with mm_scan_fwd's at the scan's fp32 tolerance:
max |y - y_ref| <= 1e-4 * max |y_ref|, likewise hT, vT.  The sizes span two
segments, so the second launch folds a record the first one wrote.  A CPU
test checks that sizes whose records exceed the array are refused before
anything is launched.

This file is collected last (its name sorts last), so that a run stopping at
the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import workloads as wl

torch = pytest.importorskip("torch")

F32_TOL = 1e-4


def _close(got, ref, what):
    g, r = got.float().cpu().numpy(), ref.float().cpu().numpy()
    err = np.abs(g - r).max()
    assert err <= F32_TOL * np.abs(r).max(), f"{what}: max abs difference {err:.3e} vs {np.abs(r).max():.3e}"


@pytest.mark.gpu
def test_no_alloc_scan_matches_mm_scan_fwd_on_two_calls_in_a_row():
    mm.mm_scan_set_path(0, 0)                 # mm_scan_fwd on its automatic path
    batch, L, D, N = 1, 32768, 2048, 16       # 2048 channels: 16384-step segments, two of them
    for call, seed in enumerate((101, 202)):
        inp = wl.scan_inputs(wl.SCAN_LONG, batch=batch, seqlen=L, dim=D, dstate=N, seed=seed)
        dev = {k: torch.from_numpy(v).cuda().contiguous() for k, v in inp.items()}
        rng = np.random.default_rng(seed)
        h0 = torch.from_numpy(rng.standard_normal((batch, D, N)).astype(np.float32)).cuda()
        v0 = torch.from_numpy((0.3 * rng.standard_normal((batch, D, N))).astype(np.float32)).cuda()
        y_ref, h_ref, v_ref = mm.scan_fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0=h0, v0=v0,
                                          beta=0.99, alpha=1.0)
        y = torch.empty_like(dev["x"])
        hT = torch.empty_like(h_ref)
        vT = torch.empty_like(v_ref)
        mm.mm_scan_fwd_noalloc(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], h0, v0, 0.99, 1.0,
                               y, hT, vT)
        torch.cuda.synchronize()
        mm.mm_device_status()
        _close(y, y_ref, f"call {call}: y")
        _close(hT, h_ref, f"call {call}: hT")
        _close(vT, v_ref, f"call {call}: vT")


def test_no_alloc_scan_refuses_sizes_beyond_its_scratch():
    # 2^20 steps of 2048 channels: 64 segments of 128 channel tiles, 33.7 MB of records
    lib = mm.load_library()
    dims = mm.ScanDims(1, 1 << 20, 2048, 16, mm.MM_F32)
    fake = [ctypes.c_void_p((k + 1) << 40) for k in range(8)]   # aligned, never dereferenced
    rc = lib.mm_scan_fwd_noalloc(fake[0], fake[1], fake[2], fake[3], fake[4], None, None, 0.9, 1.0, fake[5],
                                 fake[6], fake[7], ctypes.byref(dims), None)
    assert mm.STATUS_NAMES[rc] == "MM_ERR_UNSUPPORTED"
    msg = mm.mm_last_error()
    assert "33685504 bytes" in msg and "holds 8388608" in msg, msg
