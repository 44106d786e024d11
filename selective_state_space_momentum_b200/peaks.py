"""Measured throughput of the execution pipes the scan kernels are bound by.

Runs the probes of ``libmmprobe.so`` (``probe/pipe_peaks.cu``) on the current
CUDA device and reports, per pipe, operations per second and operations per
SM clock cycle (using the SM clock sampled through NVML while the probe runs).
The benchmark divides a kernel's exponentials by the measured MUFU rate to
report its fraction of the roofline.

    python -m selective_state_space_momentum_b200.peaks
"""
from __future__ import annotations

import ctypes
import json
import os
import statistics
import threading
import time

_PKG = os.path.dirname(os.path.abspath(__file__))
PROBE_LIB = os.path.join(_PKG, "libmmprobe.so")
KINDS = {"ex2": 0, "ffma": 1, "ffma2": 2, "ex2_lowocc": 3, "ex2_ffma2x3_lowocc": 4}
SMS = 148


def _load():
    if not os.path.exists(PROBE_LIB):
        raise RuntimeError(f"{PROBE_LIB} is missing: build it with "
                           "`python -m selective_state_space_momentum_b200.build`")
    lib = ctypes.CDLL(PROBE_LIB)
    lib.mmprobe_launch.restype = ctypes.c_int
    lib.mmprobe_launch.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_void_p]
    lib.mmprobe_ops_per_thread_round.restype = ctypes.c_int
    return lib


class _Clock:
    """SM clock samples (MHz) through NVML in a background thread."""

    def __init__(self, index: int):
        self.index, self.samples, self.max_mhz = index, [], None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._n = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self._t = None
        return self

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._n.nvmlDeviceGetClockInfo(self._h, self._n.NVML_CLOCK_SM))
            except Exception:
                return
            time.sleep(0.002)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()
        return False

    def mhz(self):
        return statistics.median(self.samples) if self.samples else self.max_mhz


def measure(kinds=("ex2", "ffma", "ffma2"), target_ms: float = 25.0, reps: int = 5) -> dict:
    """Measure each pipe's rate on the current CUDA device; returns a dict per kind."""
    import torch
    lib = _load()
    dev = torch.cuda.current_device()
    props = torch.cuda.get_device_properties(dev)
    sms = props.multi_processor_count
    blocks, threads = sms * 8, 256
    out = torch.empty(blocks * threads, device="cuda", dtype=torch.float32)
    stream = torch.cuda.current_stream()
    k_ops = lib.mmprobe_ops_per_thread_round()
    res = {}
    for kind in kinds:
        code = KINDS[kind]

        def launch(iters):
            rc = lib.mmprobe_launch(code, out.data_ptr(), blocks, threads, iters, stream.cuda_stream)
            if rc != 0:
                raise RuntimeError(f"probe {kind}: CUDA error {rc}")

        # size the loop so that one launch takes about target_ms
        iters = 256
        launch(iters)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        launch(iters)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        iters = max(256, int(iters * target_ms / max(ms, 1e-3)))
        times = []
        with _Clock(dev) as clk:
            for _ in range(reps):
                e0.record(stream)
                launch(iters)
                e1.record(stream)
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
        ms = min(times)
        ops = float(blocks) * threads * iters * k_ops
        rate = ops / (ms * 1e-3)
        mhz = clk.mhz()
        res[kind] = {"ops_per_s": rate, "ms": ms, "ops": ops, "sm_mhz": mhz, "sm_max_mhz": clk.max_mhz,
                     "sms": sms,
                     "ops_per_clk_per_sm": (rate / (mhz * 1e6) / sms) if mhz else None}
    return res


def occupancy_sweep(warps_per_sm=(2, 4, 6, 8, 16), iters: int = 20000) -> dict:
    """MUFU ex2 per clock per SM with one-warp blocks at the given warps per
    SM, alone and with 3 dependent packed FMAs after each ex2 (8 chains per
    thread; the rate is taken at the max SM clock)."""
    import torch
    lib = _load()
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    out = torch.empty(sms * 16 * 32, device="cuda", dtype=torch.float32)
    stream = torch.cuda.current_stream()
    res = {}
    with _Clock(torch.cuda.current_device()) as clk:
        for kind in ("ex2_lowocc", "ex2_ffma2x3_lowocc"):
            for w in warps_per_sm:
                blocks = sms * w
                lib.mmprobe_launch(KINDS[kind], out.data_ptr(), blocks, 32, 100, stream.cuda_stream)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                rc = lib.mmprobe_launch(KINDS[kind], out.data_ptr(), blocks, 32, iters, stream.cuda_stream)
                e1.record(stream)
                torch.cuda.synchronize()
                if rc != 0:
                    raise RuntimeError(f"probe {kind}: CUDA error {rc}")
                ms = e0.elapsed_time(e1)
                ex2 = float(blocks) * 32 * iters * 8
                res[f"{kind}/{w}"] = ex2 / (ms * 1e-3) / sms
    mhz = clk.mhz()
    return {k: v / (mhz * 1e6) for k, v in res.items()} | {"sm_mhz": mhz}


def main():
    import argparse
    import torch
    ap = argparse.ArgumentParser(description="measured pipe rates of this GPU")
    ap.add_argument("--occupancy", action="store_true", help="MUFU rate against warps per SM")
    args = ap.parse_args()
    if not torch.cuda.is_available():
        raise SystemExit("no CUDA device")
    print(json.dumps(occupancy_sweep() if args.occupancy else measure(), indent=1))


if __name__ == "__main__":
    main()
