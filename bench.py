"""Benchmark of the momentum selective scan on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one mm_scan_fwd call over one batch of the named workload (default:
the long streaming workload, fp32, batch 1, L 131072, D 2048, N 16,
beta 0.99, alpha 1.0 -- the largest scan configuration that one GPU holds),
i.e. every step of the scan: staging, discretisation, velocity and hidden
recurrences, read-out, final state.  Inputs are synthetic and seeded (see
workloads.py).

* value: state updates/s (batch * L * D * N per step, summed over ranks) with
  inputs resident in HBM, timed with CUDA events on the launching stream over
  exactly K steps between barriers; several input sets rotate so that the
  bytes a step reads were evicted from the 126 MB L2 by the steps before it.
* e2e: the same metric through the public host-memory call (mm_scan_fwd_host,
  mm_ssd_fwd_host): every step streams the inputs from pinned host memory
  through the device in time chunks, scans, and copies y, hT, vT back, with
  copy-in, kernels and copy-out overlapped (--host-chunk sets the chunk).
* roofline: the slower of the exponentials (one MUFU ex2 per state update)
  at the MUFU rate measured by libmmprobe (ex2 per clock per SM, scaled to
  148 SMs at the max SM clock) and the algorithmic bytes at the measured HBM
  copy bandwidth; for N = 16 the exponentials bind.
* cpu_baseline: the fp64 oracle on the host cores (rank 0, N = 1), on a
  bounded sample of the same workload.
* --impl reference: the oracle alone as the reference arm.
* --batch, --seqlen: the named workload resized (same value laws and seed;
  the workload name gains the new sizes), to see how a kernel's time
  depends on the shape at a fixed amount of work.

Multi-GPU (launched by torchrun): one process per GPU, each scanning its own
batch; there is no collective on the data path, only a barrier and a max of
the per-rank times (weak scaling).  With --split-l the ranks instead share
one sequence (strong scaling): each scans its piece of the time axis
(mm_scan_fwd_split_maps), the ranks all-gather their segment-map records
over NCCL, and each folds them into its piece (mm_scan_fwd_split_correct).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from selective_state_space_momentum_b200 import workloads as wl  # noqa: E402

METRIC = "selective-scan state updates/s (B·L·D·N) and % of roofline, 1×B200"
UNIT = "state updates/s"
MUFU_EX2_PER_CLK_PER_SM = 16
B200_SMS = 148
FALLBACK_SM_MAX_MHZ = 1965.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126e6

WORKLOADS = {w.name: w for w in wl.SCAN_WORKLOADS}
WORKLOADS[wl.SSD_MH.name] = wl.SSD_MH
WORKLOADS[wl.DECODE.name] = wl.DECODE
WORKLOADS[wl.SSD_MH_MOMENTUM.name] = wl.SSD_MH_MOMENTUM
ALIASES = {"small": wl.SCAN_SMALL.name, "medium": wl.SCAN_MEDIUM.name,
           "bf16": wl.SCAN_BF16.name, "long": wl.SCAN_LONG.name, "ssd": wl.SSD_MH.name,
           "decode": wl.DECODE.name, "ssd_momentum": wl.SSD_MH_MOMENTUM.name}
DEFAULT_WORKLOAD = wl.SCAN_LONG.name
IO_KEYS = ("x", "delta", "B", "C", "z")          # tensors in the workload's storage type
GATED_EXTRAS = "D skip, z SiLU gate, delta_bias, softplus"
FP32_LANES_PER_CLK_PER_SM = 128      # fp32 arithmetic lanes of one SM per clock
# fp32 operations one state update needs in the backward (an FMA counts as one):
# the forward rebuild (delta*A, w, v, h) and the reverse step (G, P, the two
# carries, B.P, a h_{t-1} G (two), A-weighted sum, dA, dB, dC), plus one ex2.
BWD_OPS_PER_UPDATE = 16


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes of one launch from the committed ncu summary (profiles/),
    or None when there is none for this workload or the kernel source has
    changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            recs = json.load(f).get(kernel)
        recs = recs if isinstance(recs, list) else [recs] if recs else []
        for rec in recs:
            if rec.get("workload") != workload:
                continue
            with open(os.path.join(ROOT, rec["source"]), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest()[:16] != rec["source_sha256_16"]:
                    return None
            # a path of several launches per call records their sum
            return float(rec.get("dram_bytes_per_step", rec.get("dram_bytes_per_launch")))
        return None
    except (OSError, ValueError, KeyError):
        return None


def resized_workload(w, batch=None, seqlen=None):
    """The workload with another batch and/or sequence length, same value
    laws and seed, under a name that says so (so no committed ncu counters
    of the original apply to it)."""
    if isinstance(w, wl.DecodeWorkload) and seqlen is not None:
        raise ValueError("a decode step has no sequence length")
    b = w.batch if batch is None else batch
    if b < 1 or (seqlen is not None and seqlen < 1):
        raise ValueError("--batch and --seqlen must be >= 1")
    if isinstance(w, wl.DecodeWorkload):
        return dataclasses.replace(w, batch=b, name=f"{w.name}_as_b{b}")
    L = w.seqlen if seqlen is None else seqlen
    extra = {"split": 0} if isinstance(w, wl.ScanWorkload) else {}
    return dataclasses.replace(w, batch=b, seqlen=L, name=f"{w.name}_as_b{b}_l{L}", **extra)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": FALLBACK_SM_MAX_MHZ}, "fallback"


def rotating_sets(step_bytes: int) -> int:
    """Input sets the timed steps rotate through, so that a step's bytes were
    evicted from L2 by the steps before it."""
    return min(4, max(2, math.ceil(2 * L2_BYTES / step_bytes) + 1))


def needs_flush(step_bytes: int) -> bool:
    """True when the rotating input sets together are too small to evict a
    step's bytes from L2: the steps are then timed one by one with L2 flushed
    in between."""
    return rotating_sets(step_bytes) * step_bytes < 2 * L2_BYTES


FLUSH_BYTES = 512 << 20


def l2_note(step_bytes: int, what: str = "input") -> str:
    n = rotating_sets(step_bytes)
    if needs_flush(step_bytes):
        return (f"{n} rotating {what} sets ({n * step_bytes / 1e6:.1f} MB) fit in L2: each step timed alone "
                f"between CUDA events, L2 flushed before it by writing {FLUSH_BYTES >> 20} MB")
    return f"{n} rotating {what} sets ({n * step_bytes / 1e6:.0f} MB) > 126 MB L2"


def timed_ms(step, steps: int, stream, step_bytes: int) -> float:
    """Device milliseconds of `steps` calls of step(i) on `stream` (CUDA
    events on that stream).  Inputs larger than L2 in rotation: one event pair
    around all steps.  Otherwise each step is timed alone, after a write of
    FLUSH_BYTES that evicts L2 (and keeps the GPU busy while the host queues
    the step); the sum of the per-step times is returned."""
    import torch
    # an NVTX range marks the timed steps for a profiler's timeline (ncu --nvtx)
    torch.cuda.nvtx.range_push(f"timed {steps} steps")
    try:
        return _timed_ms(step, steps, stream, step_bytes)
    finally:
        torch.cuda.nvtx.range_pop()


def _timed_ms(step, steps: int, stream, step_bytes: int) -> float:
    import torch
    if not needs_flush(step_bytes):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=stream.device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush.fill_(i & 0xff)
            evs[i][0].record(stream)
            step(i)
            evs[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs)


def scan_config(w, beta, alpha, world, gated=False):
    """The `config` of a scan forward line; the reference arm prints the same dict."""
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen, "dim": w.dim,
            "dstate": w.dstate, "beta": beta, "alpha": alpha, "io": w.io,
            "global_batch": w.batch * world, "parallelism": f"dp{world}",
            "l2": l2_note(algorithmic_bytes(w, gated)),
            **({"extras": GATED_EXTRAS} if gated else {})}


def ssd_config(w, world):
    """The `config` of an SSD line; the reference arm prints the same dict."""
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen, "nheads": w.nheads,
            "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups, "chunk": w.chunk,
            "beta": w.beta, "alpha": w.alpha, "global_batch": w.batch * world,
            "parallelism": f"dp{world}", "l2": l2_note(ssd_bytes(w))}


def mufu_peak_now(sm_max_mhz: float):
    """The MUFU ex2 rate measured now by libmmprobe (ex2 per clock per SM, at
    the clock sampled during the probe), scaled to the max SM clock; falls back
    to the 16 per clock per SM of the unit counts if the probe is missing."""
    try:
        from selective_state_space_momentum_b200 import peaks as pk
        r = pk.measure(("ex2",), target_ms=20.0, reps=3)["ex2"]
        per = float(r["ops_per_clk_per_sm"])
        return (per * B200_SMS * sm_max_mhz * 1e6,
                f"measured {per:.2f} ex2/clk/SM (libmmprobe, {r['sm_mhz']:.0f} MHz) x 148 SMs x {sm_max_mhz:.0f} MHz")
    except Exception as e:  # the probe library is built with the kernels; say so if it is absent
        return (MUFU_EX2_PER_CLK_PER_SM * B200_SMS * sm_max_mhz * 1e6,
                f"unit count 16 ex2/clk/SM x 148 SMs x {sm_max_mhz:.0f} MHz (probe unavailable: {e})")


def algorithmic_bytes(w: wl.ScanWorkload, gated: bool = False) -> int:
    """Bytes one call must move: x, delta, y once; B, C once; A; hT, vT; with
    the selective_scan_fn extras also z once and D, delta_bias."""
    eb = 4 if w.io == "f32" else 2
    bdl = w.batch * w.dim * w.seqlen
    extra = (bdl * eb + 2 * w.dim * 4) if gated else 0
    return 3 * bdl * eb + 2 * w.batch * w.dstate * w.seqlen * eb + w.dim * w.dstate * 4 \
        + 2 * w.batch * w.dim * w.dstate * 4 + extra


def bwd_algorithmic_bytes(w: wl.ScanWorkload, gated: bool = False) -> int:
    """Bytes the backward must move: x, delta, dy read and dx, ddelta written
    once; B, C read and dB, dC (fp32) written once; the checkpoints read once;
    A and dA; with the extras also z read and dz written, D, bias, dD, d bias."""
    eb = 4 if w.io == "f32" else 2
    bdl = w.batch * w.dim * w.seqlen
    bnl = w.batch * w.dstate * w.seqlen
    chunks = -(-w.seqlen // 16)
    extra = (2 * bdl * eb + 4 * w.dim * 4) if gated else 0
    return 5 * bdl * eb + 2 * bnl * eb + 2 * bnl * 4 + w.batch * w.dim * chunks * 2 * w.dstate * 4 \
        + 2 * w.dim * w.dstate * 4 + extra


def bwd_cpu_baseline(w: wl.ScanWorkload, beta: float, alpha: float, budget_s: float = 12.0,
                     gated: bool = False):
    """The fp64 oracle's backward (as it stands) on the first D' channels of
    batch row 0 (a whole backward of that slice: every gradient, dB and dC
    summed over the slice), D' sized to about `budget_s` of CPU time."""
    import oracle
    inp = wl.scan_inputs(w)
    if gated:
        ex = wl.scan_extras(w)
        inp["delta"] = ex["delta_raw"]
        inp.update(z=ex["z"], D=ex["D"], delta_bias=ex["delta_bias"])
    rng = np.random.default_rng(5)
    cores = oracle.num_threads()
    wall_budget = budget_s / max(cores, 1)

    def run(dd):
        sl = {k: (v[:1, :dd] if k in ("x", "delta", "z") else v[:1] if k in ("B", "C") else v[:dd])
              for k, v in inp.items()}
        dy = rng.standard_normal(sl["x"].shape).astype(np.float32)
        kw = dict(D=sl["D"], z=sl["z"], delta_bias=sl["delta_bias"], delta_softplus=True) if gated else {}
        t = time.perf_counter()
        oracle.scan_bwd(sl["x"], sl["delta"], sl["A"], sl["B"], sl["C"], dy, beta=beta, alpha=alpha, **kw)
        return time.perf_counter() - t

    probe = min(w.dim, 16)
    per_chan = run(probe) / probe
    dd = max(1, min(w.dim, int(wall_budget / max(per_chan, 1e-9))))
    dt = run(dd)
    return {"value": dd * w.seqlen * w.dstate / dt, "unit": UNIT, "cores": cores, "kind": "oracle", "cpu": cpu_model(),
            "sample": f"backward of channels 0..{dd - 1} of batch row 0 (all gradients"
                      f"{', D, z, delta_bias, softplus' if gated else ''}), beta={beta}, "
                      f"alpha={alpha}, fp64, {dt:.2f} s wall on {cores} threads"}


def run_scan_bwd(args, w, beta, alpha, rank, world):
    """Time mm_scan_bwd (the backward kernel) on resident inputs, checkpoints
    and output gradient; e2e adds the host copies of those in and of every
    gradient out."""
    import torch
    import selective_state_space_momentum_b200 as mm
    mm.mm_scan_set_deterministic(bool(args.deterministic))
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = wl.scan_inputs(w, seed=rank_seed(w.seed_index, rank))
    iodt = torch.float32 if w.io == "f32" else torch.bfloat16
    gen = torch.Generator().manual_seed(rank_seed(w.seed_index, rank) + 17)
    if args.gated:
        ex = wl.scan_extras(w, seed=rank_seed(w.seed_index, rank))
        inp["delta"] = ex["delta_raw"]
        inp.update(z=ex["z"], D=ex["D"], delta_bias=ex["delta_bias"])
    host = {k: torch.from_numpy(v).to(iodt if k in IO_KEYS else torch.float32) for k, v in inp.items()}
    host["dy"] = torch.randn(tuple(inp["x"].shape), generator=gen).to(iodt)
    step_bytes = bwd_algorithmic_bytes(w, args.gated)
    ext = dict(D=None, z=None, delta_bias=None, delta_softplus=False)
    nsets = rotating_sets(step_bytes)
    sets = []
    for _ in range(nsets):
        s = {k: v.to(dev).contiguous() for k, v in host.items()}
        if args.gated:
            ext = dict(D=s["D"], z=s["z"], delta_bias=s["delta_bias"], delta_softplus=True)
        _, _, _, s["ckpt"] = mm.scan_fwd_train(s["x"], s["delta"], s["A"], s["B"], s["C"], beta=beta,
                                               alpha=alpha, **ext)
        s["g"] = {"dx": torch.empty_like(s["x"]), "ddelta": torch.empty_like(s["x"]),
                  "dA": torch.empty((w.dim, w.dstate), device=dev),
                  "dB": torch.empty((w.batch, w.dstate, w.seqlen), device=dev),
                  "dC": torch.empty((w.batch, w.dstate, w.seqlen), device=dev),
                  "dD": torch.empty((w.dim,), device=dev) if args.gated else None,
                  "dz": torch.empty_like(s["x"]) if args.gated else None,
                  "ddelta_bias": torch.empty((w.dim,), device=dev) if args.gated else None}
        sets.append(s)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def bwd(s):
        g = s["g"]
        if args.gated:
            mm.mm_scan_bwd_gated(s["x"], s["delta"], s["A"], s["B"], s["C"], s["D"], s["z"], s["delta_bias"],
                                 True, None, None, beta, alpha, s["ckpt"], s["dy"], None, None, g["dx"],
                                 g["ddelta"], g["dA"], g["dB"], g["dC"], g["dD"], g["dz"], g["ddelta_bias"],
                                 None, None, stream)
        else:
            mm.mm_scan_bwd(s["x"], s["delta"], s["A"], s["B"], s["C"], None, None, beta, alpha, s["ckpt"],
                           s["dy"], None, None, g["dx"], g["ddelta"], g["dA"], g["dB"], g["dC"], None, None,
                           stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for i in range(args.warmup):
        bwd(sets[i % nsets])
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        ms_timed = timed_ms(lambda i: bwd(sets[i % nsets]), args.steps, stream, step_bytes)
    barrier()
    torch.cuda.synchronize()
    ms_step = max_over_ranks(ms_timed, dev) / args.steps
    value = whole_job_rate(w.updates, world, ms_step)

    # ---- end to end: host copies in, the backward, every gradient out ------
    e2e_steps = args.e2e_steps or max(3, min(20, args.steps))
    ck_host = sets[0]["ckpt"].cpu()
    pinned = {k: v.pin_memory() for k, v in host.items()}
    pinned["ckpt"] = ck_host.pin_memory()
    out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in sets[0]["g"].items()
           if v is not None}
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in out.values())

    def e2e_step():
        d = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
        ex = dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"], delta_softplus=True) if args.gated else {}
        g = mm.scan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["ckpt"], d["dy"], beta=beta,
                        alpha=alpha, stream=stream, **ex)
        for k in out:
            out[k].copy_(g[k], non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    barrier()

    if rank == 0:
        peaks, peak_kind = measured_peaks()
        clocks = clk.summary()
        sm_max = float(clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz") or FALLBACK_SM_MAX_MHZ)
        alu_peak = FP32_LANES_PER_CLK_PER_SM * B200_SMS * sm_max * 1e6
        achieved = w.updates * BWD_OPS_PER_UPDATE / (ms_step * 1e-3)
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        hbm_achieved = step_bytes / (ms_step * 1e-3) / 1e9
        line = {
            "metric": "selective-scan backward state updates/s (B·L·D·N) and % of roofline, 1×B200",
            "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.io, "data": "synthetic",
            "config": {"workload": w.name, "pass": "backward", **({"extras": GATED_EXTRAS} if args.gated else {}),
                       **({"sums": "deterministic"} if args.deterministic else {}),
                       "batch": w.batch, "seq_len": w.seqlen,
                       "dim": w.dim, "dstate": w.dstate, "beta": beta, "alpha": alpha, "io": w.io,
                       "global_batch": w.batch * world, "parallelism": f"dp{world}",
                       "l2": l2_note(step_bytes)},
            "roofline": {"bound": "alu", "kernel": "scan_bwd_kernel",
                         "achieved": achieved / 1e9, "peak": alu_peak / 1e9, "unit": "Gop/s",
                         "frac": achieved / alu_peak,
                         "traffic": (None if args.gated or args.deterministic
                                     else measured_traffic("scan_bwd_kernel", w.name)),
                         "peak_source": f"128 fp32 lanes/clk/SM x 148 SMs x {sm_max:.0f} MHz; "
                                        f"{BWD_OPS_PER_UPDATE} fp32 ops per state update",
                         "hbm": {"achieved": hbm_achieved, "peak": hbm_peak, "unit": "GB/s",
                                 "frac": hbm_achieved / hbm_peak, "peak_source": peak_kind,
                                 "algorithmic_bytes": step_bytes}},
            "e2e": {"value": whole_job_rate(w.updates, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            # the deterministic form adds the fixed-order sums as a second launch
            "gpu_launches": args.steps * (2 if args.deterministic else 1),
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = bwd_cpu_baseline(w, beta, alpha, gated=args.gated)
        print(json.dumps(line), flush=True)
    return 0


def decode_bytes(w: wl.DecodeWorkload) -> int:
    """Bytes one decode step must move: the cached h, v read and written
    once; x, delta, z read and y written; B, C; A, D, delta_bias."""
    eb = 4 if w.io == "f32" else 2
    bd = w.batch * w.dim
    return 4 * bd * w.dstate * 4 + 4 * bd * eb + 2 * w.batch * w.dstate * eb + w.dim * w.dstate * 4 \
        + 2 * w.dim * 4


def run_decode(args, w, rank, world):
    """Time mm_scan_step (one decode step for every request) on resident
    inputs and cached states; e2e adds the host copies of the step's inputs
    (x, delta, z, B, C) and of y back: the states stay on the device."""
    import torch
    import selective_state_space_momentum_b200 as mm
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = wl.decode_inputs(w, seed=rank_seed(w.seed_index, rank))
    iodt = torch.float32 if w.io == "f32" else torch.bfloat16
    io_keys = ("x", "delta", "z", "B", "C")
    host = {k: torch.from_numpy(v).to(iodt if k in io_keys else torch.float32) for k, v in inp.items()}
    step_bytes = decode_bytes(w)
    nsets = rotating_sets(step_bytes)
    sets = []
    for _ in range(nsets):
        s = {k: v.to(dev).contiguous() for k, v in host.items()}
        s["y"] = torch.empty_like(s["x"])
        sets.append(s)
    stream = torch.cuda.current_stream()

    def step(s):
        mm.mm_scan_step(s["x"], s["delta"], s["A"], s["B"], s["C"], s["D"], s["z"], s["delta_bias"], True,
                        s["h"], s["v"], w.beta, w.alpha, s["y"], stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for i in range(args.warmup):
        step(sets[i % nsets])
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        ms_timed = timed_ms(lambda i: step(sets[i % nsets]), args.steps, stream, step_bytes)
    barrier()
    torch.cuda.synchronize()
    ms_step = max_over_ranks(ms_timed, dev) / args.steps
    value = whole_job_rate(w.updates, world, ms_step)

    e2e_steps = args.e2e_steps or max(3, min(20, args.steps))
    pinned = {k: host[k].pin_memory() for k in io_keys}
    yhost = torch.empty(tuple(inp["x"].shape), dtype=iodt, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = yhost.numel() * yhost.element_size()
    s0 = sets[0]

    def e2e_step():
        d = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
        mm.mm_scan_step(d["x"], d["delta"], s0["A"], d["B"], d["C"], s0["D"], d["z"], s0["delta_bias"], True,
                        s0["h"], s0["v"], w.beta, w.alpha, s0["y"], stream)
        yhost.copy_(s0["y"], non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    barrier()

    if rank == 0:
        peaks, peak_kind = measured_peaks()
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        achieved = step_bytes / (ms_step * 1e-3) / 1e9
        line = {
            "metric": "decode-step state updates/s (B·D·N per step) and % of roofline, 1×B200",
            "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.io, "data": "synthetic",
            "config": {"workload": w.name, "pass": "decode step", "batch": w.batch, "seq_len": 1,
                       "dim": w.dim, "dstate": w.dstate, "beta": w.beta, "alpha": w.alpha, "io": w.io,
                       "extras": GATED_EXTRAS, "global_batch": w.batch * world,
                       "parallelism": f"dp{world}",
                       "l2": f"{nsets} rotating state sets ({nsets * step_bytes / 2e6:.0f} MB) > 126 MB L2"},
            "roofline": {"bound": "hbm", "kernel": "scan_step_kernel", "achieved": achieved,
                         "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                         "traffic": measured_traffic("scan_step_kernel", w.name),
                         "peak_source": f"{peak_kind} copy bandwidth", "algorithmic_bytes": step_bytes},
            "e2e": {"value": whole_job_rate(w.updates, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = decode_cpu_baseline(w)
        print(json.dumps(line), flush=True)
    return 0


def decode_cpu_baseline(w: wl.DecodeWorkload, budget_s: float = 12.0):
    """The fp64 oracle (one-step gated scan) on whole decode steps of the
    workload, as many as fit the CPU-time budget (at least one)."""
    import oracle
    inp = wl.decode_inputs(w)
    col = lambda a: a[..., None]
    cores = oracle.num_threads()

    def run():
        oracle.scan_gated(col(inp["x"]), col(inp["delta"]), inp["A"], col(inp["B"]), col(inp["C"]),
                          D=inp["D"], z=col(inp["z"]), delta_bias=inp["delta_bias"], delta_softplus=True,
                          h0=inp["h"].astype(np.float64), v0=inp["v"].astype(np.float64),
                          beta=w.beta, alpha=w.alpha)

    t = time.perf_counter()
    run()
    one = time.perf_counter() - t
    reps = max(1, min(20, int(budget_s / max(cores, 1) / max(one, 1e-9))))
    t = time.perf_counter()
    for _ in range(reps):
        run()
    dt = time.perf_counter() - t
    return {"value": reps * w.updates / dt, "unit": UNIT, "cores": cores, "kind": "oracle", "cpu": cpu_model(),
            "sample": f"{reps} whole decode step(s) of {w.batch} requests, fp64, {dt:.2f} s wall on {cores} threads"}


# ------------------------------------------------------------ clocks -------
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:  # no NVML: report that, do not fail the bench
            self.error = f"{type(e).__name__}: {e}"
        return self

    def _sample(self):
        n = self._nvml
        self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
        mask = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for bit, name in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()
            try:
                self._sample()
            except Exception:
                pass
        return False

    def summary(self):
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
               "samples": len(self.samples)}
        if self.error:
            out["error"] = self.error
        return out


# ------------------------------------------------------------ helpers ------
def split_seg_len(w: wl.ScanWorkload, world: int, forced: int = 0) -> int:
    """Segment length of the sequence split over `world` ranks: the
    sequence-split path's own length for the workload, halved until every
    rank holds at least eight segments (one round of a full cluster), never
    below one staged chunk."""
    import selective_state_space_momentum_b200 as mm
    if forced:
        return forced
    mm.mm_scan_set_path(2, 0)
    try:
        S = mm.mm_scan_segment_len(w.batch, w.seqlen, w.dim, w.dstate, 0 if w.io == "f32" else 1)
    finally:
        mm.mm_scan_set_path(0, 0)
    chunk = 32 if w.io == "f32" else 64
    while S > chunk and -(-w.seqlen // S) < 8 * world:
        S //= 2
    return S


def run_scan_split(args, w, beta, alpha, rank, world):
    """One sequence shared by the ranks along time (strong scaling): a step is
    the split's first launch on every rank's piece, the all-gather of the
    segment records (NCCL), and the second launch."""
    import torch
    import torch.distributed as dist
    import selective_state_space_momentum_b200 as mm
    dev = torch.device("cuda", torch.cuda.current_device())
    S = split_seg_len(w, world, args.seg_len)
    pieces = mm.split_pieces(w.seqlen, world, S)
    first, n = pieces[rank]
    io = mm.MM_F32 if w.io == "f32" else mm.MM_BF16
    iodt = torch.float32 if w.io == "f32" else torch.bfloat16
    per = pieces[0][1] // S if world > 1 else -(-w.seqlen // S)
    rec = mm.mm_scan_split_maps_size(w.batch, n, w.dim, w.dstate, 1, io)
    # every rank draws the whole sequence from one seed and keeps its piece
    inp = wl.scan_inputs(w, seed=rank_seed(w.seed_index, 0))
    host = {k: torch.from_numpy(np.ascontiguousarray(v[..., first:first + n]) if k in IO_KEYS else v)
            for k, v in inp.items()}
    del inp
    piece_bytes = algorithmic_bytes(w) * n // w.seqlen
    nsets = rotating_sets(piece_bytes)
    sets = []
    for _ in range(nsets):
        s = {k: host[k].to(dev).to(iodt if k in IO_KEYS else torch.float32).contiguous() for k in host}
        s["y"] = torch.empty_like(s["x"])
        s["hT"] = torch.empty((w.batch, w.dim, w.dstate), device=dev)
        s["vT"] = torch.empty_like(s["hT"])
        s["maps"] = torch.empty(per * rec, dtype=torch.uint8, device=dev)
        s["all"] = torch.empty(world * per * rec, dtype=torch.uint8, device=dev) if world > 1 else s["maps"]
        sets.append(s)
    stream = torch.cuda.current_stream()
    peers = (mm.SplitPeers(w.batch, w.dim, w.dstate, w.seqlen, S, io=io, device=dev)
             if args.exchange == "peers" else None)

    def step(i):
        s = sets[i % nsets]
        if peers is not None:
            dests, local = peers.next()
            mm.mm_scan_fwd_split_maps_peers(s["x"], s["delta"], s["A"], s["B"], s["C"], beta, alpha, s["y"],
                                            dests, S, first, w.seqlen, stream)
            peers.barrier()
            mm.mm_scan_fwd_split_correct(s["delta"], s["A"], s["C"], None, None, beta, alpha, s["y"], s["hT"],
                                         s["vT"], local, S, first, w.seqlen, stream)
            return
        mm.mm_scan_fwd_split_maps(s["x"], s["delta"], s["A"], s["B"], s["C"], beta, alpha, s["y"], s["maps"], S,
                                  stream)
        if world > 1:
            dist.all_gather_into_tensor(s["all"], s["maps"])
        mm.mm_scan_fwd_split_correct(s["delta"], s["A"], s["C"], None, None, beta, alpha, s["y"], s["hT"],
                                     s["vT"], s["all"], S, first, w.seqlen, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        ms_timed = timed_ms(step, args.steps, stream, piece_bytes)
    barrier()
    torch.cuda.synchronize()
    ms_step = max_over_ranks(ms_timed, dev) / args.steps
    updates = w.updates                        # the whole sequence, shared by the ranks
    value = updates / (ms_step * 1e-3)

    # ---- end to end: the piece from pinned host memory, the results back ----
    e2e_steps = args.e2e_steps or max(3, min(20, args.steps))
    pinned = {k: v.to(iodt if k in IO_KEYS else torch.float32).pin_memory() for k, v in host.items()}
    out = {"y": torch.empty(tuple(pinned["x"].shape), dtype=iodt, pin_memory=True),
           "hT": torch.empty((w.batch, w.dim, w.dstate), pin_memory=True),
           "vT": torch.empty((w.batch, w.dim, w.dstate), pin_memory=True)}
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in out.values())

    def e2e_step():
        d = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
        if peers is not None:
            y, hT, vT = mm.scan_fwd_split_peers(d["x"], d["delta"], d["A"], d["B"], d["C"], S, w.seqlen, peers,
                                                beta=beta, alpha=alpha)
        else:
            y, hT, vT = mm.scan_fwd_split(d["x"], d["delta"], d["A"], d["B"], d["C"], S, w.seqlen, beta=beta,
                                          alpha=alpha)
        out["y"].copy_(y, non_blocking=True)
        out["hT"].copy_(hT, non_blocking=True)
        out["vT"].copy_(vT, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    barrier()

    if rank == 0:
        peaks, peak_kind = measured_peaks()
        clocks = clk.summary()
        sm_max = float(clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz") or FALLBACK_SM_MAX_MHZ)
        mufu_peak, mufu_source = mufu_peak_now(sm_max)
        # the roofline of one rank's share: the slower of its exponentials (its piece,
        # once in the first launch) on its GPU's MUFU pipes and its piece's bytes on HBM
        share = updates * n / w.seqlen
        t_mufu = share / mufu_peak
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        t_hbm = piece_bytes / (hbm_peak * 1e9)
        note = "rank 0's piece; the step includes the record exchange and the carry-in corrections"
        if t_mufu >= t_hbm:
            roof = {"bound": "alu", "kernel": "scan_seg_kernel", "achieved": share / (ms_step * 1e-3) / 1e9,
                    "peak": mufu_peak / 1e9, "unit": "Gex2/s", "frac": t_mufu / (ms_step * 1e-3),
                    "peak_source": mufu_source, "traffic": None, "note": note}
        else:
            roof = {"bound": "hbm", "kernel": "scan_seg_kernel",
                    "achieved": piece_bytes / (ms_step * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                    "frac": t_hbm / (ms_step * 1e-3), "peak_source": f"{peak_kind} copy bandwidth",
                    "traffic": None, "note": note}
        cb = None
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(w, beta, alpha)
        cfg = scan_config(w, beta, alpha, 1)
        cfg.update(global_batch=w.batch, parallelism=f"sp{world}", l2=l2_note(piece_bytes, "piece"),
                   split={"seg_len": S, "pieces": [list(p) for p in pieces],
                          "exchange": ("none (one rank)" if world == 1 else
                                       "records stored by the first launch into every rank's buffer (CUDA IPC "
                                       "peer memory), NCCL all-reduce as the barrier"
                                       if args.exchange == "peers" else "NCCL all-gather")})
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": w.io, "data": "synthetic",
            "config": cfg, "roofline": roof,
            "e2e": {"value": updates / (e2e_ms * 1e-3), "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": 2 * args.steps,
            "clocks": clocks,
        }
        if cb is not None:
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    if peers is not None:
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()            # every rank is done with the others' buffers
        peers.close()
    return 0


def rank_seed(index: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling): a distinct, fixed seed."""
    return wl.seed_of(index) + 1000 * rank


def max_over_ranks(x: float, device) -> float:
    """Largest value of x over all ranks (the job's time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_per_step: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return units_per_rank * world / (ms_per_step * 1e-3)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), for the baseline records."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w: wl.ScanWorkload, beta: float, alpha: float, budget_s: float = 12.0,
                 gated: bool = False):
    """Time the fp64 oracle (as it stands) on whole passes over the workload,
    or on a channel slice of it when one pass would exceed the budget.
    `budget_s` is CPU time (wall time x the oracle's threads)."""
    import oracle
    inp = wl.scan_inputs(w)
    if gated:
        ex = wl.scan_extras(w)
        run_oracle = lambda **kw: oracle.scan_gated(
            inp["x"], ex["delta_raw"], inp["A"], inp["B"], inp["C"], D=ex["D"], z=ex["z"],
            delta_bias=ex["delta_bias"], delta_softplus=True, beta=beta, alpha=alpha, **kw)
    else:
        run_oracle = lambda **kw: oracle.scan_seq(**inp, beta=beta, alpha=alpha, **kw)
    nch = w.batch * w.dim
    cores = oracle.num_threads()
    wall_budget = budget_s / max(cores, 1)
    # calibrate on a small slice
    probe = np.arange(min(nch, 256), dtype=np.int64)
    t = time.perf_counter()
    run_oracle(chan=probe)
    per_chan = (time.perf_counter() - t) / len(probe)
    if per_chan * nch <= wall_budget:
        chans = None
        passes = max(1, min(50, int(wall_budget // max(per_chan * nch, 1e-9))))
        sample = f"{passes} full pass(es) over all {nch} channels"
    else:
        k = max(1, int(wall_budget / per_chan))
        chans, passes = np.linspace(0, nch - 1, k).astype(np.int64), 1
        sample = f"{k} of {nch} channels (evenly spaced), 1 pass"
    updates = (nch if chans is None else len(chans)) * w.seqlen * w.dstate * passes
    t = time.perf_counter()
    for _ in range(passes):
        run_oracle(chan=chans)
    dt = time.perf_counter() - t
    return {"value": updates / dt, "unit": UNIT, "cores": cores, "kind": "oracle", "cpu": cpu_model(),
            "sample": sample + f", beta={beta}, alpha={alpha}{', D, z, delta_bias, softplus' if gated else ''}, "
                      f"fp64, {dt:.2f} s wall on {cores} threads"}


def run_reference(args, w, beta=None, alpha=None):
    """The reference arm: the fp64 oracle as it stands, on the host cores.

    W warm-up and K timed steps, each on an evenly spaced, rotating subset of
    the workload's channels (scan) or (batch, head, channel) lanes (SSD),
    sized so that the whole run takes about `--reference-budget` seconds of
    wall time.  Rank 0 alone runs under torchrun; the others exit at once."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    ssd = isinstance(w, wl.SSDWorkload)
    if ssd:
        inp = wl.ssd_inputs(w)
        n_units = w.batch * w.nheads * w.headdim
        per_unit_updates = w.seqlen * w.dstate

        def run(sel):
            oracle.ssd_seq(**inp, beta=w.beta, alpha=w.alpha, lane=sel)
        config = ssd_config(w, args.gpus)
        unit_name = "(batch, head, channel) lanes"
    else:
        inp = wl.scan_inputs(w)
        n_units = w.batch * w.dim
        per_unit_updates = w.seqlen * w.dstate
        ex = wl.scan_extras(w) if args.gated else None

        def run(sel):
            if ex is None:
                oracle.scan_seq(**inp, beta=beta, alpha=alpha, chan=sel)
            else:
                oracle.scan_gated(inp["x"], ex["delta_raw"], inp["A"], inp["B"], inp["C"], D=ex["D"],
                                  z=ex["z"], delta_bias=ex["delta_bias"], delta_softplus=True,
                                  beta=beta, alpha=alpha, chan=sel)
        config = scan_config(w, beta, alpha, args.gpus, args.gated)
        unit_name = "channels"
    probe = np.arange(min(n_units, 64), dtype=np.int64)
    t = time.perf_counter()
    run(probe)
    per_unit = (time.perf_counter() - t) / len(probe)
    nsteps = args.steps + args.warmup
    k = int(max(1, min(n_units, args.reference_budget / nsteps / max(per_unit, 1e-9))))
    stride = max(1, n_units // k)

    def subset(i):
        return ((np.arange(k, dtype=np.int64) * stride + i) % n_units).astype(np.int64)
    for i in range(args.warmup):
        run(subset(i))
    t = time.perf_counter()
    for i in range(args.steps):
        run(subset(args.warmup + i))
    dt = time.perf_counter() - t
    value = args.steps * k * per_unit_updates / dt
    cb = {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle", "cpu": cpu_model(),
          "sample": f"{k} of {n_units} {unit_name} per step (evenly spaced, rotating), fp64"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": config, "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def ssd_algorithmic_flops(w: wl.SSDWorkload) -> float:
    """Tensor FLOPs of the chunked algorithm with chunk Q, full squares:
    C.B^T once per (batch, chunk) (groups share it), then per head the
    masked product with X, the chunk state and the read-out of the carried
    state."""
    nchunk = math.ceil(w.seqlen / w.chunk)
    Q, P, N = w.chunk, w.headdim, w.dstate
    per_bc = 2 * Q * Q * N * w.ngroups
    per_head = 2 * Q * Q * P + 2 * Q * N * P + 2 * Q * N * P
    return w.batch * nchunk * (per_bc + w.nheads * per_head)


def ssd_momentum_flops(w: wl.SSDWorkload) -> float:
    """Tensor FLOPs of the momentum chunked form with chunk Q, full squares:
    C.B^T once per (batch, chunk) (groups share it), then per head the masked
    product with X, the read-out of both carried states (h and v) and both
    chunk states."""
    nchunk = math.ceil(w.seqlen / w.chunk)
    Q, P, N = w.chunk, w.headdim, w.dstate
    per_bc = 2 * Q * Q * N * w.ngroups
    per_head = 2 * Q * Q * P + 4 * (2 * Q * N * P)
    return w.batch * nchunk * (per_bc + w.nheads * per_head)


def ssd_momentum_executed_flops(w: wl.SSDWorkload) -> float:
    """Tensor FLOPs the momentum kernel issues: per head and 128-row block,
    C.B^T (128x128x128), P.X, C.H^T, C.V^T, B^T.(w_H o X), B^T.(w_V o X)
    (128x64x128 each)."""
    nblk = math.ceil(w.seqlen / 128)
    return w.batch * w.nheads * nblk * (2 * 128 * 128 * 128 + 5 * 2 * 128 * 128 * 64)


def ssd_executed_flops(w: wl.SSDWorkload) -> float:
    """Tensor FLOPs the kernel issues: per head and 128-row block, C.B^T
    (128x128x128), M.X, B^T.Xhat and C.S^T (128x64x128 each)."""
    nblk = math.ceil(w.seqlen / 128)
    return w.batch * w.nheads * nblk * (2 * 128 * 128 * 128 + 3 * 2 * 128 * 128 * 64)


def ssd_bytes(w: wl.SSDWorkload) -> int:
    blh = w.batch * w.seqlen * w.nheads
    return 2 * blh * w.headdim * 2 + 2 * w.batch * w.seqlen * w.ngroups * w.dstate * 2 + blh * 4 \
        + w.batch * w.nheads * w.headdim * w.dstate * 4


def run_ssd(args, w, rank, world, local):
    import torch
    import selective_state_space_momentum_b200 as mm
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = wl.ssd_inputs(w, seed=rank_seed(w.seed_index, rank))
    host = {k: torch.from_numpy(v) for k, v in inp.items()}
    bf = {"x", "B", "C"}
    step_bytes = ssd_bytes(w)
    nsets = rotating_sets(step_bytes)
    sets = []
    for _ in range(nsets):
        st = {k: host[k].to(dev).to(torch.bfloat16 if k in bf else torch.float32).contiguous() for k in host}
        st["y"] = torch.empty_like(st["x"])
        st["hT"] = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), device=dev)
        sets.append(st)
    stream = torch.cuda.current_stream()

    mom = w.beta != 0.0
    for st in sets:
        st["vT"] = torch.empty_like(st["hT"]) if mom else None

    def step(i):
        st = sets[i % nsets]
        if mom:
            mm.mm_ssd_fwd_momentum(st["x"], st["delta"], st["A"], st["B"], st["C"], None, None, w.beta, w.alpha,
                                   st["y"], st["hT"], st["vT"], stream)
        else:
            mm.mm_ssd_fwd(st["x"], st["delta"], st["A"], st["B"], st["C"], None, 0.0, w.alpha,
                          st["y"], st["hT"], w.chunk, stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    mm.mm_device_status()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index if world == 1 else local) as clk:
        ms_timed = timed_ms(step, args.steps, stream, step_bytes)
    mm.mm_device_status()
    barrier()
    ms_total = max_over_ranks(ms_timed, dev)
    ms_step = ms_total / args.steps
    value = whole_job_rate(w.updates, world, ms_step)

    # end to end from pinned host memory
    pinned = {k: v.to(torch.bfloat16 if k in bf else torch.float32).pin_memory() for k, v in host.items()}
    out_y = torch.empty(tuple(inp["x"].shape), dtype=torch.bfloat16, pin_memory=True)
    out_h = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_y.numel() * 2 + out_h.numel() * 4
    e2e_steps = args.e2e_steps or max(3, min(20, args.steps))

    def e2e_step():
        # mm_ssd_fwd_host: copy-in, the chunk's device call and copy-out overlapped
        mm.ssd_fwd_host(pinned["x"], pinned["delta"], pinned["A"], pinned["B"], pinned["C"],
                        beta=w.beta if mom else 0.0, alpha=w.alpha, chunk=w.chunk,
                        out={"y": out_y, "hT": out_h}, stream=stream, chunk_steps=args.host_chunk)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    barrier()
    if rank == 0:
        peaks, peak_kind = measured_peaks()
        tf_peak = float(peaks.get("bf16_tflops", 1590.0))
        alg = ssd_algorithmic_flops(w)
        exe = ssd_executed_flops(w)
        achieved = alg / (ms_step * 1e-3) / 1e12
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        hbm_achieved = step_bytes / (ms_step * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": ssd_config(w, world),
            "roofline": {"bound": "tensor", "kernel": "ssd_fwd_kernel", "achieved": achieved,
                         "peak": tf_peak, "unit": "TFLOP/s", "frac": achieved / tf_peak,
                         "traffic": measured_traffic("ssd_fwd_kernel", w.name),
                         "peak_source": f"{peak_kind} cuBLAS bf16 burst",
                         "algorithmic_flops": alg, "executed_flops": exe,
                         "executed_tflops": exe / (ms_step * 1e-3) / 1e12,
                         "hbm": {"achieved": hbm_achieved, "peak": hbm_peak, "unit": "GB/s",
                                 "frac": hbm_achieved / hbm_peak, "algorithmic_bytes": step_bytes}},
            "e2e": {"value": whole_job_rate(w.updates, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
        }
        if mom:        # the tensor-core momentum kernel: useful FLOPs of the momentum chunked form
            alg = ssd_momentum_flops(w)
            exe = ssd_momentum_executed_flops(w)
            achieved = alg / (ms_step * 1e-3) / 1e12
            line["roofline"].update({
                "kernel": "ssd_mom_tc_kernel", "achieved": achieved, "frac": achieved / tf_peak,
                "traffic": measured_traffic("ssd_mom_tc_kernel", w.name),
                "algorithmic_flops": alg, "executed_flops": exe,
                "executed_tflops": exe / (ms_step * 1e-3) / 1e12})
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = ssd_cpu_baseline(w)
        print(json.dumps(line), flush=True)
    return 0


def ssd_cpu_baseline(w: wl.SSDWorkload, budget_s: float = 12.0):
    """The fp64 oracle (sequential definition) on a sample of (b, h, p) lanes;
    `budget_s` is CPU time (wall time x the oracle's threads)."""
    import oracle
    inp = wl.ssd_inputs(w)
    nl = w.batch * w.nheads * w.headdim
    cores = oracle.num_threads()
    probe = np.arange(64, dtype=np.int64)
    t = time.perf_counter()
    oracle.ssd_seq(**inp, beta=w.beta, alpha=w.alpha, lane=probe)
    per = (time.perf_counter() - t) / len(probe)
    k = int(max(64, min(nl, budget_s / max(cores, 1) / max(per, 1e-9))))
    lanes = np.linspace(0, nl - 1, k).astype(np.int64)
    t = time.perf_counter()
    oracle.ssd_seq(**inp, beta=w.beta, alpha=w.alpha, lane=lanes)
    dt = time.perf_counter() - t
    return {"value": k * w.seqlen * w.dstate / dt, "unit": UNIT, "cores": cores, "kind": "oracle", "cpu": cpu_model(),
            "sample": f"{k} of {nl} (batch, head, channel) lanes, fp64, {dt:.2f} s wall on {cores} threads"}


# -------------------------------------------------------------- main -------
def main(argv=None):
    ap = argparse.ArgumentParser(description="momentum selective scan benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--beta", type=float, default=None)
    ap.add_argument("--alpha", type=float, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--host-chunk", type=int, default=0,
                    help="time steps per chunk of the host-buffer call in the e2e leg (0: automatic)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-budget", type=float, default=60.0,
                    help="wall seconds for the whole --impl reference run")
    ap.add_argument("--gated", action="store_true",
                    help="time mm_scan_fwd_gated with D, z, delta_bias and softplus (scan workloads)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward mm_scan_bwd (scan workloads)")
    ap.add_argument("--deterministic", action="store_true",
                    help="with --backward: the fixed-order sums of mm_scan_set_deterministic(1)")
    ap.add_argument("--tile", default=None, help="force SPTxWARPS[xTIME_LANES], e.g. 4x2 or 4x2x2 (tuning)")
    ap.add_argument("--path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="scan path: 0 automatic, 1 register-resident, 2 sequence-split, 3 sequence-split "
                         "as one fused launch (tuning)")
    ap.add_argument("--seg-len", type=int, default=0,
                    help="segment length of the sequence-split path (a multiple of 32; 0 automatic)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (exploration; renames the workload)")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="override the workload's sequence length (scan and SSD workloads)")
    ap.add_argument("--split-l", action="store_true",
                    help="scan workloads: the ranks share one sequence, split along time (strong scaling)")
    ap.add_argument("--exchange", default="gather", choices=["gather", "peers"],
                    help="--split-l: records all-gathered by NCCL, or stored by the first launch straight into "
                         "every rank's buffer (CUDA IPC peer memory) with a barrier")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[ALIASES.get(args.workload, args.workload)]
    if args.batch is not None or args.seqlen is not None:
        try:
            w = resized_workload(w, args.batch, args.seqlen)
        except ValueError as e:
            ap.error(str(e))
    if (args.gated or args.backward) and not isinstance(w, wl.ScanWorkload):
        ap.error("--gated and --backward apply to the scan workloads")
    if isinstance(w, wl.DecodeWorkload):
        if args.impl == "reference":
            ap.error("--impl reference times the forward scan")
        import torch
        rank, world, local = dist_env()
        if world > 1:
            import datetime
            import torch.distributed as dist
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            torch.cuda.set_device(0)
        rc = run_decode(args, w, rank, world)
        if world > 1:
            torch.distributed.destroy_process_group()
        return rc
    if args.backward and args.impl == "reference":
        ap.error("--impl reference times the forward")
    if args.deterministic and not args.backward:
        ap.error("--deterministic applies to --backward")
    if isinstance(w, wl.SSDWorkload):
        if args.impl == "reference":
            return run_reference(args, w)
        import torch
        rank, world, local = dist_env()
        if world > 1:
            import datetime
            import torch.distributed as dist
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            torch.cuda.set_device(0)
        rc = run_ssd(args, w, rank, world, local)
        if world > 1:
            torch.distributed.destroy_process_group()
        return rc
    default = (0.9, 1.0) if (0.9, 1.0) in w.runs else w.runs[0]
    beta = args.beta if args.beta is not None else default[0]
    alpha = args.alpha if args.alpha is not None else default[1]
    if args.impl == "reference":
        return run_reference(args, w, beta, alpha)

    import torch
    import selective_state_space_momentum_b200 as mm

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if args.backward:
        rc = run_scan_bwd(args, w, beta, alpha, rank, world)
        if world > 1:
            torch.distributed.destroy_process_group()
        return rc
    if args.split_l:
        if args.gated:
            ap.error("--split-l times the plain forward")
        rc = run_scan_split(args, w, beta, alpha, rank, world)
        if world > 1:
            torch.distributed.destroy_process_group()
        return rc
    dev = torch.device("cuda", torch.cuda.current_device())
    if args.tile:
        parts = [int(v) for v in args.tile.split("x")]
        mm.mm_scan_set_tile(parts[0], parts[1], parts[2] if len(parts) > 2 else 1)
    if args.path or args.seg_len:
        mm.mm_scan_set_path(args.path or 2, args.seg_len)

    # Each rank scans its own batch (seed offset by rank): weak scaling.
    inp = wl.scan_inputs(w, seed=rank_seed(w.seed_index, rank))
    iodt = torch.float32 if w.io == "f32" else torch.bfloat16
    if args.gated:
        ex = wl.scan_extras(w, seed=rank_seed(w.seed_index, rank))
        inp["delta"] = ex["delta_raw"]
        inp.update(z=ex["z"], D=ex["D"], delta_bias=ex["delta_bias"])
    host = {k: torch.from_numpy(v) for k, v in inp.items()}
    step_bytes = algorithmic_bytes(w, args.gated)
    # enough input sets that a step's bytes were evicted by the steps before it
    nsets = rotating_sets(step_bytes)
    sets = []
    for _ in range(nsets):
        s = {k: host[k].to(dev).to(iodt if k in IO_KEYS else torch.float32).contiguous()
             for k in host}
        s["y"] = torch.empty_like(s["x"])
        s["hT"] = torch.empty((w.batch, w.dim, w.dstate), device=dev)
        s["vT"] = torch.empty_like(s["hT"])
        sets.append(s)
    stream = torch.cuda.current_stream()

    def step(i):
        s = sets[i % nsets]
        if args.gated:
            mm.mm_scan_fwd_gated(s["x"], s["delta"], s["A"], s["B"], s["C"], s["D"], s["z"],
                                 s["delta_bias"], 1, None, None, beta, alpha, s["y"], s["hT"], s["vT"],
                                 None, stream)
        else:
            mm.mm_scan_fwd(s["x"], s["delta"], s["A"], s["B"], s["C"], None, None, beta, alpha,
                           s["y"], s["hT"], s["vT"], stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index if world == 1 else local) as clk:
        ms_timed = timed_ms(step, args.steps, stream, step_bytes)
    barrier()
    torch.cuda.synchronize()
    ms_total = max_over_ranks(ms_timed, dev)
    ms_step = ms_total / args.steps
    updates = w.updates
    value = whole_job_rate(updates, world, ms_step)

    # ---- end to end through the host-memory call -------------------------
    e2e_steps = args.e2e_steps or max(3, min(20, args.steps))
    pinned = {k: v.to(iodt if k in IO_KEYS else torch.float32).pin_memory()
              for k, v in host.items()}
    extras = dict(D=pinned["D"], z=pinned["z"], delta_bias=pinned["delta_bias"],
                  delta_softplus=True) if args.gated else {}
    out = {"y": torch.empty(tuple(inp["x"].shape), dtype=iodt, pin_memory=True),
           "hT": torch.empty((w.batch, w.dim, w.dstate), pin_memory=True),
           "vT": torch.empty((w.batch, w.dim, w.dstate), pin_memory=True)}
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in out.values())
    for _ in range(2):
        mm.scan_fwd_host(pinned["x"], pinned["delta"], pinned["A"], pinned["B"], pinned["C"],
                         beta=beta, alpha=alpha, out=out, stream=stream, chunk_steps=args.host_chunk, **extras)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        mm.scan_fwd_host(pinned["x"], pinned["delta"], pinned["A"], pinned["B"], pinned["C"],
                         beta=beta, alpha=alpha, out=out, stream=stream, chunk_steps=args.host_chunk, **extras)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    barrier()

    if rank == 0:
        peaks, peak_kind = measured_peaks()
        clocks = clk.summary()
        sm_max = float(clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz") or FALLBACK_SM_MAX_MHZ)
        mufu_peak, mufu_source = mufu_peak_now(sm_max)
        achieved = updates / (ms_step * 1e-3)      # one ex2 per update, per launch
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        hbm_achieved = step_bytes / (ms_step * 1e-3) / 1e9
        # the roofline is the slower of the exponentials on MUFU and the bytes on HBM
        t_mufu = updates / mufu_peak
        t_hbm = step_bytes / (hbm_peak * 1e9)
        kernel = ("scan_seg_kernel" if not args.gated and
                  mm.mm_scan_segment_len(w.batch, w.seqlen, w.dim, w.dstate, 0 if w.io == "f32" else 1) > 0
                  else "scan_fwd_kernel")
        # the sequence-split path runs two launches per call (fused: one, path 3)
        launches_per_step = 2 if kernel == "scan_seg_kernel" and args.path != 3 else 1
        if t_mufu >= t_hbm:
            roof = {"bound": "alu", "kernel": kernel, "achieved": achieved / 1e9, "peak": mufu_peak / 1e9,
                    "unit": "Gex2/s", "frac": t_mufu / (ms_step * 1e-3), "peak_source": mufu_source}
        else:
            roof = {"bound": "hbm", "kernel": kernel, "achieved": hbm_achieved, "peak": hbm_peak,
                    "unit": "GB/s", "frac": t_hbm / (ms_step * 1e-3), "peak_source": f"{peak_kind} copy bandwidth"}
        roof["traffic"] = None if args.gated else measured_traffic(kernel, w.name)
        if launches_per_step > 1:
            roof["launches_per_step"] = launches_per_step
            roof["note"] = ("two launches per call (main passes writing segment records, then folds and "
                            "corrections): achieved, frac and traffic cover both")
        roof["hbm"] = {"achieved": hbm_achieved, "peak": hbm_peak, "unit": "GB/s", "frac": hbm_achieved / hbm_peak,
                       "peak_source": peak_kind, "algorithmic_bytes": step_bytes}
        roof["mufu"] = {"achieved": achieved / 1e9, "peak": mufu_peak / 1e9, "unit": "Gex2/s",
                        "frac": achieved / mufu_peak, "peak_source": mufu_source}
        cb = None
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(w, beta, alpha, gated=args.gated)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.io, "data": "synthetic",
            "config": scan_config(w, beta, alpha, world, args.gated),
            "roofline": roof,
            "e2e": {"value": whole_job_rate(updates, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * launches_per_step,
            "clocks": clocks,
        }
        if cb is not None:
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
