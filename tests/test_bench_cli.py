"""bench.py's command line and JSON contract, on the CPU.

The reference arm (the fp64 oracle on the host cores) runs here; the GPU
arms are exercised by the GPU runs.  Also the argument checks and the
algorithmic byte counts the roofline divides by.
"""
import json
import os
import subprocess
import sys

import pytest

import bench
from selective_state_space_momentum_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REQUIRED = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config")


def _bench(*args, timeout=300):
    env = dict(os.environ, OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, timeout=timeout, cwd=ROOT, env=env)


@pytest.mark.parametrize("workload", ["small", "ssd"])
def test_reference_arm_prints_one_json_line(workload):
    r = _bench("--impl", "reference", "--workload", workload, "--steps", "2", "--warmup", "3",
               "--reference-budget", "2")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in REQUIRED:
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["cpu"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == bench.WORKLOADS[bench.ALIASES[workload]].name


@pytest.mark.parametrize("args", [
    ("--warmup", "2"),                                  # fewer than three warm-up steps
    ("--workload", "ssd", "--gated"),                  # the extras belong to the scan
    ("--workload", "ssd", "--backward"),
    ("--backward", "--impl", "reference"),             # the reference arm times the forward
    ("--deterministic",),                               # the fixed-order sums belong to the backward
    ("--workload", "decode", "--impl", "reference"),
])
def test_bad_arguments_are_refused(args):
    r = _bench(*args, timeout=120)
    assert r.returncode == 2, (args, r.stdout[-500:], r.stderr[-500:])


def test_algorithmic_bytes_match_the_workload_definitions():
    # x, delta, y once; B, C once; A; the final states (fp32 medium workload)
    assert bench.algorithmic_bytes(wl.SCAN_MEDIUM) == 152_928_256
    # bf16: half the streamed bytes
    assert bench.algorithmic_bytes(wl.SCAN_BF16) == 3 * 8 * 2048 * 4096 * 2 + 2 * 8 * 16 * 4096 * 2 \
        + 2048 * 16 * 4 + 2 * 8 * 2048 * 16 * 4
    # decode: h and v read and written (4 D N fp32 a request) dominate
    d = wl.DECODE
    assert bench.decode_bytes(d) > 4 * d.batch * d.dim * d.dstate * 4
    assert bench.decode_bytes(d) < 1.05 * 4 * d.batch * d.dim * d.dstate * 4
    # the backward moves every forward stream plus dy, dx, ddelta and the checkpoints
    assert bench.bwd_algorithmic_bytes(wl.SCAN_MEDIUM) > bench.algorithmic_bytes(wl.SCAN_MEDIUM)


def test_reference_arm_under_torchrun_runs_on_rank_zero_only():
    """Launched by torchrun with two ranks, rank 1 exits 0 at once with no
    output and rank 0 alone prints the reference line."""
    def run(rank):
        env = dict(os.environ, OMP_NUM_THREADS="2", RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT="29555")
        return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                               "--gpus", "2", "--workload", "small", "--steps", "2", "--warmup", "3",
                               "--reference-budget", "2"], capture_output=True, text=True, timeout=300,
                              cwd=ROOT, env=env)
    r1 = run(1)
    assert r1.returncode == 0 and r1.stdout.strip() == "", r1.stdout + r1.stderr[-1000:]
    r0 = run(0)
    assert r0.returncode == 0, r0.stderr[-2000:]
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["cpu_baseline"]["kind"] == "oracle"


def test_resized_workloads_keep_their_laws_and_change_their_name():
    w = bench.resized_workload(wl.SSD_MH, batch=16, seqlen=1024)
    assert (w.batch, w.seqlen, w.nheads, w.seed_index) == (16, 1024, wl.SSD_MH.nheads, wl.SSD_MH.seed_index)
    assert w.name == wl.SSD_MH.name + "_as_b16_l1024"
    s = bench.resized_workload(wl.SCAN_LONG, seqlen=8192)
    assert (s.batch, s.seqlen, s.split) == (1, 8192, 0)
    assert bench.measured_traffic("scan_fwd_kernel", s.name) is None     # no counters for another shape
    assert bench.resized_workload(wl.DECODE, batch=8).batch == 8
    with pytest.raises(ValueError):
        bench.resized_workload(wl.DECODE, seqlen=4)
    with pytest.raises(ValueError):
        bench.resized_workload(wl.SCAN_SMALL, batch=0)


def test_reference_arm_on_a_resized_workload():
    r = _bench("--impl", "reference", "--workload", "small", "--batch", "2", "--seqlen", "64",
               "--steps", "2", "--warmup", "3", "--reference-budget", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["config"]["workload"] == wl.SCAN_SMALL.name + "_as_b2_l64"
    assert d["config"]["batch"] == 2 and d["config"]["seq_len"] == 64
    assert _bench("--workload", "decode", "--seqlen", "4", timeout=120).returncode == 2


def test_split_segment_length_gives_every_rank_a_full_round():
    # the long workload: 16384-step segments on one rank (eight of them); over eight
    # ranks, halved until each rank holds eight segments
    import selective_state_space_momentum_b200 as mm
    from selective_state_space_momentum_b200 import build as mmbuild
    mmbuild.build()
    w = wl.SCAN_LONG
    assert bench.split_seg_len(w, 1) == 16384
    assert bench.split_seg_len(w, 2) == 8192
    assert bench.split_seg_len(w, 8) == 2048
    assert bench.split_seg_len(w, 8, forced=4096) == 4096
    for world in (1, 2, 4, 8):
        S = bench.split_seg_len(w, world)
        pieces = mm.split_pieces(w.seqlen, world, S)
        assert all(n // S >= 8 for _, n in pieces)
