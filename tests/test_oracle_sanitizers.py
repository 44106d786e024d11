"""The oracle built with AddressSanitizer and UndefinedBehaviorSanitizer and
driven through every entry point on random and ragged shapes (channel and
lane selections, odd chunk lengths, groups, all optional arguments): no
out-of-bounds access, no use of freed memory, no undefined behaviour in the
reference the parity tests trust.  Runs in a child process with the
sanitizer runtimes preloaded; skipped where gcc has no such runtimes."""
import os
import subprocess
import sys

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _runtime(name):
    r = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True)
    path = r.stdout.strip()
    return path if r.returncode == 0 and os.path.isabs(path) and os.path.exists(path) else None


def test_oracle_entry_points_under_sanitizers(tmp_path):
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not (asan and ubsan):
        pytest.skip("gcc sanitizer runtimes not available")
    lib = oracle.build(force=True, out_path=str(tmp_path / "liboracle_san.so"),
                       extra_flags=("-g", "-O1", "-fsanitize=address,undefined", "-fno-omit-frame-pointer",
                                    "-fno-sanitize-recover=undefined"))
    env = dict(os.environ, LD_PRELOAD=f"{asan} {ubsan}", ASAN_OPTIONS="detect_leaks=0", OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(HERE, "oracle_sanitizer_drive.py"), lib],
                       capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0 and "oracle under sanitizers: ok" in r.stdout, (r.stdout + r.stderr)[-3000:]
