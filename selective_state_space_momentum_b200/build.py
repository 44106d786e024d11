"""Build libmmscan.so (the sm_100a CUDA kernels and the C ABI) in-tree.

    python -m selective_state_space_momentum_b200.build [--force]

Compiles every source under ``csrc/`` with nvcc for ``sm_100a`` only
(``-gencode arch=compute_100a,code=sm_100a``), links the CUDA runtime
statically, and writes ``libmmscan.so`` next to this file.  The library then
depends on no CUDA shared object at load time, so it can be loaded (to check
its exported symbols) on a machine without a GPU; compute calls need a B200.
Object files go to ``_build/`` and are reused while their sources are
unchanged.
"""
from __future__ import annotations

import argparse
import hashlib
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(PKG, "_build")
LIB_PATH = os.path.join(PKG, "libmmscan.so")
PROBE_SRC = os.path.join(PKG, "probe", "pipe_peaks.cu")
PROBE_LIB = os.path.join(PKG, "libmmprobe.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-Xptxas", "-warn-spills", *ARCH]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmmscan.so")


def _sources():
    out = []
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cpp")):
            out.append(os.path.join(CSRC, name))
    return out


def _headers_digest() -> str:
    h = hashlib.sha256()
    for d in (CSRC, INCLUDE):
        for name in sorted(os.listdir(d)):
            if name.endswith((".h", ".cuh")):
                with open(os.path.join(d, name), "rb") as f:
                    h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def _compile(src: str, hdr: str, extra: list[str], verbose: bool) -> str:
    with open(src, "rb") as f:
        key = hashlib.sha256(f.read() + hdr.encode() + " ".join(NVCC_FLAGS + extra).encode()).hexdigest()[:16]
    obj = os.path.join(BUILD_DIR, f"{os.path.basename(src)}.{key}.o")
    if os.path.exists(obj):
        return obj
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj + ".tmp"]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, flush=True)
    os.replace(obj + ".tmp", obj)
    return obj


def _link(objs: list[str], out: str, verbose: bool, force: bool) -> None:
    stamp = hashlib.sha256("|".join(objs).encode()).hexdigest()[:16]
    stamp_path = os.path.join(BUILD_DIR, os.path.basename(out) + ".stamp")
    if (not force and os.path.exists(out) and os.path.exists(stamp_path)
            and open(stamp_path).read() == stamp):
        return
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-lpthread", "-ldl", "-lrt"]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, out)
    with open(stamp_path, "w") as f:
        f.write(stamp)


def build_probe(force: bool = False, verbose: bool = False) -> str:
    """Compile libmmprobe.so (the pipe-throughput probes the benchmark uses); return its path."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    obj = _compile(PROBE_SRC, "", [], verbose)
    _link([obj], PROBE_LIB, verbose, force)
    return PROBE_LIB


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    """Compile and link libmmscan.so (and libmmprobe.so); return libmmscan's path."""
    extra = list(extra or [])
    os.makedirs(BUILD_DIR, exist_ok=True)
    if force:
        for name in os.listdir(BUILD_DIR):
            if name.endswith(".o"):
                os.remove(os.path.join(BUILD_DIR, name))
    hdr = _headers_digest()
    srcs = _sources()
    with ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, hdr, extra, verbose), srcs))
    _link(objs, LIB_PATH, verbose, force)
    build_probe(force=force, verbose=verbose)
    return LIB_PATH


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills per kernel")
    args = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if args.ptxas_info else []
    print(build(force=args.force or args.ptxas_info, verbose=args.verbose or args.ptxas_info, extra=extra))


if __name__ == "__main__":
    sys.exit(main())
