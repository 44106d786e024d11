"""fp64 CPU oracle for the Momentum Mamba forward scan and its SSD form.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
library (``selective_state_space_momentum_b200``) never imports, loads or
calls it, and it never imports the product: the two share no code.  The only
thing both sides consume is the seeded input arrays.

The arithmetic lives in ``mm_oracle.c`` (plain C, double precision, one time
step after another); this module compiles it with gcc into ``_build/`` and
marshals numpy arrays through ctypes.  Each wrapper's docstring names the
passage its C function follows; see the header of ``mm_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mm_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64
_f64 = ctypes.c_double


def build(force: bool = False, out_path: str | None = None,
          extra_flags: tuple[str, ...] = ()) -> str:
    """Compile mm_oracle.c with gcc -O2 -fopenmp into a shared library.

    Returns the library path.  ``extra_flags`` exist for tests that build a
    deliberately broken copy of the oracle (a planted mistake) to show that
    the pins catch it; the default build never passes any.
    """
    path = out_path or _LIB_PATH
    if not force and os.path.exists(path) and os.path.getmtime(path) >= os.path.getmtime(_SRC):
        return path
    os.makedirs(os.path.dirname(path), exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-shared", "-fPIC", "-std=c11", "-Wall", *extra_flags,
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


def _declare(lib):
    lib.oracle_scan_seq.restype = ctypes.c_int
    lib.oracle_scan_seq.argtypes = [
        _f32p, _f32p, _f32p, _f32p, _f32p, _f64p, _f64p, _f64, _f64,
        _i64, _i64, _i64, _i64, _i64p, _i64, _f64p, _f64p, _f64p]
    lib.oracle_scan_gated.restype = ctypes.c_int
    lib.oracle_scan_gated.argtypes = [
        _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, ctypes.c_int, _f64p, _f64p,
        _f64, _f64, _i64, _i64, _i64, _i64, _i64p, _i64, _f64p, _f64p, _f64p]
    lib.oracle_scan_bwd.restype = ctypes.c_int
    lib.oracle_scan_bwd.argtypes = [
        _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, ctypes.c_int, _f64p, _f64p,
        _f64, _f64, _f32p, _f64p, _f64p, _i64, _i64, _i64, _i64, _i64p, _i64, _i64p, _i64,
        _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p]
    lib.oracle_scan_chunked.restype = ctypes.c_int
    lib.oracle_scan_chunked.argtypes = [
        _f32p, _f32p, _f32p, _f32p, _f32p, _f64p, _f64p, _f64, _f64,
        _i64, _i64, _i64, _i64, _i64, _i64p, _i64, _f64p, _f64p, _f64p]
    lib.oracle_ssd_seq.restype = ctypes.c_int
    lib.oracle_ssd_seq.argtypes = [
        _f32p, _f32p, _f32p, _f32p, _f32p, _f64p, _f64p, _f64, _f64,
        _i64, _i64, _i64, _i64, _i64, _i64, _i64p, _i64, _f64p, _f64p, _f64p]
    lib.oracle_ssd_chunked.restype = ctypes.c_int
    lib.oracle_ssd_chunked.argtypes = [
        _f32p, _f32p, _f32p, _f32p, _f32p, _f64p, _f64, _f64,
        _i64, _i64, _i64, _i64, _i64, _i64, _i64, _f64p, _f64p]
    lib.oracle_ssd_chunked_momentum.restype = ctypes.c_int
    lib.oracle_ssd_chunked_momentum.argtypes = [
        _f32p, _f32p, _f32p, _f32p, _f32p, _f64p, _f64p, _f64, _f64,
        _i64, _i64, _i64, _i64, _i64, _i64, _i64, _f64p, _f64p, _f64p]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _f32(a, name):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a, a.ctypes.data_as(_f32p)


def _f32opt(a, shape, name):
    if a is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    if a.shape != tuple(shape):
        raise ValueError(f"{name}: shape {a.shape}, expected {tuple(shape)}")
    return a, a.ctypes.data_as(_f32p)


def _f64opt(a, shape, name):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float64)
    if a.shape != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {a.shape}")
    return a, a.ctypes.data_as(_f64p)


def _idx(a):
    if a is None:
        return None, None, 0
    a = np.ascontiguousarray(a, dtype=np.int64)
    return a, a.ctypes.data_as(_i64p), int(a.size)


def _check(rc, fn):
    if rc != 0:
        raise RuntimeError(f"{fn} failed with code {rc}")


def scan_seq(x, delta, A, B, C, h0=None, v0=None, beta=0.0, alpha=1.0,
             chan=None, lib=None):
    """Momentum scan, sequential definition (mm_oracle.c: oracle_scan_seq).

    Momentum Mamba README, "Momentum Mamba Recurrence" and "Discretization
    Note"; layouts of its "selective_scan_fn" section.  x, delta: (batch, dim,
    L); A: (dim, N); B, C: (batch, N, L); h0, v0: (batch, dim, N) or None.
    ``chan`` selects channels b*dim + d.  Returns fp64 (y, hT, vT) with y of
    shape (nchan, L) and states (nchan, N).
    """
    lib = lib or load()
    batch, dim, L = x.shape
    N = A.shape[1]
    xs, xp = _f32(x, "x")
    ds, dp = _f32(delta, "delta")
    As, Ap = _f32(A, "A")
    Bs, Bp = _f32(B, "B")
    Cs, Cp = _f32(C, "C")
    h0s, h0p = _f64opt(h0, (batch, dim, N), "h0")
    v0s, v0p = _f64opt(v0, (batch, dim, N), "v0")
    cs, cp, nc = _idx(chan)
    n = nc if chan is not None else batch * dim
    y = np.empty((n, L), np.float64)
    hT = np.empty((n, N), np.float64)
    vT = np.empty((n, N), np.float64)
    rc = lib.oracle_scan_seq(xp, dp, Ap, Bp, Cp, h0p, v0p, float(beta), float(alpha),
                             batch, L, dim, N, cp, nc,
                             y.ctypes.data_as(_f64p), hT.ctypes.data_as(_f64p),
                             vT.ctypes.data_as(_f64p))
    _check(rc, "oracle_scan_seq")
    return y, hT, vT


def scan_gated(x, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=False,
               h0=None, v0=None, beta=0.0, alpha=1.0, chan=None, lib=None):
    """The full selective_scan_fn forward (mm_oracle.c: oracle_scan_gated).

    Momentum Mamba README, "selective_scan_fn" (arguments D, z, delta_bias,
    delta_softplus); the gate as placed by "Mamba: Choosing What to Remember
    Based on the Input", "Where the state computation sits in a Mamba block".
    delta' = softplus(delta + delta_bias) (each part optional), the momentum
    recurrence with delta', then out = (y + D x) * silu(z).  D, delta_bias:
    (dim,) or None; z: (batch, dim, L) or None.  Returns fp64 (out, hT, vT)
    shaped as :func:`scan_seq`.
    """
    lib = lib or load()
    batch, dim, L = x.shape
    N = A.shape[1]
    xs, xp = _f32(x, "x")
    ds, dp = _f32(delta, "delta")
    As, Ap = _f32(A, "A")
    Bs, Bp = _f32(B, "B")
    Cs, Cp = _f32(C, "C")
    Ds, Dp = _f32opt(D, (dim,), "D")
    zs, zp = _f32opt(z, (batch, dim, L), "z")
    bs, bp = _f32opt(delta_bias, (dim,), "delta_bias")
    h0s, h0p = _f64opt(h0, (batch, dim, N), "h0")
    v0s, v0p = _f64opt(v0, (batch, dim, N), "v0")
    cs, cp, nc = _idx(chan)
    n = nc if chan is not None else batch * dim
    y = np.empty((n, L), np.float64)
    hT = np.empty((n, N), np.float64)
    vT = np.empty((n, N), np.float64)
    rc = lib.oracle_scan_gated(xp, dp, Ap, Bp, Cp, Dp, zp, bp, 1 if delta_softplus else 0,
                               h0p, v0p, float(beta), float(alpha), batch, L, dim, N, cp, nc,
                               y.ctypes.data_as(_f64p), hT.ctypes.data_as(_f64p),
                               vT.ctypes.data_as(_f64p))
    _check(rc, "oracle_scan_gated")
    return y, hT, vT


def scan_bwd(x, delta, A, B, C, dout, D=None, z=None, delta_bias=None, delta_softplus=False,
             h0=None, v0=None, dhT=None, dvT=None, beta=0.0, alpha=1.0, chan=None, bn=None,
             lib=None):
    """Gradients of the full selective_scan_fn forward (mm_oracle.c: oracle_scan_bwd).

    Momentum Mamba README, "Gradient Flow" and "Backward Pass: Reconstructed
    Forward + Reverse Scans", with the adjoint recursions derived from the
    forward recurrence (the C header states them).  ``dout`` is the gradient
    reaching the output (batch, dim, L); ``dhT``, ``dvT`` those reaching the
    final states (batch, dim, N) or None.  Returns a dict of fp64 arrays:
    dx, ddelta (and dz when z is given) (nchan, L); dh0, dv0 (nchan, N);
    dA (dim, N); dD, ddelta_bias (dim,); dB, dC (nbn, L).  ``chan`` selects
    channels b*dim + d for the per-channel results (dA, dD and ddelta_bias
    then sum only those); ``bn`` selects (b, n) rows b*N + n of dB and dC.
    """
    lib = lib or load()
    batch, dim, L = x.shape
    N = A.shape[1]
    xs, xp = _f32(x, "x")
    ds, dp = _f32(delta, "delta")
    As, Ap = _f32(A, "A")
    Bs, Bp = _f32(B, "B")
    Cs, Cp = _f32(C, "C")
    os_, op_ = _f32(dout, "dout")
    Ds, Dp = _f32opt(D, (dim,), "D")
    zs, zp = _f32opt(z, (batch, dim, L), "z")
    bs, bp = _f32opt(delta_bias, (dim,), "delta_bias")
    h0s, h0p = _f64opt(h0, (batch, dim, N), "h0")
    v0s, v0p = _f64opt(v0, (batch, dim, N), "v0")
    gTs, gTp = _f64opt(dhT, (batch, dim, N), "dhT")
    pTs, pTp = _f64opt(dvT, (batch, dim, N), "dvT")
    cs, cp, nc = _idx(chan)
    ks, kp, nk = _idx(bn)
    n = nc if chan is not None else batch * dim
    m = nk if bn is not None else batch * N
    out = {"dx": np.empty((n, L)), "ddelta": np.empty((n, L)), "dh0": np.empty((n, N)),
           "dv0": np.empty((n, N)), "dA": np.empty((dim, N)), "dD": np.empty(dim),
           "ddelta_bias": np.empty(dim), "dB": np.empty((m, L)), "dC": np.empty((m, L))}
    if z is not None:
        out["dz"] = np.empty((n, L))
    ptr = lambda k: out[k].ctypes.data_as(_f64p) if k in out else None
    rc = lib.oracle_scan_bwd(xp, dp, Ap, Bp, Cp, Dp, zp, bp, 1 if delta_softplus else 0,
                             h0p, v0p, float(beta), float(alpha), op_, gTp, pTp,
                             batch, L, dim, N, cp, nc, kp, nk,
                             ptr("dx"), ptr("ddelta"), ptr("dz"), ptr("dh0"), ptr("dv0"),
                             ptr("dA"), ptr("dD"), ptr("ddelta_bias"), ptr("dB"), ptr("dC"))
    _check(rc, "oracle_scan_bwd")
    return out


def scan_chunked(x, delta, A, B, C, h0=None, v0=None, beta=0.0, alpha=1.0,
                 chunk=64, chan=None, lib=None):
    """Momentum scan through per-chunk affine maps and a carry fold.

    mm_oracle.c: oracle_scan_chunked; Momentum Mamba README, "Forward Pass:
    Two-Stage Parallel Scan" (affine composition with a running prefix).
    Same arguments and results as :func:`scan_seq` plus the chunk length.
    """
    lib = lib or load()
    batch, dim, L = x.shape
    N = A.shape[1]
    xs, xp = _f32(x, "x")
    ds, dp = _f32(delta, "delta")
    As, Ap = _f32(A, "A")
    Bs, Bp = _f32(B, "B")
    Cs, Cp = _f32(C, "C")
    h0s, h0p = _f64opt(h0, (batch, dim, N), "h0")
    v0s, v0p = _f64opt(v0, (batch, dim, N), "v0")
    cs, cp, nc = _idx(chan)
    n = nc if chan is not None else batch * dim
    y = np.empty((n, L), np.float64)
    hT = np.empty((n, N), np.float64)
    vT = np.empty((n, N), np.float64)
    rc = lib.oracle_scan_chunked(xp, dp, Ap, Bp, Cp, h0p, v0p, float(beta), float(alpha),
                                 batch, L, dim, N, int(chunk), cp, nc,
                                 y.ctypes.data_as(_f64p), hT.ctypes.data_as(_f64p),
                                 vT.ctypes.data_as(_f64p))
    _check(rc, "oracle_scan_chunked")
    return y, hT, vT


def ssd_seq(x, delta, A, B, C, h0=None, v0=None, beta=0.0, alpha=1.0,
            lane=None, lib=None):
    """Multi-head scalar-A form, sequential definition (oracle_ssd_seq).

    Mamba-2 page, "Multi-Head Expansion", with the recurrence of the Momentum
    Mamba README.  x: (batch, L, H, P); delta: (batch, L, H); A: (H);
    B, C: (batch, L, G, N); h0, v0: (batch, H, P, N) or None.  ``lane``
    selects (b*H + h)*P + p.  Returns fp64 y (nlane, L) and hT, vT (nlane, N).
    """
    lib = lib or load()
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    xs, xp = _f32(x, "x")
    ds, dp = _f32(delta, "delta")
    As, Ap = _f32(A, "A")
    Bs, Bp = _f32(B, "B")
    Cs, Cp = _f32(C, "C")
    h0s, h0p = _f64opt(h0, (batch, H, P, N), "h0")
    v0s, v0p = _f64opt(v0, (batch, H, P, N), "v0")
    ls, lp, nl = _idx(lane)
    n = nl if lane is not None else batch * H * P
    y = np.empty((n, L), np.float64)
    hT = np.empty((n, N), np.float64)
    vT = np.empty((n, N), np.float64)
    rc = lib.oracle_ssd_seq(xp, dp, Ap, Bp, Cp, h0p, v0p, float(beta), float(alpha),
                            batch, L, H, P, N, G, lp, nl,
                            y.ctypes.data_as(_f64p), hT.ctypes.data_as(_f64p),
                            vT.ctypes.data_as(_f64p))
    _check(rc, "oracle_ssd_seq")
    return y, hT, vT


def ssd_chunked(x, delta, A, B, C, h0=None, alpha=1.0, chunk=256, lib=None):
    """The 4-step chunked SSD algorithm in fp64 (oracle_ssd_chunked).

    Mamba-2 page, "4-Step Algorithm" and its L_ij matrix form; plain
    recurrence (beta = 0).  Returns fp64 y (batch, L, H, P) and
    hT (batch, H, P, N).
    """
    lib = lib or load()
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    xs, xp = _f32(x, "x")
    ds, dp = _f32(delta, "delta")
    As, Ap = _f32(A, "A")
    Bs, Bp = _f32(B, "B")
    Cs, Cp = _f32(C, "C")
    h0s, h0p = _f64opt(h0, (batch, H, P, N), "h0")
    y = np.empty((batch, L, H, P), np.float64)
    hT = np.empty((batch, H, P, N), np.float64)
    rc = lib.oracle_ssd_chunked(xp, dp, Ap, Bp, Cp, h0p, 0.0, float(alpha),
                                batch, L, H, P, N, G, int(chunk),
                                y.ctypes.data_as(_f64p), hT.ctypes.data_as(_f64p))
    _check(rc, "oracle_ssd_chunked")
    return y, hT


def num_threads(lib=None) -> int:
    """OpenMP threads the oracle's channel loops use."""
    return int((lib or load()).oracle_num_threads())


def ssd_chunked_momentum(x, delta, A, B, C, h0=None, v0=None, beta=0.9, alpha=1.0, chunk=64, lib=None):
    """The momentum recurrence in the SSD chunked form
    (mm_oracle.c: oracle_ssd_chunked_momentum).

    Momentum Mamba README, "Momentum Mamba Recurrence", in the form of
    "Mamba-2 -- SSM = structured matrix multiply", "4-Step Algorithm": per
    chunk the mask M_ij = sum_{k=j}^{i} exp(cs_i - cs_k) beta^(k-j) and two
    carried states (h, v).  Layouts as :func:`ssd_seq`; returns fp64
    (y (batch, L, H, P), hT, vT (batch, H, P, N)).
    """
    lib = lib or load()
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    xs, xp = _f32(x, "x")
    ds, dp = _f32(delta, "delta")
    As, Ap = _f32(A, "A")
    Bs, Bp = _f32(B, "B")
    Cs, Cp = _f32(C, "C")
    h0s, h0p = _f64opt(h0, (batch, H, P, N), "h0")
    v0s, v0p = _f64opt(v0, (batch, H, P, N), "v0")
    y = np.empty((batch, L, H, P), np.float64)
    hT = np.empty((batch, H, P, N), np.float64)
    vT = np.empty((batch, H, P, N), np.float64)
    rc = lib.oracle_ssd_chunked_momentum(xp, dp, Ap, Bp, Cp, h0p, v0p, float(beta), float(alpha),
                                         batch, L, H, P, N, G, chunk, y.ctypes.data_as(_f64p),
                                         hT.ctypes.data_as(_f64p), vT.ctypes.data_as(_f64p))
    _check(rc, "oracle_ssd_chunked_momentum")
    return y, hT, vT
