"""B200-native Momentum Mamba selective scan (and its Mamba-2 SSD form).

Thin Python binding over ``libmmscan.so`` (include/mm_scan.h).  Functions
named like the C entry points (``mm_scan_fwd``, ``mm_ssd_fwd``, ...) only
marshal arguments: every step of the computation runs in the library's CUDA
kernels.  PyTorch provides device memory and streams.  There is no CPU
fallback: without the built library (``python -m
selective_state_space_momentum_b200.build``) every compute call raises.

Convenience wrappers allocate outputs:

* :func:`scan_fwd` -- ``(y, last_state, last_velocity)`` like the Momentum
  Mamba page's ``selective_scan_fn`` with D, z, delta_bias unset and no
  softplus on delta.
* :func:`ssd_fwd` -- ``(y, last_state)`` of the multi-head scalar-A form.
* :func:`scan_fwd_host` -- end-to-end call on host arrays (copies in, scan,
  copies out) for callers whose data lives in host memory.
* :func:`scan_fwd_split` -- one sequence cut into pieces over the ranks of a
  process group: each rank scans its piece, the ranks exchange their segment
  maps (all-gather), and each folds them into its piece's carry-in.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "MMError", "MM_F32", "MM_BF16", "load_library", "library_path",
    "mm_scan_fwd", "mm_scan_fwd_gated", "mm_scan_ckpt_size", "mm_scan_bwd", "mm_scan_bwd_gated",
    "mm_scan_step", "mm_ssd_fwd", "mm_ssd_fwd_momentum", "ssd_fwd_momentum",
    "mm_status_string", "mm_last_error", "mm_scan_set_tile", "mm_version",
    "mm_scan_set_path", "mm_scan_segment_len", "mm_scan_set_deterministic",
    "mm_scan_fwd_host", "mm_scan_fwd_host_workspace_size", "mm_ssd_fwd_host",
    "mm_ssd_fwd_host_workspace_size",
    "mm_scan_split_maps_size", "mm_scan_fwd_split_maps", "mm_scan_fwd_split_correct",
    "mm_scan_fwd_noalloc", "mm_scan_fwd_split_maps_peers", "mm_ipc_get_handle", "mm_ipc_open_handle",
    "mm_ipc_close_handle", "SplitPeers", "mm_device_status", "scan_fwd", "scan_fwd_train", "scan_bwd", "ssd_fwd", "scan_fwd_host",
    "ssd_fwd_host", "split_pieces", "scan_fwd_split", "scan_fwd_split_peers",
    "EXPORTED_SYMBOLS", "MM_SCAN_CKPT_STEPS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libmmscan.so")
_lock = threading.Lock()
_lib = None

MM_F32 = 0
MM_BF16 = 1
MM_SCAN_CKPT_STEPS = 16     # steps between two checkpoints of the forward's state

STATUS_NAMES = {
    0: "MM_OK", 1: "MM_ERR_NULL", 2: "MM_ERR_DIMS", 3: "MM_ERR_SCALAR", 4: "MM_ERR_DTYPE",
    5: "MM_ERR_ALIGN", 6: "MM_ERR_UNSUPPORTED", 7: "MM_ERR_CUDA", 8: "MM_ERR_DEVICE_TIMEOUT",
    9: "MM_ERR_ALIAS",
}

# Every function include/mm_scan.h declares.
EXPORTED_SYMBOLS = ("mm_scan_fwd", "mm_scan_fwd_gated", "mm_scan_ckpt_size", "mm_scan_bwd",
                    "mm_scan_bwd_gated", "mm_scan_step", "mm_ssd_fwd_momentum",
                    "mm_ssd_fwd",
                    "mm_device_status",
                    "mm_status_string", "mm_last_error", "mm_scan_set_tile", "mm_version",
                    "mm_scan_set_path", "mm_scan_segment_len", "mm_scan_set_deterministic",
                    "mm_scan_fwd_host_workspace_size", "mm_scan_fwd_host",
                    "mm_ssd_fwd_host_workspace_size", "mm_ssd_fwd_host",
                    "mm_scan_split_maps_size", "mm_scan_fwd_split_maps", "mm_scan_fwd_split_correct",
                    "mm_scan_fwd_noalloc", "mm_scan_fwd_split_maps_peers", "mm_ipc_get_handle",
                    "mm_ipc_open_handle", "mm_ipc_close_handle")


class MMError(RuntimeError):
    """A libmmscan call returned a status other than MM_OK."""

    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{where}: {self.name}: {detail}")


class ScanDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("io", ctypes.c_int32)]


class SSDDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64),
                ("ngroups", ctypes.c_int64), ("chunk", ctypes.c_int64)]


def library_path() -> str:
    return _LIB_PATH


def _declare(lib):
    vp, f = ctypes.c_void_p, ctypes.c_float
    lib.mm_scan_fwd.restype = ctypes.c_int
    lib.mm_scan_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, f, f, vp, vp, vp,
                                ctypes.POINTER(ScanDims), vp]
    lib.mm_scan_fwd_gated.restype = ctypes.c_int
    lib.mm_scan_fwd_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, f, f,
                                      vp, vp, vp, vp, ctypes.POINTER(ScanDims), vp]
    lib.mm_scan_ckpt_size.restype = ctypes.c_int
    lib.mm_scan_ckpt_size.argtypes = [ctypes.POINTER(ScanDims), ctypes.POINTER(ctypes.c_size_t)]
    lib.mm_scan_step.restype = ctypes.c_int
    lib.mm_scan_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, f, f, vp,
                                 ctypes.POINTER(ScanDims), vp]
    lib.mm_scan_bwd_gated.restype = ctypes.c_int
    lib.mm_scan_bwd_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, f, f, vp, vp,
                                      vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                      ctypes.POINTER(ScanDims), vp]
    lib.mm_scan_bwd.restype = ctypes.c_int
    lib.mm_scan_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, f, f, vp, vp, vp, vp,
                                vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(ScanDims), vp]
    lib.mm_ssd_fwd.restype = ctypes.c_int
    lib.mm_ssd_fwd.argtypes = [vp, vp, vp, vp, vp, vp, f, f, vp, vp, ctypes.POINTER(SSDDims), vp]
    lib.mm_ssd_fwd_momentum.restype = ctypes.c_int
    lib.mm_ssd_fwd_momentum.argtypes = [vp, vp, vp, vp, vp, vp, vp, f, f, vp, vp, vp,
                                        ctypes.POINTER(SSDDims), vp]
    i64, sz = ctypes.c_int64, ctypes.c_size_t
    lib.mm_scan_fwd_host_workspace_size.restype = ctypes.c_int
    lib.mm_scan_fwd_host_workspace_size.argtypes = [ctypes.POINTER(ScanDims), ctypes.c_int, i64,
                                                    ctypes.POINTER(sz)]
    lib.mm_scan_fwd_host.restype = ctypes.c_int
    lib.mm_scan_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, f, f, vp, vp, vp,
                                     vp, sz, i64, ctypes.POINTER(ScanDims), vp]
    lib.mm_ssd_fwd_host_workspace_size.restype = ctypes.c_int
    lib.mm_ssd_fwd_host_workspace_size.argtypes = [ctypes.POINTER(SSDDims), ctypes.c_int, i64,
                                                   ctypes.POINTER(sz)]
    lib.mm_ssd_fwd_host.restype = ctypes.c_int
    lib.mm_ssd_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, f, f, vp, vp, vp, vp, sz, i64,
                                    ctypes.POINTER(SSDDims), vp]
    lib.mm_scan_split_maps_size.restype = ctypes.c_int
    lib.mm_scan_split_maps_size.argtypes = [ctypes.POINTER(ScanDims), i64, ctypes.POINTER(sz)]
    lib.mm_scan_fwd_split_maps.restype = ctypes.c_int
    lib.mm_scan_fwd_split_maps.argtypes = [vp, vp, vp, vp, vp, f, f, vp, vp, i64, ctypes.POINTER(ScanDims), vp]
    lib.mm_scan_fwd_split_correct.restype = ctypes.c_int
    lib.mm_scan_fwd_split_correct.argtypes = [vp, vp, vp, vp, vp, f, f, vp, vp, vp, vp, i64, i64, i64,
                                              ctypes.POINTER(ScanDims), vp]
    lib.mm_scan_fwd_split_maps_peers.restype = ctypes.c_int
    lib.mm_scan_fwd_split_maps_peers.argtypes = [vp, vp, vp, vp, vp, f, f, vp, vp, ctypes.c_int, i64, i64, i64,
                                                 ctypes.POINTER(ScanDims), vp]
    lib.mm_ipc_get_handle.restype = ctypes.c_int
    lib.mm_ipc_get_handle.argtypes = [vp, vp, ctypes.POINTER(i64)]
    lib.mm_ipc_open_handle.restype = ctypes.c_int
    lib.mm_ipc_open_handle.argtypes = [vp, i64, ctypes.POINTER(ctypes.c_void_p)]
    lib.mm_ipc_close_handle.restype = ctypes.c_int
    lib.mm_ipc_close_handle.argtypes = [vp, i64]
    lib.mm_scan_fwd_noalloc.restype = ctypes.c_int
    lib.mm_scan_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, f, f, vp, vp, vp, ctypes.POINTER(ScanDims), vp]
    lib.mm_status_string.restype = ctypes.c_char_p
    lib.mm_status_string.argtypes = [ctypes.c_int]
    lib.mm_last_error.restype = ctypes.c_char_p
    lib.mm_last_error.argtypes = []
    lib.mm_scan_set_tile.restype = ctypes.c_int
    lib.mm_scan_set_tile.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.mm_scan_set_path.restype = ctypes.c_int
    lib.mm_scan_set_path.argtypes = [ctypes.c_int, ctypes.c_int64]
    lib.mm_scan_set_deterministic.restype = ctypes.c_int
    lib.mm_scan_set_deterministic.argtypes = [ctypes.c_int]
    lib.mm_scan_segment_len.restype = ctypes.c_int
    lib.mm_scan_segment_len.argtypes = [ctypes.POINTER(ScanDims), ctypes.POINTER(ctypes.c_int64)]
    lib.mm_version.restype = ctypes.c_int
    lib.mm_version.argtypes = []
    lib.mm_device_status.restype = ctypes.c_int
    lib.mm_device_status.argtypes = []
    return lib


def load_library(path: str | None = None):
    """Load libmmscan.so (raises if it has not been built)."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -m selective_state_space_momentum_b200.build` (needs nvcc)")
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _check(rc: int, where: str):
    if rc != 0:
        lib = load_library()
        raise MMError(rc, where, lib.mm_last_error().decode())


# ------------------------------------------------------- C-named calls -----
def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _io_code(dtype) -> int:
    import torch
    if dtype == torch.float32:
        return MM_F32
    if dtype == torch.bfloat16:
        return MM_BF16
    raise TypeError(f"unsupported storage type {dtype}; use float32 or bfloat16")


# Argument checks of the C-named calls.  The library sizes every operand
# from the sizes it is given and reads raw device pointers, so a tensor on the
# host, on another device, of another type or shape, or a strided view would
# be read wrongly or past its end; each call checks its tensors here first
# (TypeError for a wrong type, ValueError for the rest).
def _require(name, t, shape, dtypes, device, optional=False):
    import torch
    if t is None:
        if optional:
            return
        raise TypeError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}; expected {' or '.join(str(d) for d in dtypes)}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}; expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (call .contiguous() on views)")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, x on {device}")


def _lead(x, ndim, name="x"):
    """Check the tensor that fixes the call's sizes, device and storage type."""
    import torch
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(x).__name__}")
    if x.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(x.shape)}")
    _io_code(x.dtype)
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous (call .contiguous() on views)")
    return x.device, x.dtype


def _on_cuda(device):
    if device.type != "cuda":
        raise ValueError(f"the operands must be CUDA tensors (got device {device})")


def _on_host(device):
    if device.type != "cpu":
        raise ValueError(f"the host entry points take CPU tensors (got device {device})")


def _require_workspace(ws):
    import torch
    if not isinstance(ws, torch.Tensor) or ws.device.type != "cuda" or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return ws.numel() * ws.element_size()


def _require_scan(x, A, tensors, seq_dims=3, host=False):
    """x (batch, dim, L) -- or (batch, dim) for a decode step -- and A (dim, N)
    fix the sizes; `tensors` is a list of (name, tensor, kind, optional) with
    kind one of io (like x), io_bc (batch, N[, L]) in x's type, state
    (batch, dim, N) fp32, a (dim, N) fp32, vec (dim,) fp32, bc32 (batch, N, L)
    fp32, ckpt (batch, dim, ceil(L / 16), 2, N) fp32."""
    import torch
    load_library()            # no library: fail first, whatever the arguments
    dev, io = _lead(x, seq_dims)
    if not isinstance(A, torch.Tensor) or A.dim() != 2:
        raise ValueError("A must be a 2-D (dim, dstate) tensor")
    batch, dim = x.shape[0], x.shape[1]
    N = A.shape[1]
    _require("A", A, (dim, N), (torch.float32,), dev)
    f32 = (torch.float32,)
    tail = tuple(x.shape[2:])
    shapes = {"io": (tuple(x.shape), (io,)),
              "io_bc": ((batch, N) + tail, (io,)),
              "state": ((batch, dim, N), f32),
              "a": ((dim, N), f32),
              "vec": ((dim,), f32),
              "bc32": ((batch, N) + tail, f32)}
    if tail:
        shapes["ckpt"] = ((batch, dim, (tail[0] + MM_SCAN_CKPT_STEPS - 1) // MM_SCAN_CKPT_STEPS, 2, N), f32)
    for name, t, kind, optional in tensors:
        shape, dts = shapes[kind]
        _require(name, t, shape, dts, dev, optional)
    (_on_host if host else _on_cuda)(dev)


def _require_ssd(x, delta, A, B, C, y, states=(), host=False):
    import torch
    load_library()
    dev, io = _lead(x, 4)
    if io != torch.bfloat16:
        raise TypeError("the SSD path takes bf16 x, B, C and y")
    batch, L, H, P = x.shape
    if not isinstance(B, torch.Tensor) or B.dim() != 4:
        raise ValueError("B must be a 4-D (batch, L, G, N) tensor")
    G, N = B.shape[2], B.shape[3]
    bf, f32 = (torch.bfloat16,), (torch.float32,)
    _require("delta", delta, (batch, L, H), f32, dev)
    _require("A", A, (H,), f32, dev)
    _require("B", B, (batch, L, G, N), bf, dev)
    _require("C", C, (batch, L, G, N), bf, dev)
    _require("y", y, (batch, L, H, P), bf, dev)
    for name, t in states:
        _require(name, t, (batch, H, P, N), f32, dev, optional=True)
    (_on_host if host else _on_cuda)(dev)


def mm_scan_fwd(x, delta, A, B, C, h0, v0, beta, alpha, y, hT, vT, stream=None):
    """C entry point mm_scan_fwd on torch CUDA tensors (marshalling only).

    Shapes: x, delta, y (batch, dim, L); A (dim, N) fp32; B, C (batch, N, L);
    h0, v0, hT, vT (batch, dim, N) fp32 or None.  x, delta, B, C, y share one
    storage type (fp32 or bf16).  Raises MMError on a non-OK status.
    """
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("h0", h0, "state", True), ("v0", v0, "state", True), ("y", y, "io", False),
                         ("hT", hT, "state", True), ("vT", vT, "state", True)])
    batch, dim, L = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(x.dtype))
    rc = load_library().mm_scan_fwd(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0),
                                    _ptr(v0), float(beta), float(alpha), _ptr(y), _ptr(hT), _ptr(vT),
                                    ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_fwd")


def mm_scan_fwd_gated(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, v0, beta, alpha,
                      y, hT, vT, ckpt=None, stream=None):
    """C entry point mm_scan_fwd_gated (marshalling only): mm_scan_fwd plus the
    optional D (dim,) fp32, z (batch, dim, L) in the storage type of x,
    delta_bias (dim,) fp32, the softplus switch and the checkpoint output
    ckpt (batch, dim, ceil(L / 16), 2, N) fp32."""
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("D", D, "vec", True), ("z", z, "io", True), ("delta_bias", delta_bias, "vec", True),
                         ("h0", h0, "state", True), ("v0", v0, "state", True), ("y", y, "io", False),
                         ("hT", hT, "state", True), ("vT", vT, "state", True), ("ckpt", ckpt, "ckpt", True)])
    batch, dim, L = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(x.dtype))
    rc = load_library().mm_scan_fwd_gated(
        _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if delta_softplus else 0, _ptr(h0), _ptr(v0), float(beta), float(alpha), _ptr(y), _ptr(hT),
        _ptr(vT), _ptr(ckpt), ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_fwd_gated")


def mm_scan_ckpt_size(batch, seqlen, dim, dstate, io=MM_F32) -> int:
    """C entry point mm_scan_ckpt_size: bytes of the checkpoint buffer."""
    dims = ScanDims(batch, seqlen, dim, dstate, io)
    out = ctypes.c_size_t(0)
    _check(load_library().mm_scan_ckpt_size(ctypes.byref(dims), ctypes.byref(out)), "mm_scan_ckpt_size")
    return int(out.value)


def mm_scan_bwd(x, delta, A, B, C, h0, v0, beta, alpha, ckpt, dy, dhT, dvT,
                dx, ddelta, dA, dB, dC, dh0, dv0, stream=None):
    """C entry point mm_scan_bwd on torch CUDA tensors (marshalling only).

    Inputs as given to the forward, ckpt as the forward wrote it, dy (batch,
    dim, L) in the storage type of x, dhT, dvT (batch, dim, N) fp32 or None.
    Outputs: dx, ddelta like x; dA (dim, N), dB, dC (batch, N, L) fp32;
    dh0, dv0 (batch, dim, N) fp32 or None.
    """
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("h0", h0, "state", True), ("v0", v0, "state", True), ("ckpt", ckpt, "ckpt", True),
                         ("dy", dy, "io", False), ("dhT", dhT, "state", True), ("dvT", dvT, "state", True),
                         ("dx", dx, "io", False), ("ddelta", ddelta, "io", False), ("dA", dA, "a", False),
                         ("dB", dB, "bc32", False), ("dC", dC, "bc32", False), ("dh0", dh0, "state", True),
                         ("dv0", dv0, "state", True)])
    batch, dim, L = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(x.dtype))
    rc = load_library().mm_scan_bwd(
        _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0), _ptr(v0), float(beta),
        float(alpha), _ptr(ckpt), _ptr(dy), _ptr(dhT), _ptr(dvT), _ptr(dx), _ptr(ddelta), _ptr(dA),
        _ptr(dB), _ptr(dC), _ptr(dh0), _ptr(dv0), ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_bwd")


def mm_ssd_fwd(x, delta, A, B, C, h0, beta, alpha, y, hT, chunk, stream=None):
    """C entry point mm_ssd_fwd on torch CUDA tensors (marshalling only).

    x, y (batch, L, H, P) bf16; delta (batch, L, H) fp32; A (H) fp32;
    B, C (batch, L, G, N) bf16; h0, hT (batch, H, P, N) fp32 or None.
    """
    _require_ssd(x, delta, A, B, C, y, states=(("h0", h0), ("hT", hT)))
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dims = SSDDims(batch, L, H, P, N, G, chunk)
    rc = load_library().mm_ssd_fwd(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0),
                                   float(beta), float(alpha), _ptr(y), _ptr(hT),
                                   ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_ssd_fwd")


def mm_ssd_fwd_momentum(x, delta, A, B, C, h0, v0, beta, alpha, y, hT, vT, stream=None):
    """C entry point mm_ssd_fwd_momentum (marshalling only).  Layouts as
    mm_ssd_fwd; v0, vT (batch, H, P, N) fp32 or None."""
    _require_ssd(x, delta, A, B, C, y, states=(("h0", h0), ("v0", v0), ("hT", hT), ("vT", vT)))
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dims = SSDDims(batch, L, H, P, N, G, 64)
    rc = load_library().mm_ssd_fwd_momentum(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0),
                                            _ptr(v0), float(beta), float(alpha), _ptr(y), _ptr(hT),
                                            _ptr(vT), ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_ssd_fwd_momentum")


def mm_scan_fwd_host_workspace_size(batch, seqlen, dim, dstate, io=MM_F32, with_z=False, chunk_steps=0) -> int:
    """C entry point mm_scan_fwd_host_workspace_size: device bytes the host
    entry needs for these sizes."""
    dims = ScanDims(batch, seqlen, dim, dstate, io)
    out = ctypes.c_size_t(0)
    _check(load_library().mm_scan_fwd_host_workspace_size(ctypes.byref(dims), 1 if with_z else 0,
                                                          int(chunk_steps), ctypes.byref(out)),
           "mm_scan_fwd_host_workspace_size")
    return int(out.value)


def mm_scan_fwd_host(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, v0, beta, alpha,
                     y, hT, vT, workspace, chunk_steps=0, stream=None):
    """C entry point mm_scan_fwd_host (marshalling only): mm_scan_fwd_gated
    on CPU tensors (page-locked for overlap) through a CUDA workspace tensor
    of at least mm_scan_fwd_host_workspace_size bytes.  Queues the work on
    ``stream`` and returns; synchronise before reading y, hT, vT."""
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("D", D, "vec", True), ("z", z, "io", True), ("delta_bias", delta_bias, "vec", True),
                         ("h0", h0, "state", True), ("v0", v0, "state", True), ("y", y, "io", False),
                         ("hT", hT, "state", True), ("vT", vT, "state", True)], host=True)
    nbytes = _require_workspace(workspace)
    batch, dim, L = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(x.dtype))
    rc = load_library().mm_scan_fwd_host(
        _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if delta_softplus else 0, _ptr(h0), _ptr(v0), float(beta), float(alpha), _ptr(y), _ptr(hT),
        _ptr(vT), _ptr(workspace), nbytes, int(chunk_steps), ctypes.byref(dims),
        _stream_handle(stream))
    _check(rc, "mm_scan_fwd_host")


def mm_ssd_fwd_host_workspace_size(batch, seqlen, nheads, headdim, dstate, ngroups=1, chunk=256,
                                   momentum=False, chunk_steps=0) -> int:
    """C entry point mm_ssd_fwd_host_workspace_size."""
    dims = SSDDims(batch, seqlen, nheads, headdim, dstate, ngroups, chunk)
    out = ctypes.c_size_t(0)
    _check(load_library().mm_ssd_fwd_host_workspace_size(ctypes.byref(dims), 1 if momentum else 0,
                                                         int(chunk_steps), ctypes.byref(out)),
           "mm_ssd_fwd_host_workspace_size")
    return int(out.value)


def mm_ssd_fwd_host(x, delta, A, B, C, h0, v0, beta, alpha, y, hT, vT, workspace, chunk=256,
                    chunk_steps=0, stream=None):
    """C entry point mm_ssd_fwd_host (marshalling only): the SSD scan on CPU
    tensors (layouts as mm_ssd_fwd) through a CUDA workspace tensor."""
    _require_ssd(x, delta, A, B, C, y, states=(("h0", h0), ("v0", v0), ("hT", hT), ("vT", vT)), host=True)
    nbytes = _require_workspace(workspace)
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dims = SSDDims(batch, L, H, P, N, G, chunk)
    rc = load_library().mm_ssd_fwd_host(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0), _ptr(v0),
                                        float(beta), float(alpha), _ptr(y), _ptr(hT), _ptr(vT),
                                        _ptr(workspace), nbytes, int(chunk_steps), ctypes.byref(dims),
                                        _stream_handle(stream))
    _check(rc, "mm_ssd_fwd_host")


def mm_status_string(status: int) -> str:
    return load_library().mm_status_string(status).decode()


def mm_last_error() -> str:
    return load_library().mm_last_error().decode()


def mm_scan_set_tile(states_per_thread: int, warps_per_block: int, time_lanes: int = 1):
    _check(load_library().mm_scan_set_tile(states_per_thread, warps_per_block, time_lanes),
           "mm_scan_set_tile")


def mm_scan_set_path(path: int, seg_len: int = 0):
    """Force the scan path (0 automatic, 1 register-resident, 2 sequence-split)
    and the segment length (0 automatic)."""
    _check(load_library().mm_scan_set_path(int(path), int(seg_len)), "mm_scan_set_path")


def mm_scan_set_deterministic(on: bool):
    """C entry point mm_scan_set_deterministic: the backward's parameter
    gradients (dA, dB, dC, dD, d bias) summed in a fixed order, bit-identical
    between runs (True), or added atomically (False, the default)."""
    _check(load_library().mm_scan_set_deterministic(1 if on else 0), "mm_scan_set_deterministic")


def mm_scan_segment_len(batch, seqlen, dim, dstate, io=MM_F32) -> int:
    """C entry point mm_scan_segment_len: the segment length of the
    sequence-split path for these sizes (0 on the register-resident path)."""
    dims = ScanDims(batch, seqlen, dim, dstate, io)
    out = ctypes.c_int64(0)
    _check(load_library().mm_scan_segment_len(ctypes.byref(dims), ctypes.byref(out)), "mm_scan_segment_len")
    return int(out.value)


def mm_scan_split_maps_size(batch, seqlen, dim, dstate, segments, io=MM_F32) -> int:
    """C entry point mm_scan_split_maps_size: bytes of `segments` segment-map
    records of a split scan over (batch, dim)."""
    dims = ScanDims(batch, seqlen, dim, dstate, io)
    out = ctypes.c_size_t(0)
    _check(load_library().mm_scan_split_maps_size(ctypes.byref(dims), int(segments), ctypes.byref(out)),
           "mm_scan_split_maps_size")
    return int(out.value)


def _require_maps(name, maps, nbytes, device):
    import torch
    if not isinstance(maps, torch.Tensor) or maps.dtype != torch.uint8 or not maps.is_contiguous():
        raise TypeError(f"{name} must be a contiguous uint8 tensor")
    if maps.device != device:
        raise ValueError(f"{name} is on {maps.device}, x on {device}")
    if maps.numel() < nbytes:
        raise ValueError(f"{name} holds {maps.numel()} bytes; the call needs {nbytes}")


def mm_scan_fwd_split_maps(x, delta, A, B, C, beta, alpha, y, maps, seg_len, stream=None):
    """C entry point mm_scan_fwd_split_maps (marshalling only): the main pass
    of this rank's piece x, delta, B, C (shapes as mm_scan_fwd); y gets the
    zero-start read-out, `maps` (uint8, at least mm_scan_split_maps_size(...,
    ceil(L / seg_len)) bytes) the piece's segment records."""
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("y", y, "io", False)])
    batch, dim, L = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(x.dtype))
    if seg_len >= 1:
        need = mm_scan_split_maps_size(batch, L, dim, N, -(-L // int(seg_len)), dims.io)
        _require_maps("maps", maps, need, x.device)
    rc = load_library().mm_scan_fwd_split_maps(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), float(beta),
                                               float(alpha), _ptr(y), _ptr(maps), int(seg_len),
                                               ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_fwd_split_maps")


def mm_scan_fwd_split_maps_peers(x, delta, A, B, C, beta, alpha, y, dests, seg_len, seq_first, seqlen_total,
                                 stream=None):
    """C entry point mm_scan_fwd_split_maps_peers (marshalling only): the
    split's first launch storing each segment record straight into every
    buffer whose device pointer the int64 CUDA tensor `dests` holds."""
    import torch
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("y", y, "io", False)])
    if not isinstance(dests, torch.Tensor) or dests.dtype != torch.int64 or dests.dim() != 1 or \
            not dests.is_contiguous() or dests.device != x.device:
        raise TypeError("dests must be a contiguous 1-D int64 tensor of device pointers on x's device")
    batch, dim, L = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(x.dtype))
    rc = load_library().mm_scan_fwd_split_maps_peers(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), float(beta),
                                                     float(alpha), _ptr(y), _ptr(dests), int(dests.numel()),
                                                     int(seq_first), int(seg_len), int(seqlen_total),
                                                     ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_fwd_split_maps_peers")


MM_IPC_HANDLE_BYTES = 64


def mm_ipc_get_handle(t):
    """C entry point mm_ipc_get_handle: (handle bytes, byte offset) of a CUDA
    tensor's memory within the allocation that holds it."""
    buf = ctypes.create_string_buffer(MM_IPC_HANDLE_BYTES)
    off = ctypes.c_int64(0)
    _check(load_library().mm_ipc_get_handle(ctypes.c_void_p(t.data_ptr()), buf, ctypes.byref(off)),
           "mm_ipc_get_handle")
    return buf.raw, int(off.value)


def mm_ipc_open_handle(handle: bytes, offset: int) -> int:
    """C entry point mm_ipc_open_handle: a device pointer to another process's memory."""
    if len(handle) != MM_IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle is {MM_IPC_HANDLE_BYTES} bytes")
    out = ctypes.c_void_p(0)
    _check(load_library().mm_ipc_open_handle(ctypes.create_string_buffer(handle, MM_IPC_HANDLE_BYTES),
                                             int(offset), ctypes.byref(out)), "mm_ipc_open_handle")
    return int(out.value)


def mm_ipc_close_handle(ptr: int, offset: int):
    _check(load_library().mm_ipc_close_handle(ctypes.c_void_p(ptr), int(offset)), "mm_ipc_close_handle")


def mm_scan_fwd_split_correct(delta, A, C, h0, v0, beta, alpha, y, hT, vT, maps_all, seg_len, seq_first,
                              seqlen_total, stream=None):
    """C entry point mm_scan_fwd_split_correct (marshalling only): fold the
    whole sequence's records `maps_all` into this piece's carry-ins, add their
    response to y (mm_scan_fwd_split_maps' output) and write the final
    states of the whole sequence to hT, vT (or None)."""
    _require_scan(delta, A, [("C", C, "io_bc", False), ("h0", h0, "state", True), ("v0", v0, "state", True),
                             ("y", y, "io", False), ("hT", hT, "state", True), ("vT", vT, "state", True)])
    batch, dim, L = delta.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(delta.dtype))
    if seg_len >= 1:
        need = mm_scan_split_maps_size(batch, L, dim, N, -(-int(seqlen_total) // int(seg_len)), dims.io)
        _require_maps("maps_all", maps_all, need, delta.device)
    rc = load_library().mm_scan_fwd_split_correct(_ptr(delta), _ptr(A), _ptr(C), _ptr(h0), _ptr(v0),
                                                  float(beta), float(alpha), _ptr(y), _ptr(hT), _ptr(vT),
                                                  _ptr(maps_all), int(seg_len), int(seq_first),
                                                  int(seqlen_total), ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_fwd_split_correct")


def mm_scan_fwd_noalloc(x, delta, A, B, C, h0, v0, beta, alpha, y, hT, vT, stream=None):
    """C entry point mm_scan_fwd_noalloc (marshalling only): mm_scan_fwd for
    callers that cannot allocate device memory; the records between its two
    launches live in the library's fixed 8 MiB device array.  Shapes as
    mm_scan_fwd; hT, vT may not be h0, v0."""
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("h0", h0, "state", True), ("v0", v0, "state", True), ("y", y, "io", False),
                         ("hT", hT, "state", True), ("vT", vT, "state", True)])
    batch, dim, L = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(x.dtype))
    rc = load_library().mm_scan_fwd_noalloc(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0), _ptr(v0),
                                            float(beta), float(alpha), _ptr(y), _ptr(hT), _ptr(vT),
                                            ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_fwd_noalloc")


def mm_version() -> int:
    return int(load_library().mm_version())


def mm_device_status():
    """Synchronise the device; raise MMError if a kernel gave up a bounded wait."""
    _check(load_library().mm_device_status(), "mm_device_status")


# ------------------------------------------------------------ wrappers -----
def scan_fwd(x, delta, A, B, C, h0=None, v0=None, beta=0.9, alpha=1.0,
             return_last_state=True, stream=None, D=None, z=None, delta_bias=None,
             delta_softplus=False):
    """Allocate outputs and run mm_scan_fwd, or mm_scan_fwd_gated when any of
    D, z, delta_bias, delta_softplus is given; returns (y, hT, vT) (states
    None when ``return_last_state`` is False)."""
    import torch
    y = torch.empty_like(x)
    hT = vT = None
    if return_last_state:
        shape = (x.shape[0], x.shape[1], A.shape[1])
        hT = torch.empty(shape, device=x.device, dtype=torch.float32)
        vT = torch.empty(shape, device=x.device, dtype=torch.float32)
    if D is None and z is None and delta_bias is None and not delta_softplus:
        mm_scan_fwd(x, delta, A, B, C, h0, v0, beta, alpha, y, hT, vT, stream)
    else:
        mm_scan_fwd_gated(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, v0, beta, alpha,
                          y, hT, vT, None, stream)
    return y, hT, vT


def mm_scan_step(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h, v, beta, alpha, y,
                 stream=None):
    """C entry point mm_scan_step (marshalling only): one decode step.

    x, delta, z, y (batch, dim) and B, C (batch, N) in one storage type; A
    (dim, N), D, delta_bias (dim,) fp32; h, v (batch, dim, N) fp32, updated
    in place.
    """
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("D", D, "vec", True), ("z", z, "io", True), ("delta_bias", delta_bias, "vec", True),
                         ("h", h, "state", False), ("v", v, "state", False), ("y", y, "io", False)],
                  seq_dims=2)
    batch, dim = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, 1, dim, N, _io_code(x.dtype))
    rc = load_library().mm_scan_step(
        _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if delta_softplus else 0, _ptr(h), _ptr(v), float(beta), float(alpha), _ptr(y),
        ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_step")


def mm_scan_bwd_gated(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, v0, beta, alpha,
                      ckpt, dy, dhT, dvT, dx, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dh0, dv0,
                      stream=None):
    """C entry point mm_scan_bwd_gated (marshalling only): mm_scan_bwd through
    D, z, delta_bias and softplus, with the extra outputs dD, dz, ddelta_bias."""
    _require_scan(x, A, [("delta", delta, "io", False), ("B", B, "io_bc", False), ("C", C, "io_bc", False),
                         ("D", D, "vec", True), ("z", z, "io", True), ("delta_bias", delta_bias, "vec", True),
                         ("h0", h0, "state", True), ("v0", v0, "state", True), ("ckpt", ckpt, "ckpt", True),
                         ("dy", dy, "io", False), ("dhT", dhT, "state", True), ("dvT", dvT, "state", True),
                         ("dx", dx, "io", False), ("ddelta", ddelta, "io", False), ("dA", dA, "a", False),
                         ("dB", dB, "bc32", False), ("dC", dC, "bc32", False), ("dD", dD, "vec", True),
                         ("dz", dz, "io", True), ("ddelta_bias", ddelta_bias, "vec", True),
                         ("dh0", dh0, "state", True), ("dv0", dv0, "state", True)])
    batch, dim, L = x.shape
    N = A.shape[1]
    dims = ScanDims(batch, L, dim, N, _io_code(x.dtype))
    rc = load_library().mm_scan_bwd_gated(
        _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if delta_softplus else 0, _ptr(h0), _ptr(v0), float(beta), float(alpha), _ptr(ckpt), _ptr(dy),
        _ptr(dhT), _ptr(dvT), _ptr(dx), _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dz),
        _ptr(ddelta_bias), _ptr(dh0), _ptr(dv0), ctypes.byref(dims), _stream_handle(stream))
    _check(rc, "mm_scan_bwd_gated")


def scan_fwd_train(x, delta, A, B, C, h0=None, v0=None, beta=0.9, alpha=1.0, stream=None,
                   D=None, z=None, delta_bias=None, delta_softplus=False):
    """Forward that also keeps the checkpoints the backward restarts from:
    returns (y, hT, vT, ckpt), ckpt (batch, dim, ceil(L / 16), 2, N) fp32.
    D, z, delta_bias, delta_softplus as for scan_fwd."""
    import torch
    batch, dim, L = x.shape
    N = A.shape[1]
    y = torch.empty_like(x)
    hT = torch.empty((batch, dim, N), device=x.device, dtype=torch.float32)
    vT = torch.empty_like(hT)
    ckpt = torch.empty((batch, dim, (L + MM_SCAN_CKPT_STEPS - 1) // MM_SCAN_CKPT_STEPS, 2, N), device=x.device,
                       dtype=torch.float32)
    mm_scan_fwd_gated(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, v0, beta, alpha, y, hT, vT,
                      ckpt, stream)
    return y, hT, vT, ckpt


def scan_bwd(x, delta, A, B, C, ckpt, dy, h0=None, v0=None, dhT=None, dvT=None, beta=0.9,
             alpha=1.0, stream=None, D=None, z=None, delta_bias=None, delta_softplus=False):
    """Allocate the gradients and run mm_scan_bwd (mm_scan_bwd_gated when any
    of D, z, delta_bias, delta_softplus is given); returns a dict with dx,
    ddelta, dA, dB, dC, dh0, dv0 and, with the extras, dD, dz, ddelta_bias."""
    import torch
    batch, dim, L = x.shape
    N = A.shape[1]
    f32 = dict(device=x.device, dtype=torch.float32)
    g = {"dx": torch.empty_like(x), "ddelta": torch.empty_like(x), "dA": torch.empty((dim, N), **f32),
         "dB": torch.empty((batch, N, L), **f32), "dC": torch.empty((batch, N, L), **f32),
         "dh0": torch.empty((batch, dim, N), **f32), "dv0": torch.empty((batch, dim, N), **f32)}
    if D is None and z is None and delta_bias is None and not delta_softplus:
        mm_scan_bwd(x, delta, A, B, C, h0, v0, beta, alpha, ckpt, dy, dhT, dvT, g["dx"], g["ddelta"],
                    g["dA"], g["dB"], g["dC"], g["dh0"], g["dv0"], stream)
        return g
    g["dD"] = torch.empty((dim,), **f32)
    g["ddelta_bias"] = torch.empty((dim,), **f32)
    g["dz"] = torch.empty_like(x) if z is not None else None
    mm_scan_bwd_gated(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, v0, beta, alpha, ckpt, dy,
                      dhT, dvT, g["dx"], g["ddelta"], g["dA"], g["dB"], g["dC"], g["dD"], g["dz"],
                      g["ddelta_bias"], g["dh0"], g["dv0"], stream)
    return g


def ssd_fwd(x, delta, A, B, C, h0=None, alpha=1.0, chunk=256, return_last_state=True, stream=None):
    """Allocate outputs and run mm_ssd_fwd; returns (y, hT)."""
    import torch
    batch, L, H, P = x.shape
    N = B.shape[3]
    y = torch.empty_like(x)
    hT = torch.empty((batch, H, P, N), device=x.device, dtype=torch.float32) if return_last_state else None
    mm_ssd_fwd(x, delta, A, B, C, h0, 0.0, alpha, y, hT, chunk, stream)
    return y, hT


def ssd_fwd_momentum(x, delta, A, B, C, h0=None, v0=None, beta=0.9, alpha=1.0, stream=None):
    """Allocate outputs and run mm_ssd_fwd_momentum; returns (y, hT, vT)."""
    import torch
    batch, L, H, P = x.shape
    N = B.shape[3]
    y = torch.empty_like(x)
    hT = torch.empty((batch, H, P, N), device=x.device, dtype=torch.float32)
    vT = torch.empty_like(hT)
    mm_ssd_fwd_momentum(x, delta, A, B, C, h0, v0, beta, alpha, y, hT, vT, stream)
    return y, hT, vT


_ws_cache = {}


def _cached_workspace(device, nbytes):
    """A device workspace of at least ``nbytes`` per device, kept between
    calls (calls on one stream may share it; calls that may run at the same
    time on different streams must pass workspaces of their own)."""
    import torch
    dev = torch.device(device)
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    with _lock:
        ws = _ws_cache.get(dev.index)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
            _ws_cache[dev.index] = ws
    return ws


def scan_fwd_host(x, delta, A, B, C, h0=None, v0=None, beta=0.9, alpha=1.0, device="cuda",
                  out=None, stream=None, D=None, z=None, delta_bias=None, delta_softplus=False,
                  chunk_steps=0, workspace=None):
    """End-to-end scan of host (CPU, ideally page-locked) tensors through
    mm_scan_fwd_host: the sequence is streamed through the device in time
    chunks with copy-in, kernels and copy-out overlapped.  Results go to
    ``out`` (a dict of host tensors y, hT, vT; page-locked ones are allocated
    if None), returned after the stream has been synchronised."""
    import torch
    with torch.cuda.device(torch.device(device)):
        s = stream or torch.cuda.current_stream()
        batch, dim, L = x.shape
        N = A.shape[1]
        if out is None:
            out = {"y": torch.empty(x.shape, dtype=x.dtype, pin_memory=True),
                   "hT": torch.empty((batch, dim, N), dtype=torch.float32, pin_memory=True),
                   "vT": torch.empty((batch, dim, N), dtype=torch.float32, pin_memory=True)}
        if workspace is None:
            need = mm_scan_fwd_host_workspace_size(batch, L, dim, N, _io_code(x.dtype), z is not None,
                                                   chunk_steps)
            workspace = _cached_workspace(device, need)
        mm_scan_fwd_host(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, v0, beta, alpha,
                         out["y"], out.get("hT"), out.get("vT"), workspace, chunk_steps, s)
        s.synchronize()
    return out


def ssd_fwd_host(x, delta, A, B, C, h0=None, v0=None, beta=0.0, alpha=1.0, chunk=256, device="cuda",
                 out=None, stream=None, chunk_steps=0, workspace=None):
    """End-to-end SSD scan of host tensors through mm_ssd_fwd_host (the
    momentum form when beta > 0 or v0 is given).  Results go to ``out`` (y,
    hT and, with momentum, vT; page-locked ones allocated if None),
    returned after the stream has been synchronised."""
    import torch
    momentum = beta != 0.0 or v0 is not None
    with torch.cuda.device(torch.device(device)):
        s = stream or torch.cuda.current_stream()
        batch, L, H, P = x.shape
        G, N = B.shape[2], B.shape[3]
        if out is None:
            out = {"y": torch.empty(x.shape, dtype=x.dtype, pin_memory=True),
                   "hT": torch.empty((batch, H, P, N), dtype=torch.float32, pin_memory=True)}
            if momentum:
                out["vT"] = torch.empty((batch, H, P, N), dtype=torch.float32, pin_memory=True)
        if workspace is None:
            need = mm_ssd_fwd_host_workspace_size(batch, L, H, P, N, G, chunk, momentum, chunk_steps)
            workspace = _cached_workspace(device, need)
        mm_ssd_fwd_host(x, delta, A, B, C, h0, v0, beta, alpha, out["y"], out.get("hT"), out.get("vT"),
                        workspace, chunk, chunk_steps, s)
        s.synchronize()
    return out


# ------------------------------------------------- sequence split ---------
def split_pieces(seqlen_total: int, world: int, seg_len: int):
    """The pieces of a sequence of ``seqlen_total`` steps over ``world`` ranks:
    a list of (first step, steps), rank order.  Every piece but the last holds
    the same whole number of segments of ``seg_len`` steps; the last holds
    the rest.  Raises ValueError when a rank would get no step."""
    if seqlen_total < 1 or world < 1 or seg_len < 1:
        raise ValueError("seqlen_total, world and seg_len must be >= 1")
    nseg = -(-seqlen_total // seg_len)
    per = -(-nseg // world)
    pieces = []
    for r in range(world):
        lo = min(r * per * seg_len, seqlen_total)
        hi = min((r + 1) * per * seg_len, seqlen_total)
        if hi <= lo:
            raise ValueError(f"{seqlen_total} steps in segments of {seg_len} leave rank {r} of {world} "
                             "without a piece")
        pieces.append((lo, hi - lo))
    return pieces


def _all_gather_bytes(local, world, group):
    """Concatenate every rank's byte buffer in rank order.  NCCL gathers in
    device memory; a backend without CUDA support (gloo) goes through host
    memory."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return local
    out = torch.empty(world * local.numel(), dtype=torch.uint8, device=local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, local, group=group)
        return out
    parts = [torch.empty(local.numel(), dtype=torch.uint8) for _ in range(world)]
    dist.all_gather(parts, local.cpu(), group=group)
    out.copy_(torch.cat(parts))
    return out


def scan_fwd_split(x, delta, A, B, C, seg_len, seqlen_total, h0=None, v0=None, beta=0.9, alpha=1.0,
                   group=None, stream=None):
    """This rank's part of one scan whose sequence is cut over the ranks of
    ``group`` (a torch.distributed process group; None: the default group,
    or a single rank without one).  x, delta, B, C are this rank's piece,
    ``split_pieces(seqlen_total, world, seg_len)[rank]``; h0, v0 the state
    at step 0 of the whole sequence.  Returns (y of the piece, hT, vT of the
    whole sequence), equal bit for bit to one mm_scan_fwd over the whole
    sequence on the sequence-split path with segment length ``seg_len``."""
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        rank, world = dist.get_rank(group), dist.get_world_size(group)
    else:
        rank, world = 0, 1
    first, steps = split_pieces(int(seqlen_total), world, int(seg_len))[rank]
    if x.dim() != 3 or x.shape[2] != steps:
        raise ValueError(f"rank {rank} holds steps [{first}, {first + steps}): x must be (batch, dim, {steps})")
    batch, dim, _ = x.shape
    N = A.shape[1]
    io = _io_code(x.dtype)
    per = split_pieces(int(seqlen_total), world, int(seg_len))[0][1] // int(seg_len) if world > 1 else \
        -(-steps // int(seg_len))
    rec = mm_scan_split_maps_size(batch, steps, dim, N, 1, io)
    local = torch.empty(per * rec, dtype=torch.uint8, device=x.device)
    y = torch.empty_like(x)
    mm_scan_fwd_split_maps(x, delta, A, B, C, beta, alpha, y, local, seg_len, stream)
    if world > 1:
        # the collective runs on torch's current stream: order it after the launch
        if stream is not None:
            torch.cuda.current_stream(x.device).wait_stream(stream)
        gathered = _all_gather_bytes(local, world, group)
        if stream is not None:
            stream.wait_stream(torch.cuda.current_stream(x.device))
    else:
        gathered = local
    hT = torch.empty((batch, dim, N), device=x.device, dtype=torch.float32)
    vT = torch.empty_like(hT)
    mm_scan_fwd_split_correct(delta, A, C, h0, v0, beta, alpha, y, hT, vT, gathered, seg_len, first,
                              seqlen_total, stream)
    return y, hT, vT


class SplitPeers:
    """The records buffers of a split whose exchange is done by the first
    launch itself: every rank holds buffers of the whole sequence's records,
    and every rank's first launch stores its records into all ranks' buffers
    through peer pointers (CUDA IPC).  Two sets alternate from call to call:
    a rank's next first launch writes into the set no rank can still be
    reading (every rank passed the barrier of the call in between).
    Collective over ``group``: every rank builds it with the same sizes and
    makes the same calls.  ``close()`` releases the peer mappings."""

    def __init__(self, batch, dim, dstate, seqlen_total, seg_len, io=MM_F32, group=None, device=None):
        import torch
        import torch.distributed as dist
        self.group = group
        if dist.is_available() and dist.is_initialized():
            self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        else:
            self.rank, self.world = 0, 1
        device = device or torch.device("cuda", torch.cuda.current_device())
        nseg = -(-int(seqlen_total) // int(seg_len))
        self.nbytes = mm_scan_split_maps_size(batch, int(seqlen_total), dim, dstate, nseg, io)
        self.locals = [torch.empty(self.nbytes, dtype=torch.uint8, device=device) for _ in range(2)]
        self._opened = []
        self.dests = []
        for buf in self.locals:
            ptrs = [0] * self.world
            ptrs[self.rank] = buf.data_ptr()
            if self.world > 1:
                handles = [None] * self.world
                dist.all_gather_object(handles, mm_ipc_get_handle(buf), group=group)
                for r, (h, off) in enumerate(handles):
                    if r != self.rank:
                        ptrs[r] = mm_ipc_open_handle(h, off)
                        self._opened.append((ptrs[r], off))
            self.dests.append(torch.tensor(ptrs, dtype=torch.int64, device=device))
        self._turn = 0

    def next(self):
        """(device array of every rank's buffer, this rank's buffer) of the next call."""
        k = self._turn
        self._turn ^= 1
        return self.dests[k], self.locals[k]

    def barrier(self, stream=None):
        """Every rank's first launch has completed (stream-ordered for NCCL, on
        the host for a backend without CUDA support)."""
        import torch
        import torch.distributed as dist
        if self.world == 1:
            return
        dev = self.locals[0].device
        if dist.get_backend(self.group) == "nccl":
            # the collective runs on torch's current stream: order it after `stream`'s launch
            cur = torch.cuda.current_stream(dev)
            if stream is not None:
                cur.wait_stream(stream)
            flag = torch.zeros(1, device=dev)
            dist.all_reduce(flag, group=self.group)
            if stream is not None:
                stream.wait_stream(cur)
        else:
            torch.cuda.synchronize(dev)
            dist.barrier(group=self.group)

    def close(self):
        for p, off in self._opened:
            mm_ipc_close_handle(p, off)
        self._opened = []


def scan_fwd_split_peers(x, delta, A, B, C, seg_len, seqlen_total, peers, h0=None, v0=None, beta=0.9, alpha=1.0,
                         stream=None):
    """scan_fwd_split with the exchange folded into the first launch: each
    rank's records go straight into every rank's buffer (``peers``, a
    SplitPeers built for these sizes), a barrier, then the second launch on
    the local buffer.  Same results as scan_fwd_split, bit for bit."""
    import torch
    first, steps = split_pieces(int(seqlen_total), peers.world, int(seg_len))[peers.rank]
    if x.dim() != 3 or x.shape[2] != steps:
        raise ValueError(f"rank {peers.rank} holds steps [{first}, {first + steps}): x must be (batch, dim, {steps})")
    batch, dim, _ = x.shape
    N = A.shape[1]
    y = torch.empty_like(x)
    dests, local = peers.next()
    mm_scan_fwd_split_maps_peers(x, delta, A, B, C, beta, alpha, y, dests, seg_len, first, seqlen_total, stream)
    peers.barrier(stream)
    hT = torch.empty((batch, dim, N), device=x.device, dtype=torch.float32)
    vT = torch.empty_like(hT)
    mm_scan_fwd_split_correct(delta, A, C, h0, v0, beta, alpha, y, hT, vT, local, seg_len, first,
                              seqlen_total, stream)
    return y, hT, vT
