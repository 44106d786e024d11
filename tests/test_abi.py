"""CPU checks of the C ABI: the library loads, exports every function that
include/*.h declares, and rejects bad arguments on the host.

No test here launches anything: every call either fails a host-side check
(which returns before any CUDA call) or takes the fault-injection path that
returns MM_ERR_CUDA without launching.  Pointers are fake, aligned integers.
"""
import ctypes
import glob
import os
import re

import pytest

import selective_state_space_momentum_b200 as mm
from selective_state_space_momentum_b200 import build as mmbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mmbuild.build()
    return mm.load_library()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(mm_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_every_declared_function_is_exported(lib):
    declared = _declared_functions()
    assert declared, "no declarations found in include/*.h"
    assert declared == set(mm.EXPORTED_SYMBOLS)
    for name in declared:
        assert hasattr(lib, name), name


def test_library_needs_no_cuda_shared_object():
    path = mmbuild.build()
    out = os.popen(f"ldd {path}").read()
    assert "libcudart" not in out and "libcuda.so" not in out


def test_status_strings(lib):
    for code in range(10):
        assert lib.mm_status_string(code)
    assert mm.mm_version() >= 100


A16 = 1 << 20   # a fake, 16-byte aligned address


def _fake(k):
    return ctypes.c_void_p(A16 * (k + 1))


def _scan(lib, dims, beta=0.9, alpha=1.0, **over):
    args = dict(x=_fake(0), delta=_fake(1), A=_fake(2), B=_fake(3), C=_fake(4), h0=None, v0=None,
                y=_fake(5), hT=None, vT=None)
    args.update(over)
    return lib.mm_scan_fwd(args["x"], args["delta"], args["A"], args["B"], args["C"], args["h0"],
                           args["v0"], beta, alpha, args["y"], args["hT"], args["vT"],
                           ctypes.byref(dims) if dims is not None else None, None)


def D(batch=1, L=64, dim=8, N=16, io=0):
    return mm.ScanDims(batch, L, dim, N, io)


def test_scan_rejects_bad_arguments(lib):
    assert _scan(lib, None) == 1                                  # dims NULL
    assert _scan(lib, D(), x=None) == 1
    assert _scan(lib, D(), y=None) == 1
    assert _scan(lib, D(L=0)) == 2
    assert _scan(lib, D(batch=-1)) == 2
    assert _scan(lib, D(N=17)) == 6
    assert _scan(lib, D(io=7)) == 4
    assert _scan(lib, D(), beta=1.0) == 3
    assert _scan(lib, D(), beta=-0.1) == 3
    assert _scan(lib, D(), beta=float("nan")) == 3
    assert _scan(lib, D(), alpha=-1.0) == 3
    assert _scan(lib, D(), alpha=float("inf")) == 3
    assert _scan(lib, D(), x=ctypes.c_void_p(A16 + 4)) == 5      # misaligned
    assert "x is not 16-byte aligned" in mm.mm_last_error()


def test_scan_rejects_aliasing(lib):
    # y on top of delta
    assert _scan(lib, D(), y=_fake(1)) == 9
    # hT on top of A (sizes: A = 8*16*4 bytes)
    assert _scan(lib, D(), hT=_fake(2)) == 9
    # hT overlapping vT
    assert _scan(lib, D(), hT=_fake(6), vT=ctypes.c_void_p(A16 * 7 + 64)) == 9


def test_scan_fault_injection_returns_cuda_error(lib, monkeypatch):
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    # in-place streaming (hT == h0, vT == v0) is allowed and reaches the launch step
    rc = _scan(lib, D(), h0=_fake(6), hT=_fake(6), v0=_fake(7), vT=_fake(7))
    assert rc == 7
    assert "injected" in mm.mm_last_error()


def test_gated_checks_its_extras(lib, monkeypatch):
    dims = D(L=64, dim=8)
    def call(**over):
        a = dict(x=_fake(0), delta=_fake(1), A=_fake(2), B=_fake(3), C=_fake(4), D=None, z=None,
                 bias=None, sp=0, h0=None, v0=None, y=_fake(5), hT=None, vT=None, ckpt=None)
        a.update(over)
        return lib.mm_scan_fwd_gated(a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"],
                                     a["bias"], a["sp"], a["h0"], a["v0"], 0.9, 1.0, a["y"], a["hT"],
                                     a["vT"], a["ckpt"], ctypes.byref(dims), None)
    assert call(z=ctypes.c_void_p(A16 * 7 + 4)) == 5              # misaligned gate
    assert "z is not 16-byte aligned" in mm.mm_last_error()
    assert call(z=_fake(5)) == 9                                  # y on top of z
    assert call(D=_fake(5)) == 9                                  # y on top of D
    assert call(ckpt=_fake(5)) == 9                               # checkpoints on top of y
    assert call(ckpt=_fake(1)) == 9                               # ... or of an input
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    assert call(D=_fake(6), z=_fake(7), bias=_fake(8), sp=1, ckpt=_fake(9)) == 7  # passes every check


def test_ckpt_size(lib):
    dims = D(L=130, dim=8)          # 9 blocks of 16 steps
    size = ctypes.c_size_t(0)
    assert lib.mm_scan_ckpt_size(ctypes.byref(dims), ctypes.byref(size)) == 0
    assert size.value == dims.batch * 8 * 9 * 2 * dims.dstate * 4
    assert mm.mm_scan_ckpt_size(dims.batch, 130, 8, dims.dstate) == size.value
    assert lib.mm_scan_ckpt_size(ctypes.byref(D(L=0, dim=8)), ctypes.byref(size)) == 2


def test_bwd_checks_its_arguments(lib, monkeypatch):
    dims = D(L=200, dim=8)
    def call(**over):
        a = dict(x=_fake(0), delta=_fake(1), A=_fake(2), B=_fake(3), C=_fake(4), h0=None, v0=None,
                 ckpt=_fake(10), dy=_fake(11), dhT=None, dvT=None, dx=_fake(12), dd=_fake(13),
                 dA=_fake(14), dB=_fake(15), dC=_fake(16), dh0=None, dv0=None, beta=0.9)
        a.update(over)
        return lib.mm_scan_bwd(a["x"], a["delta"], a["A"], a["B"], a["C"], a["h0"], a["v0"], a["beta"],
                               1.0, a["ckpt"], a["dy"], a["dhT"], a["dvT"], a["dx"], a["dd"], a["dA"],
                               a["dB"], a["dC"], a["dh0"], a["dv0"], ctypes.byref(dims), None)
    assert call(dy=None) == 1
    assert call(ckpt=None) == 1                                   # needed past 16 steps
    assert "ckpt" in mm.mm_last_error()
    assert call(beta=1.0) == 3
    assert call(dB=ctypes.c_void_p(A16 * 15 + 8)) == 5
    assert call(dx=_fake(0)) == 9                                 # gradient over an input
    assert call(dC=_fake(15)) == 9                                # two gradients on one buffer
    assert call(dh0=_fake(10)) == 9                               # over the checkpoints
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    assert call() == 7                                            # passes every check
    assert call(ckpt=None, **{}) == 1
    short = D(L=16, dim=8)
    rc = lib.mm_scan_bwd(_fake(0), _fake(1), _fake(2), _fake(3), _fake(4), None, None, 0.5, 1.0,
                         None, _fake(11), None, None, _fake(12), _fake(13), _fake(14), _fake(15),
                         _fake(16), None, None, ctypes.byref(short), None)
    assert rc == 7                                                # one block: no checkpoint needed


def test_bwd_gated_checks_its_extras(lib, monkeypatch):
    dims = D(L=200, dim=8)
    def call(**over):
        a = dict(x=_fake(0), delta=_fake(1), A=_fake(2), B=_fake(3), C=_fake(4), D=None, z=None, bias=None,
                 sp=0, h0=None, v0=None, ckpt=_fake(10), dy=_fake(11), dhT=None, dvT=None, dx=_fake(12),
                 dd=_fake(13), dA=_fake(14), dB=_fake(15), dC=_fake(16), dD=None, dz=None, db=None,
                 dh0=None, dv0=None)
        a.update(over)
        return lib.mm_scan_bwd_gated(a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"],
                                     a["sp"], a["h0"], a["v0"], 0.9, 1.0, a["ckpt"], a["dy"], a["dhT"], a["dvT"],
                                     a["dx"], a["dd"], a["dA"], a["dB"], a["dC"], a["dD"], a["dz"], a["db"],
                                     a["dh0"], a["dv0"], ctypes.byref(dims), None)
    assert call(z=ctypes.c_void_p(A16 * 17 + 4)) == 5            # misaligned gate
    assert call(z=_fake(17), dz=_fake(17)) == 9                   # dz over z
    assert call(D=_fake(18), dD=_fake(18)) == 9                   # dD over D
    assert call(dD=_fake(12)) == 9                                # dD over dx
    assert call(db=_fake(1)) == 9                                 # d bias over delta
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    assert call(D=_fake(18), z=_fake(17), bias=_fake(19), sp=1, dD=_fake(20), dz=_fake(21),
                db=_fake(22)) == 7                                # passes every check


def test_step_checks_its_arguments(lib, monkeypatch):
    def call(L=1, **over):
        a = dict(x=_fake(0), delta=_fake(1), A=_fake(2), B=_fake(3), C=_fake(4), D=None, z=None,
                 bias=None, sp=0, h=_fake(5), v=_fake(6), y=_fake(7), beta=0.9)
        a.update(over)
        return lib.mm_scan_step(a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"],
                                a["sp"], a["h"], a["v"], a["beta"], 1.0, a["y"],
                                ctypes.byref(D(batch=4, L=L, dim=64)), None)
    assert call(h=None) == 1
    assert call(L=2) == 2                                         # a step is one time step
    assert call(beta=-0.1) == 3
    assert call(z=ctypes.c_void_p(A16 * 9 + 8)) == 5
    assert call(y=_fake(0)) == 9                                  # output over an input
    assert call(v=_fake(5)) == 9                                  # h and v on one buffer
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    assert call(D=_fake(8), z=_fake(9), bias=_fake(10), sp=1) == 7


def test_ssd_momentum_checks_its_arguments(lib, monkeypatch):
    def call(P=64, N=128, H=4, G=2, beta=0.9, **over):
        a = dict(x=_fake(0), delta=_fake(1), A=_fake(2), B=_fake(3), C=_fake(4), h0=None, v0=None,
                 y=_fake(5), hT=None, vT=None)
        a.update(over)
        dims = mm.SSDDims(1, 128, H, P, N, G, 64)
        return lib.mm_ssd_fwd_momentum(a["x"], a["delta"], a["A"], a["B"], a["C"], a["h0"], a["v0"], beta, 1.0,
                                       a["y"], a["hT"], a["vT"], ctypes.byref(dims), None)
    assert call(y=None) == 1
    assert call(G=3) == 2                                         # groups must divide heads
    assert call(P=128) == 6 and call(N=256) == 6                  # past the kernel's tile
    assert call(beta=1.0) == 3
    assert call(y=_fake(0)) == 9                                  # output over an input
    assert call(vT=_fake(6), hT=_fake(6)) == 9                    # two outputs on one buffer
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    assert call(h0=_fake(6), hT=_fake(6), v0=_fake(7), vT=_fake(7)) == 7   # in place: allowed


def test_set_tile(lib):
    assert lib.mm_scan_set_tile(3, 2, 1) == 6
    assert lib.mm_scan_set_tile(4, 2, 3) == 6
    assert lib.mm_scan_set_tile(4, 1, 2) == 6                    # time split needs >= 8 channels per CTA
    assert lib.mm_scan_set_tile(4, 2, 1) == 0
    assert lib.mm_scan_set_tile(4, 2, 2) == 0
    assert lib.mm_scan_set_tile(0, 0, 0) == 0


def test_deterministic_switch(lib):
    assert lib.mm_scan_set_deterministic(2) == 6
    assert lib.mm_scan_set_deterministic(-1) == 6
    assert lib.mm_scan_set_deterministic(1) == 0
    assert lib.mm_scan_set_deterministic(0) == 0


def test_set_path_and_segment_length_query(lib):
    assert lib.mm_scan_set_path(4, 0) == 6
    assert lib.mm_scan_set_path(3, 0) == 0                        # the sequence split as one fused launch
    seg3 = ctypes.c_int64(-1)
    assert lib.mm_scan_segment_len(ctypes.byref(mm.ScanDims(4, 2048, 1536, 16, 0)), ctypes.byref(seg3)) == 0
    assert seg3.value == 16384                                    # forced onto the sequence-split path
    assert lib.mm_scan_set_path(0, 0) == 0
    assert lib.mm_scan_set_path(2, 48) == 6                       # not a multiple of 32
    assert lib.mm_scan_set_path(2, 16) == 6                       # below 32
    assert lib.mm_scan_set_path(2, (1 << 30) + 32) == 6           # above 2^30
    seg = ctypes.c_int64(-1)
    dims = mm.ScanDims(1, 131072, 2048, 16, 0)
    assert lib.mm_scan_segment_len(ctypes.byref(dims), ctypes.byref(seg)) == 0 and seg.value == 16384
    one_segment = mm.ScanDims(1, 16384, 2048, 16, 0)               # L <= S: the register-resident path
    assert lib.mm_scan_segment_len(ctypes.byref(one_segment), ctypes.byref(seg)) == 0 and seg.value == 0
    just_over = mm.ScanDims(1, 16388, 2048, 16, 0)
    assert lib.mm_scan_segment_len(ctypes.byref(just_over), ctypes.byref(seg)) == 0 and seg.value == 16384
    assert lib.mm_scan_set_path(2, 256) == 0
    assert lib.mm_scan_segment_len(ctypes.byref(mm.ScanDims(4, 2048, 1536, 16, 0)), ctypes.byref(seg)) == 0
    assert seg.value == 256                                       # forced onto the sequence-split path
    assert lib.mm_scan_set_path(2, 14592) == 0                    # any whole number of 32-step chunks
    assert lib.mm_scan_segment_len(ctypes.byref(dims), ctypes.byref(seg)) == 0 and seg.value == 14592
    assert lib.mm_scan_set_path(2, 96) == 0
    assert lib.mm_scan_segment_len(ctypes.byref(mm.ScanDims(1, 2048, 64, 16, 1)), ctypes.byref(seg)) == 0
    assert seg.value == 128                                       # bf16: rounded up to whole 64-step chunks
    assert lib.mm_scan_set_path(2, 32) == 0
    assert lib.mm_scan_segment_len(ctypes.byref(mm.ScanDims(1, 2048, 64, 16, 1)), ctypes.byref(seg)) == 0
    assert seg.value == 64                                        # bf16: at least one 64-step chunk
    assert lib.mm_scan_segment_len(ctypes.byref(mm.ScanDims(1, 2048, 64, 16, 0)), ctypes.byref(seg)) == 0
    assert seg.value == 32
    assert lib.mm_scan_set_path(1, 0) == 0
    assert lib.mm_scan_segment_len(ctypes.byref(dims), ctypes.byref(seg)) == 0 and seg.value == 0
    assert lib.mm_scan_set_path(0, 0) == 0
    unaligned = mm.ScanDims(1, 131071, 2048, 16, 0)               # rows not whole 16-byte pieces
    assert lib.mm_scan_segment_len(ctypes.byref(unaligned), ctypes.byref(seg)) == 0 and seg.value == 0
    assert lib.mm_scan_segment_len(None, ctypes.byref(seg)) == 1
    assert lib.mm_scan_segment_len(ctypes.byref(mm.ScanDims(0, 1, 1, 1, 0)), ctypes.byref(seg)) == 2


def test_split_sizes_and_checks(lib, monkeypatch):
    """The sequence split's host checks: record sizes, the segment length, the
    piece's place in the whole sequence, and aliasing."""
    size = ctypes.c_size_t(0)
    # one record per (batch row, 16-channel tile) of a segment: 8 float4 maps of 32 lanes and a flag
    assert lib.mm_scan_split_maps_size(ctypes.byref(D(batch=2, dim=40)), 3, ctypes.byref(size)) == 0
    assert size.value == 3 * 2 * 3 * 257 * 16
    assert lib.mm_scan_split_maps_size(ctypes.byref(D()), -1, ctypes.byref(size)) == 2
    assert lib.mm_scan_split_maps_size(None, 1, ctypes.byref(size)) == 1

    def maps(S=64, d=None, **over):
        a = dict(x=_fake(0), delta=_fake(1), A=_fake(2), B=_fake(3), C=_fake(4), y=_fake(5), maps=_fake(6))
        a.update(over)
        dims = d if d is not None else D(L=128)
        return lib.mm_scan_fwd_split_maps(a["x"], a["delta"], a["A"], a["B"], a["C"], 0.9, 1.0, a["y"], a["maps"],
                                          S, ctypes.byref(dims), None)

    def correct(S=64, first=0, total=128, d=None, **over):
        a = dict(delta=_fake(1), A=_fake(2), C=_fake(4), h0=None, v0=None, y=_fake(5), hT=_fake(7), vT=None,
                 maps=_fake(6))
        a.update(over)
        dims = d if d is not None else D(L=128)
        return lib.mm_scan_fwd_split_correct(a["delta"], a["A"], a["C"], a["h0"], a["v0"], 0.9, 1.0, a["y"],
                                             a["hT"], a["vT"], a["maps"], S, first, total, ctypes.byref(dims), None)

    assert maps(S=48) == 6 and maps(S=16) == 6                    # not a power of two >= one chunk
    assert maps(S=32, d=D(L=128, io=1)) == 6                      # bf16: a chunk is 64 steps
    assert maps(d=D(L=129)) == 6                                  # rows not whole 16-byte pieces
    assert maps(maps=None) == 1
    assert maps(maps=ctypes.c_void_p(A16 * 7 + 8)) == 5
    assert maps(maps=_fake(1)) == 9                               # records on top of delta
    assert maps(y=_fake(6)) == 9                                  # y on top of the records
    assert correct(first=32) == 6                                 # piece not at a segment boundary
    assert correct(first=64, total=128) == 6                      # piece past the end
    assert correct(first=0, total=300, d=D(L=96)) == 6            # an inner piece of a partial segment
    assert correct(total=0) == 6
    assert correct(hT=_fake(6)) == 9                              # hT on top of the records
    assert correct(h0=_fake(7), hT=_fake(7)) == 9                 # no in-place state here
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    assert maps() == 7                                            # in range: reaches the launch step
    assert correct(first=128, total=300) == 7                     # the last piece may be partial


def test_peer_split_and_ipc_checks(lib, monkeypatch):
    dims = D(L=128)
    call = lambda nd, first=0, total=128, dests=_fake(9): lib.mm_scan_fwd_split_maps_peers(
        _fake(0), _fake(1), _fake(2), _fake(3), _fake(4), 0.9, 1.0, _fake(5), dests, nd, first, 64, total,
        ctypes.byref(dims), None)
    assert call(0) == 6 and call(65) == 6                         # 1 .. MM_SPLIT_MAX_RANKS destinations
    assert call(2, dests=None) == 1
    assert call(2, dests=ctypes.c_void_p(A16 * 10 + 4)) == 5      # the pointer array is 8-byte aligned
    assert call(2, first=32, total=256) == 6                      # piece off a segment boundary
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    assert call(2, first=128, total=256) == 7                     # in range: reaches the launch step
    monkeypatch.delenv("MMSCAN_FAULT_INJECT")
    off = ctypes.c_int64(0)
    ptr = ctypes.c_void_p(0)
    handle = ctypes.create_string_buffer(64)
    assert lib.mm_ipc_get_handle(None, handle, ctypes.byref(off)) == 1
    assert lib.mm_ipc_open_handle(None, 0, ctypes.byref(ptr)) == 1
    assert lib.mm_ipc_open_handle(handle, -16, ctypes.byref(ptr)) == 2
    assert lib.mm_ipc_close_handle(None, 0) == 1


def test_ssd_rejects_bad_arguments(lib, monkeypatch):
    dims = mm.SSDDims(1, 512, 4, 64, 128, 1, 256)

    def call(beta=0.0, alpha=1.0, d=None, **over):
        a = dict(x=_fake(0), delta=_fake(1), A=_fake(2), B=_fake(3), C=_fake(4), h0=None,
                 y=_fake(5), hT=None)
        a.update(over)
        return lib.mm_ssd_fwd(a["x"], a["delta"], a["A"], a["B"], a["C"], a["h0"], beta, alpha,
                              a["y"], a["hT"], ctypes.byref(d or dims), None)
    assert call(x=None) == 1
    assert call(beta=1.5) == 3
    assert call(alpha=-2.0) == 3
    assert call(y=_fake(0)) == 9
    assert call(hT=_fake(3)) == 9
    assert call(B=ctypes.c_void_p(A16 * 4 + 8)) == 5
    assert call(d=mm.SSDDims(1, 512, 4, 64, 128, 3, 256)) == 2                # H % G != 0
    for odd in (mm.SSDDims(1, 512, 4, 48, 128, 1, 256), mm.SSDDims(1, 512, 4, 64, 64, 1, 256),
                mm.SSDDims(1, 512, 4, 64, 128, 1, 64)):
        assert call(d=odd) == 6
    monkeypatch.setenv("MMSCAN_FAULT_INJECT", "launch")
    assert call() == 7
    assert call(h0=_fake(6), hT=_fake(6)) == 7                   # in-place final state
    assert call(beta=0.5) == 7                                    # momentum: the chunked momentum path


@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++11")])
def test_header_compiles_standalone(tmp_path, lang, std):
    """include/mm_scan.h is a plain C header: it compiles on its own as C99
    (pedantic) and as C++, with no CUDA or torch headers."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / ("t.c" if lang == "c" else "t.cpp")
    src.write_text('#include "mm_scan.h"\n'
                   "int main(void) { mm_scan_dims d = {1, 1, 1, 1, MM_F32}; (void)d; return (int)MM_OK; }\n")
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    r = subprocess.run([cc, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, "-fsyntax-only",
                        str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_plain_c_program_uses_the_abi(tmp_path):
    """A C program (tests/c/abi_check.c) links libmmscan.so through the header
    and gets the documented statuses back: the boundary needs no Python."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no host compiler")
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    lib = mm.library_path()
    exe = tmp_path / "abi_check"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        os.path.join(here, "c", "abi_check.c"), lib, "-o", str(exe),
                        "-Wl,-rpath," + os.path.dirname(lib)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and "abi ok" in run.stdout, run.stdout + run.stderr


def test_sizes_past_the_32_bit_index_range_are_refused(lib):
    """The kernels index time coordinates, grids and channels in 32 bits:
    seqlen past 2^30, and batch, dim or batch * heads from 2^31, are refused
    on the host with MM_ERR_UNSUPPORTED (and 64-bit byte-count overflow
    with MM_ERR_DIMS) before anything is launched."""
    assert _scan(lib, D(L=(1 << 30) + 1)) == 6
    assert _scan(lib, D(batch=1 << 31)) == 6
    assert _scan(lib, D(dim=1 << 31)) == 6
    assert _scan(lib, D(batch=(1 << 31) - 1, dim=(1 << 31) - 1, L=1 << 30)) == 2   # bytes overflow
    for dims in (mm.SSDDims(1, (1 << 30) + 1, 4, 64, 128, 1, 256), mm.SSDDims(1 << 29, 64, 4, 64, 128, 1, 256),
                 mm.SSDDims(1 << 40, 64, 1 << 40, 64, 128, 1, 256)):
        assert lib.mm_ssd_fwd(_fake(0), _fake(1), _fake(2), _fake(3), _fake(4), None, 0.0, 1.0, _fake(5), None,
                              ctypes.byref(dims), None) == 6
        st = lib.mm_ssd_fwd_momentum(_fake(0), _fake(1), _fake(2), _fake(3), _fake(4), None, None, 0.9, 1.0,
                                     _fake(5), None, None, ctypes.byref(dims), None)
        assert st == 6


def test_host_checks_under_sanitizers(tmp_path):
    """mm_api.cpp built with AddressSanitizer and UndefinedBehaviorSanitizer
    against a stand-in runtime and stub launchers (tests/c/api_checks_sanitized.cpp):
    every entry point, with sizes at and past every limit and non-finite
    scalars, returns a documented status without undefined behaviour, and
    the in-range calls reach their launchers."""
    import shutil
    import subprocess
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    csrc = os.path.join(root, "selective_state_space_momentum_b200", "csrc")
    exe = tmp_path / "api_checks"
    r = subprocess.run([cxx, "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined", "-fno-omit-frame-pointer",
                        "-fno-sanitize-recover=undefined", "-Wall", "-Werror",
                        "-I", os.path.join(here, "c", "stub_cuda"), "-I", os.path.join(root, "include"), "-I", csrc,
                        os.path.join(here, "c", "api_checks_sanitized.cpp"), os.path.join(csrc, "mm_api.cpp"),
                        "-o", str(exe)], capture_output=True, text=True)
    if r.returncode != 0 and "sanitize" in r.stderr and "cannot find" in r.stderr:
        pytest.skip("sanitizer runtimes not available")
    assert r.returncode == 0, r.stderr[-3000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300,
                         env=dict(os.environ, ASAN_OPTIONS="detect_leaks=0"))
    assert run.returncode == 0 and "api checks ok" in run.stdout, (run.stdout + run.stderr)[-3000:]


def test_host_pipeline_under_sanitizers(tmp_path):
    """mm_host.cpp (the host-buffer entry points) and mm_api.cpp built with
    AddressSanitizer and UndefinedBehaviorSanitizer against a stand-in
    runtime whose streams are queues run in adversarial orders, with CPU
    stand-ins for the kernels (tests/c/host_pipeline_sanitized.cpp): every
    chunked call reproduces one device call byte for byte under 24
    schedules, every copy and kernel operand stays inside its buffer, the
    argument checks answer before anything is queued, and dropping any one
    of the pipeline's waits makes some schedule fail."""
    import shutil
    import subprocess
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    csrc = os.path.join(root, "selective_state_space_momentum_b200", "csrc")
    exe = tmp_path / "host_pipeline"
    r = subprocess.run([cxx, "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined", "-fno-omit-frame-pointer",
                        "-fno-sanitize-recover=undefined", "-Wall", "-Werror",
                        "-I", os.path.join(here, "c", "stub_cuda"), "-I", os.path.join(root, "include"), "-I", csrc,
                        os.path.join(here, "c", "host_pipeline_sanitized.cpp"), os.path.join(csrc, "mm_api.cpp"),
                        os.path.join(csrc, "mm_host.cpp"), "-o", str(exe)], capture_output=True, text=True)
    if r.returncode != 0 and "sanitize" in r.stderr and "cannot find" in r.stderr:
        pytest.skip("sanitizer runtimes not available")
    assert r.returncode == 0, r.stderr[-3000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300,
                         env=dict(os.environ, ASAN_OPTIONS="detect_leaks=0"))
    assert run.returncode == 0 and "host pipeline ok" in run.stdout, (run.stdout + run.stderr)[-3000:]
