"""The Python binding checks every tensor before calling the library (no GPU).

The C ABI takes raw device pointers and sizes every operand from x's and A's
shapes, so the binding refuses, before any call, tensors that would be read
wrongly or past their end: host tensors, wrong storage types, wrong shapes
(a B shorter than x) and strided views.  These checks run on CPU tensors:
each failure is raised before the device check, and a call whose tensors are
all correct but on the host is refused for that.
"""
import pytest

import selective_state_space_momentum_b200 as mm

torch = pytest.importorskip("torch")


def _scan_args(batch=2, dim=8, L=32, N=16, dt=torch.float32):
    x = torch.zeros(batch, dim, L, dtype=dt)
    return dict(x=x, delta=torch.zeros_like(x), A=torch.zeros(dim, N), B=torch.zeros(batch, N, L, dtype=dt),
                C=torch.zeros(batch, N, L, dtype=dt), h0=None, v0=None, beta=0.9, alpha=1.0,
                y=torch.zeros_like(x), hT=torch.zeros(batch, dim, N), vT=torch.zeros(batch, dim, N))


def _call(**over):
    a = _scan_args()
    a.update(over)
    mm.mm_scan_fwd(**a)


def test_host_tensors_are_refused():
    with pytest.raises(ValueError, match="CUDA"):
        _call()


def test_wrong_storage_type_is_refused():
    with pytest.raises(TypeError, match="delta"):
        _call(delta=torch.zeros(2, 8, 32, dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="h0"):
        _call(h0=torch.zeros(2, 8, 16, dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="A"):
        _call(A=torch.zeros(8, 16, dtype=torch.float64))
    with pytest.raises(TypeError):
        _call(x=torch.zeros(2, 8, 32, dtype=torch.float16))


def test_short_or_misshapen_operands_are_refused():
    with pytest.raises(ValueError, match="B"):
        _call(B=torch.zeros(2, 16, 16))                  # shorter than x along L
    with pytest.raises(ValueError, match="C"):
        _call(C=torch.zeros(1, 16, 32))                  # one batch row
    with pytest.raises(ValueError, match="vT"):
        _call(vT=torch.zeros(2, 8, 8))
    with pytest.raises(ValueError, match="A"):
        _call(A=torch.zeros(4, 16))


def test_strided_views_are_refused():
    big = torch.zeros(2, 8, 64)
    with pytest.raises(ValueError, match="contiguous"):
        _call(x=big[..., 32:])
    with pytest.raises(ValueError, match="contiguous"):
        _call(delta=torch.zeros(2, 32, 8).transpose(1, 2))


def test_backward_and_step_check_their_operands():
    a = _scan_args()
    g = dict(dx=torch.zeros_like(a["x"]), ddelta=torch.zeros_like(a["x"]), dA=torch.zeros(8, 16),
             dB=torch.zeros(2, 16, 32), dC=torch.zeros(2, 16, 32), dh0=None, dv0=None)
    ck = torch.zeros(2, 8, 2, 2, 16)
    with pytest.raises(ValueError, match="dB"):
        mm.mm_scan_bwd(a["x"], a["delta"], a["A"], a["B"], a["C"], None, None, 0.9, 1.0, ck, a["x"], None,
                       None, g["dx"], g["ddelta"], g["dA"], torch.zeros(2, 16, 31), g["dC"], None, None)
    with pytest.raises(ValueError, match="ckpt"):
        mm.mm_scan_bwd(a["x"], a["delta"], a["A"], a["B"], a["C"], None, None, 0.9, 1.0,
                       torch.zeros(2, 8, 1, 2, 16), a["x"], None, None, g["dx"], g["ddelta"], g["dA"], g["dB"],
                       g["dC"], None, None)
    x = torch.zeros(4, 8)
    with pytest.raises(ValueError, match="h"):
        mm.mm_scan_step(x, x, torch.zeros(8, 16), torch.zeros(4, 16), torch.zeros(4, 16), None, None, None,
                        False, torch.zeros(4, 8, 15), torch.zeros(4, 8, 16), 0.9, 1.0, torch.zeros(4, 8))


def test_ssd_calls_check_their_operands():
    bf = torch.bfloat16
    x = torch.zeros(1, 64, 4, 64, dtype=bf)
    args = dict(x=x, delta=torch.zeros(1, 64, 4), A=torch.zeros(4), B=torch.zeros(1, 64, 1, 128, dtype=bf),
                C=torch.zeros(1, 64, 1, 128, dtype=bf), h0=None, beta=0.0, alpha=1.0, y=torch.zeros_like(x),
                hT=None, chunk=256)
    with pytest.raises(ValueError, match="CUDA"):
        mm.mm_ssd_fwd(**args)
    with pytest.raises(TypeError, match="bf16"):
        mm.mm_ssd_fwd(**{**args, "x": x.float()})
    with pytest.raises(ValueError, match="delta"):
        mm.mm_ssd_fwd(**{**args, "delta": torch.zeros(1, 64, 3)})
    with pytest.raises(ValueError, match="hT"):
        mm.mm_ssd_fwd(**{**args, "hT": torch.zeros(1, 4, 64, 64)})
