"""Seeded synthetic workloads for the momentum selective scan and its SSD form.

This module only draws random numbers and rounds them to the storage type.
It holds none of the scan's arithmetic: both the CUDA path and the fp64
oracle consume the arrays it returns, unchanged.

Shapes and value laws follow the pages' workloads:

* Momentum Mamba README, "Mamba Module": d_state = 16, dt_min = 1e-3,
  dt_max = 1e-1, so the step delta is drawn log-uniform on [1e-3, 1e-1]; the
  state matrix starts from the S4D-Real law A[d, n] = -(n + 1).
* Mamba-2 page, "Multi-Head Expansion": head dimension P = 64.

Every tensor has its own sub-stream of ``numpy.random.SeedSequence(seed)``
spawned in the fixed order x, delta, A-scale, B, C, so a tensor's values do
not depend on which other tensors are drawn.  "N(0, s)" means standard
deviation s.  bf16 tensors are rounded from fp32 with round-to-nearest-even
and returned as the fp32 numbers they represent (``bf16_bits`` gives the
16-bit patterns for the device copy).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

SEED_BASE = 20261202
_BLOCK = 1 << 24  # elements drawn per block, bounds temporary memory


# ---------------------------------------------------------------- bf16 -----
def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits.

    NaN stays a quiet NaN; infinities and overflow to infinity behave as IEEE
    rounding prescribes.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to the fp32 values they encode."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 value, returned as fp32."""
    return bf16_to_f32(bf16_bits(a))


# ------------------------------------------------------------ samplers -----
def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), np.float32)
    for s in range(0, out.size, _BLOCK):
        e = min(out.size, s + _BLOCK)
        out[s:e] = rng.standard_normal(e - s, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out.reshape(shape)


def _log_uniform(rng: np.random.Generator, shape, lo: float, hi: float) -> np.ndarray:
    """exp(U(ln lo, ln hi)), computed in fp64 and stored as fp32."""
    out = np.empty(int(np.prod(shape)), np.float32)
    a, b = math.log(lo), math.log(hi)
    for s in range(0, out.size, _BLOCK):
        e = min(out.size, s + _BLOCK)
        u = rng.random(e - s)
        out[s:e] = np.exp(a + (b - a) * u)
    return out.reshape(shape)


def _softplus_normal(rng: np.random.Generator, shape, std: float, shift: float) -> np.ndarray:
    """softplus(N(0, std) + shift) in fp64, stored as fp32."""
    out = np.empty(int(np.prod(shape)), np.float32)
    for s in range(0, out.size, _BLOCK):
        e = min(out.size, s + _BLOCK)
        z = rng.standard_normal(e - s) * std + shift
        out[s:e] = np.logaddexp(0.0, z)
    return out.reshape(shape)


# ------------------------------------------------------------- configs -----
@dataclass(frozen=True)
class ScanWorkload:
    """One Mamba-1 momentum-scan workload: shapes, value laws, (beta, alpha) runs."""
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    io: str = "f32"                     # "f32" or "bf16" for x/delta/B/C/y
    a_law: str = "s4d"                  # "s4d": -(n+1); "s4d_scaled": -(n+1)*U(0.5,2) per d
    bc_std: float = 1.0
    delta_law: str = "log_uniform"      # or "softplus_normal"
    runs: tuple = ((0.9, 1.0),)         # (beta, alpha) pairs
    split: int = 0                      # >0: also run as calls of this length, carrying state
    seed_index: int = 0

    @property
    def updates(self) -> int:
        return self.batch * self.seqlen * self.dim * self.dstate


@dataclass(frozen=True)
class SSDWorkload:
    """One Mamba-2 scalar-A multi-head workload (chunked SSD form)."""
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    beta: float = 0.0
    alpha: float = 1.0
    seed_index: int = 4

    @property
    def updates(self) -> int:
        return self.batch * self.seqlen * self.nheads * self.headdim * self.dstate


@dataclass(frozen=True)
class DecodeWorkload:
    """Single-token decode: one recurrence step for `batch` requests on their
    cached states (the Mamba module's step()), with the selective_scan_fn
    extras (delta bias and softplus, D skip, z gate) a Mamba layer applies."""
    name: str
    batch: int
    dim: int
    dstate: int
    io: str = "bf16"                    # x, delta, z, B, C, y; the states are fp32
    beta: float = 0.9
    alpha: float = 1.0
    seed_index: int = 5

    @property
    def updates(self) -> int:
        return self.batch * self.dim * self.dstate


SCAN_SMALL = ScanWorkload("scan_f32_b1_l256_d64_n16", 1, 256, 64, 16,
                          runs=((0.9, 1.0), (0.0, 1.0)), seed_index=0)
SCAN_MEDIUM = ScanWorkload("scan_f32_b4_l2048_d1536_n16", 4, 2048, 1536, 16,
                           a_law="s4d_scaled",
                           runs=tuple((b, a) for b in (0.0, 0.5, 0.9) for a in (0.5, 1.0, 2.0)),
                           seed_index=1)
SCAN_BF16 = ScanWorkload("scan_bf16_b8_l4096_d2048_n16", 8, 4096, 2048, 16, io="bf16",
                         bc_std=1.0 / math.sqrt(16), delta_law="softplus_normal",
                         runs=((0.9, 1.0),), seed_index=2)
SCAN_LONG = ScanWorkload("scan_f32_b1_l131072_d2048_n16_stream", 1, 131072, 2048, 16,
                         runs=((0.99, 1.0),), split=65536, seed_index=3)
SSD_MH = SSDWorkload("ssd_bf16_b4_l4096_h32_p64_n128_g1_q256", 4, 4096, 32, 64, 128, 1, 256,
                     seed_index=4)
# the same shapes and inputs with the momentum velocity (beta = 0.9)
# chunk: the 128-step block of the tensor-core momentum kernel (the momentum
# call takes no chunk argument; this is the Q of the FLOP count)
SSD_MH_MOMENTUM = SSDWorkload("ssd_momentum_bf16_b4_l4096_h32_p64_n128_g1", 4, 4096, 32, 64, 128, 1, 128,
                              beta=0.9, seed_index=4)

DECODE = DecodeWorkload("decode_bf16_b512_d2048_n16", 512, 2048, 16)

SCAN_WORKLOADS = (SCAN_SMALL, SCAN_MEDIUM, SCAN_BF16, SCAN_LONG)


def seed_of(index: int) -> int:
    return SEED_BASE + index


def _streams(seed: int, k: int):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(k)]


def scan_inputs(w: ScanWorkload, *, batch: int | None = None, seqlen: int | None = None,
                dim: int | None = None, dstate: int | None = None, seed: int | None = None):
    """Draw x, delta, A, B, C for a scan workload (optionally resized).

    Returns a dict of fp32 numpy arrays with layouts x, delta: (batch, dim, L);
    A: (dim, N); B, C: (batch, N, L).  For bf16 workloads x, delta, B, C hold
    bf16-rounded values (A stays fp32).
    """
    bsz = batch or w.batch
    L = seqlen or w.seqlen
    D = dim or w.dim
    N = dstate or w.dstate
    rx, rd, ra, rb, rc = _streams(seed if seed is not None else seed_of(w.seed_index), 5)
    x = _normal(rx, (bsz, D, L))
    if w.delta_law == "log_uniform":
        delta = _log_uniform(rd, (bsz, D, L), 1e-3, 1e-1)
    elif w.delta_law == "softplus_normal":
        delta = _softplus_normal(rd, (bsz, D, L), 0.5, math.log(math.expm1(0.01)))
    else:
        raise ValueError(w.delta_law)
    base = -(np.arange(N, dtype=np.float64) + 1.0)
    if w.a_law == "s4d":
        A = np.broadcast_to(base, (D, N)).astype(np.float32)
    elif w.a_law == "s4d_scaled":
        s = ra.uniform(0.5, 2.0, size=D)
        A = (s[:, None] * base[None, :]).astype(np.float32)
    else:
        raise ValueError(w.a_law)
    B = _normal(rb, (bsz, N, L), w.bc_std)
    C = _normal(rc, (bsz, N, L), w.bc_std)
    if w.io == "bf16":
        x, delta, B, C = (bf16_round(t) for t in (x, delta, B, C))
    return {"x": x, "delta": delta, "A": np.ascontiguousarray(A), "B": B, "C": C}


def scan_extras(w: ScanWorkload, *, batch: int | None = None, seqlen: int | None = None,
                dim: int | None = None, seed: int | None = None):
    """Draw the selective_scan_fn extras for a scan workload: a raw delta
    ~ N(0, 0.5) (batch, dim, L) meant to go through softplus(delta + bias),
    delta_bias = ln(expm1(dt)) with dt log-uniform on [1e-3, 1e-1] per channel
    (so that softplus(delta + bias) has the workloads' usual size), a skip
    weight D ~ U(0.5, 1.5) per channel and a gate z ~ N(0, 1) (batch, dim,
    L).  Their own seed stream (the workload's seed + 1000); for bf16
    workloads delta and z hold bf16-rounded values."""
    bsz = batch or w.batch
    L = seqlen or w.seqlen
    D = dim or w.dim
    rd, rb, rs, rz = _streams((seed if seed is not None else seed_of(w.seed_index)) + 1000, 4)
    delta_raw = _normal(rd, (bsz, D, L), 0.5)
    dt = _log_uniform(rb, (D,), 1e-3, 1e-1).astype(np.float64)
    bias = np.log(np.expm1(dt)).astype(np.float32)
    Dskip = rs.uniform(0.5, 1.5, D).astype(np.float32)
    z = _normal(rz, (bsz, D, L))
    if w.io == "bf16":
        delta_raw = bf16_round(delta_raw)
        z = bf16_round(z)
    return {"delta_raw": delta_raw, "delta_bias": bias, "D": Dskip, "z": z}


def ssd_inputs(w: SSDWorkload, *, batch: int | None = None, seqlen: int | None = None,
               nheads: int | None = None, headdim: int | None = None,
               dstate: int | None = None, ngroups: int | None = None,
               seed: int | None = None):
    """Draw x, delta, A, B, C for an SSD workload (optionally resized).

    Layouts: x (batch, L, H, P) bf16 values; delta (batch, L, H) fp32 drawn
    log-uniform on [1e-3, 1e-1]; A (H) fp32 = -U(1, 16); B, C (batch, L, G, N)
    bf16 values with standard deviation 1/sqrt(N).
    """
    bsz = batch or w.batch
    L = seqlen or w.seqlen
    H = nheads or w.nheads
    P = headdim or w.headdim
    N = dstate or w.dstate
    G = ngroups or w.ngroups
    rx, rd, ra, rb, rc = _streams(seed if seed is not None else seed_of(w.seed_index), 5)
    x = bf16_round(_normal(rx, (bsz, L, H, P)))
    delta = _log_uniform(rd, (bsz, L, H), 1e-3, 1e-1)
    A = (-ra.uniform(1.0, 16.0, size=H)).astype(np.float32)
    B = bf16_round(_normal(rb, (bsz, L, G, N), 1.0 / math.sqrt(N)))
    C = bf16_round(_normal(rc, (bsz, L, G, N), 1.0 / math.sqrt(N)))
    return {"x": x, "delta": delta, "A": A, "B": B, "C": C}


def decode_inputs(w: DecodeWorkload, *, batch: int | None = None, dim: int | None = None,
                  dstate: int | None = None, seed: int | None = None):
    """Draw one decode step's inputs and cached states.

    Layouts: x, delta, z (batch, dim); B, C (batch, N); A (dim, N); D,
    delta_bias (dim); h, v (batch, dim, N) fp32.  Laws as the scan workloads
    and their extras: x, z ~ N(0, 1); a raw delta ~ N(0, 0.5) fed with
    delta_bias = ln(expm1(dt)), dt log-uniform on [1e-3, 1e-1]; A = -(n + 1)
    U(0.5, 2) per channel; B, C ~ N(0, 1/4); D ~ U(0.5, 1.5); the cached
    states h ~ N(0, 1), v ~ N(0, 0.1).  bf16 tensors hold bf16-rounded values.
    """
    bsz = batch or w.batch
    D = dim or w.dim
    N = dstate or w.dstate
    rx, rd, ra, rb, rc, rbias, rs, rz, rh, rv = _streams(
        seed if seed is not None else seed_of(w.seed_index), 10)
    x = _normal(rx, (bsz, D))
    delta = _normal(rd, (bsz, D), 0.5)
    A = ((ra.uniform(0.5, 2.0, size=D)[:, None]) * -(np.arange(N, dtype=np.float64) + 1.0)[None, :])
    B = _normal(rb, (bsz, N), 0.25)
    C = _normal(rc, (bsz, N), 0.25)
    dt = _log_uniform(rbias, (D,), 1e-3, 1e-1).astype(np.float64)
    bias = np.log(np.expm1(dt)).astype(np.float32)
    Dskip = rs.uniform(0.5, 1.5, D).astype(np.float32)
    z = _normal(rz, (bsz, D))
    h = _normal(rh, (bsz, D, N))
    v = _normal(rv, (bsz, D, N), 0.1)
    if w.io == "bf16":
        x, delta, B, C, z = (bf16_round(t) for t in (x, delta, B, C, z))
    return {"x": x, "delta": delta, "A": np.ascontiguousarray(A.astype(np.float32)), "B": B, "C": C,
            "D": Dskip, "z": z, "delta_bias": bias, "h": h, "v": v}
