"""Calls every oracle entry point on random small and ragged inputs, for
tests/test_oracle_sanitizers.py, which runs it in a child process with the
oracle built under AddressSanitizer and UndefinedBehaviorSanitizer (the path
of that build is the first argument)."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import oracle  # noqa: E402

lib = oracle.load(sys.argv[1])
rng = np.random.default_rng(0)
f32 = np.float32
for it in range(40):
    b, d, L, N = int(rng.integers(1, 3)), int(rng.integers(1, 5)), int(rng.integers(1, 50)), int(rng.integers(1, 17))
    x = rng.standard_normal((b, d, L)).astype(f32); dl = rng.uniform(0.01, 0.3, (b, d, L)).astype(f32)
    A = -rng.uniform(0.1, 2, (d, N)).astype(f32); B = rng.standard_normal((b, N, L)).astype(f32); C = rng.standard_normal((b, N, L)).astype(f32)
    h0 = rng.standard_normal((b, d, N)); v0 = rng.standard_normal((b, d, N))
    chan = np.array(sorted(set(rng.integers(0, b * d, 2).tolist())), np.int64)
    oracle.scan_seq(x, dl, A, B, C, h0=h0, v0=v0, beta=0.9, alpha=1.0, lib=lib)
    oracle.scan_seq(x, dl, A, B, C, beta=0.5, alpha=2.0, chan=chan, lib=lib)
    oracle.scan_chunked(x, dl, A, B, C, h0=h0, v0=v0, beta=0.9, alpha=1.0, chunk=int(rng.integers(1, 70)), lib=lib)
    D = rng.uniform(0.5, 1.5, d).astype(f32); z = rng.standard_normal((b, d, L)).astype(f32); bias = rng.uniform(-3, -1, d).astype(f32)
    oracle.scan_gated(x, dl, A, B, C, D=D, z=z, delta_bias=bias, delta_softplus=True, h0=h0, v0=v0, beta=0.9, lib=lib)
    dout = rng.standard_normal((b, d, L)).astype(f32)
    bn = np.array(sorted(set(rng.integers(0, b * N, 2).tolist())), np.int64)
    oracle.scan_bwd(x, dl, A, B, C, dout, D=D, z=z, delta_bias=bias, delta_softplus=True, h0=h0, v0=v0,
                    dhT=rng.standard_normal((b, d, N)), dvT=rng.standard_normal((b, d, N)), beta=0.9, lib=lib)
    oracle.scan_bwd(x, dl, A, B, C, dout, beta=0.0, chan=chan, bn=bn, lib=lib)
    H, G = [(1, 1), (2, 1), (2, 2), (4, 2)][it % 4]; P = int(rng.integers(1, 5)); Ns = int(rng.integers(1, 9))
    xs = rng.standard_normal((b, L, H, P)).astype(f32); ds = rng.uniform(0.01, 0.3, (b, L, H)).astype(f32)
    As = -rng.uniform(0.1, 2, H).astype(f32); Bs = rng.standard_normal((b, L, G, Ns)).astype(f32); Cs = rng.standard_normal((b, L, G, Ns)).astype(f32)
    hs = rng.standard_normal((b, H, P, Ns)); vs = rng.standard_normal((b, H, P, Ns))
    oracle.ssd_seq(xs, ds, As, Bs, Cs, h0=hs, v0=vs, beta=0.9, lib=lib)
    oracle.ssd_seq(xs, ds, As, Bs, Cs, lane=np.array([0], np.int64), lib=lib)
    oracle.ssd_chunked(xs, ds, As, Bs, Cs, h0=hs, chunk=int(2 ** rng.integers(0, 7)), lib=lib)
    oracle.ssd_chunked_momentum(xs, ds, As, Bs, Cs, h0=hs, v0=vs, beta=0.9, chunk=int(rng.integers(1, 60)), lib=lib)
print("oracle under sanitizers: ok")
