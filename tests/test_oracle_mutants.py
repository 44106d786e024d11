"""Planted mistakes: every plausible slip in the oracle must fail a pin.

Each case copies mm_oracle.c to a temporary directory, applies one textual
mutation (a dropped term, a wrong sign, an operand swap, an off-by-one, an
ignored initial state), builds it with the same flags, and runs a handful of
the pins from test_oracle_pins against it.  The test passes when at least one
pin rejects the mutant.  The real oracle is never modified.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _brute_force_scan, GOLDEN

SRC = os.path.join(os.path.dirname(oracle.__file__), "mm_oracle.c")

MUTANTS = {
    "drop_momentum": ("v = beta * v + alpha * (dt * (double)Bn[t] * (double)xr[t]);",
                      "v = alpha * (dt * (double)Bn[t] * (double)xr[t]);"),
    "read_before_update": ("                h = abar * h + v;\n                yr[t] += (double)Cn[t] * h;",
                           "                yr[t] += (double)Cn[t] * h;\n                h = abar * h + v;"),
    "exp_sign": ("const double abar = exp(dt * a_dn);\n                v = beta * v",
                 "const double abar = exp(-dt * a_dn);\n                v = beta * v"),
    "swap_B_C": ("yr[t] += (double)Cn[t] * h;\n            }\n            if (hT) hT[r * dstate + n] = h;\n            if (vT) vT[r * dstate + n] = v;\n        }\n    }\n    return ORACLE_OK;\n}\n\n/* ----",
                 "yr[t] += (double)Bn[t] * h;\n            }\n            if (hT) hT[r * dstate + n] = h;\n            if (vT) vT[r * dstate + n] = v;\n        }\n    }\n    return ORACLE_OK;\n}\n\n/* ----"),
    "drop_alpha": ("v = beta * v + alpha * (dt * (double)Bn[t] * (double)xr[t]);",
                   "v = beta * v + (dt * (double)Bn[t] * (double)xr[t]);"),
    "x_off_by_one": ("v = beta * v + alpha * (dt * (double)Bn[t] * (double)xr[t]);",
                     "v = beta * v + alpha * (dt * (double)Bn[t] * (double)xr[t > 0 ? t - 1 : 0]);"),
    "B_time_shift": ("v = beta * v + alpha * (dt * (double)Bn[t] * (double)xr[t]);",
                     "v = beta * v + alpha * (dt * (double)Bn[t + 1 < seqlen ? t + 1 : t] * (double)xr[t]);"),
    "ignore_h0": ("double h = h0 ? h0[c * dstate + n] : 0.0;\n            double v = v0 ? v0[c * dstate + n] : 0.0;\n            const double a_dn",
                  "double h = 0.0;\n            double v = v0 ? v0[c * dstate + n] : 0.0;\n            const double a_dn"),
    "ignore_v0": ("double h = h0 ? h0[c * dstate + n] : 0.0;\n            double v = v0 ? v0[c * dstate + n] : 0.0;\n            const double a_dn",
                  "double h = h0 ? h0[c * dstate + n] : 0.0;\n            double v = 0.0;\n            const double a_dn"),
    "A_transposed": ("const double a_dn = (double)A[d * dstate + n];",
                     "const double a_dn = (double)A[(n % dim) * dstate + (d % dstate)];"),
}

SSD_MUTANTS = {
    "ssd_offdiag_no_decay": ("Y_AT(t0 + i, p) += ei * yo;", "Y_AT(t0 + i, p) += yo;"),
    "ssd_state_decay_index": ("acc2 += exp(cs_last - cs[j])", "acc2 += exp(cs_last - cs[0])"),
    "ssd_noncausal_mask": ("for (int64_t j = 0; j <= i; ++j) {\n                    double cb",
                           "for (int64_t j = 0; j < q; ++j) {\n                    double cb"),
    "ssd_carry_no_decay": ("for (int64_t k = 0; k < PN; ++k) S[k] = decay * S[k] + s[k];",
                           "for (int64_t k = 0; k < PN; ++k) S[k] = S[k] + s[k];"),
    "ssd_drop_delta": ("const double lij = cb * exp(cs[i] - cs[j]) * alpha * D_AT(t0 + j);",
                       "const double lij = cb * exp(cs[i] - cs[j]) * alpha;"),
}


GATED_MUTANTS = {
    "softplus_dropped": ("                if (softplus) dt = softplus_f64(dt);\n", ""),
    "softplus_log_not_log1p": ("return (u > 0.0 ? u : 0.0) + log1p(exp(-fabs(u)));",
                               "return (u > 0.0 ? u : 0.0) + log(exp(-fabs(u)));"),
    "bias_sign": ("double dt = (double)dr[t] + (dbias ? (double)dbias[d] : 0.0);",
                  "double dt = (double)dr[t] - (dbias ? (double)dbias[d] : 0.0);"),
    "skip_without_x": ("double o = yr[t] + (Dv ? (double)Dv[d] * (double)xr[t] : 0.0);",
                       "double o = yr[t] + (Dv ? (double)Dv[d] : 0.0);"),
    "gate_sigmoid_not_silu": ("o *= zt / (1.0 + exp(-zt));", "o *= 1.0 / (1.0 + exp(-zt));"),
    "skip_after_gate": ("double o = yr[t] + (Dv ? (double)Dv[d] * (double)xr[t] : 0.0);\n            if (z) {\n"
                        "                const double zt = (double)z[c * seqlen + t];\n"
                        "                o *= zt / (1.0 + exp(-zt));\n            }",
                        "double o = yr[t];\n            if (z) {\n"
                        "                const double zt = (double)z[c * seqlen + t];\n"
                        "                o *= zt / (1.0 + exp(-zt));\n            }\n"
                        "            o += (Dv ? (double)Dv[d] * (double)xr[t] : 0.0);"),
}


# Backward: each is a plausible slip in the adjoint recursions or a local term,
# the first one the velocity recursion exactly as the pages print it (the
# read-out gradient only, without the hidden state's full gradient).
BWD_MUTANTS = {
    "bwd_velocity_adjoint_as_printed": ("const double p = g + cp;",
                                        "const double p = dy[t] * (double)Cn[t] + cp;"),
    "bwd_decay_a_t_not_a_t1": ("cg = as[t] * g;", "cg = (t > 0 ? as[t - 1] : as[0]) * g;"),
    "bwd_velocity_no_beta": ("cp = beta * p;", "cp = p;"),
    "bwd_ddelta_no_exp_path": (" + a_dn * decay_term;", ";"),
    "bwd_dA_without_delta": ("acc_a += dp[t] * decay_term;", "acc_a += decay_term;"),
    "bwd_dB_without_alpha": ("dB[k * seqlen + t] += alpha * dp[t]", "dB[k * seqlen + t] += dp[t]"),
    "bwd_dC_previous_state": ("dC[k * seqlen + t] += dy[t] * hs[t];",
                              "dC[k * seqlen + t] += dy[t] * (t > 0 ? hs[t - 1] : 0.0);"),
    "bwd_silu_grad_missing_term": ("dy[t] * ot * st * (1.0 + zt * (1.0 - st))",
                                   "dy[t] * ot * st * (1.0 - st)"),
    "bwd_softplus_grad_dropped": ("g_delta *= 1.0 / (1.0 + exp(-u));", ""),
    "bwd_skip_grad_ungated": ("(Dv ? (double)Dv[d] * dy[t] : 0.0)",
                              "(Dv ? (double)Dv[d] * (double)dout[c * seqlen + t] : 0.0)"),
    "bwd_dhT_ignored": ("dhT ? dhT[c * dstate + n] : 0.0, dvT ? dvT[c * dstate + n] : 0.0,",
                        "0.0, dvT ? dvT[c * dstate + n] : 0.0,"),
}


# Chunked momentum SSD: slips in the mask, the carry weights or the carried velocity.
SSDM_MUTANTS = {
    "ssdm_mask_without_beta": ("sum += exp(cs[i] - cs[k]) * pow(beta, (double)(k - j));",
                               "sum += exp(cs[i] - cs[k]);"),
    "ssdm_mask_beta_from_i": ("sum += exp(cs[i] - cs[k]) * pow(beta, (double)(k - j));",
                              "sum += exp(cs[i] - cs[k]) * pow(beta, (double)(i - k));"),
    "ssdm_carry_weight_power": ("sm += exp(cs[i] - cs[k]) * pow(beta, (double)(k + 1));",
                                "sm += exp(cs[i] - cs[k]) * pow(beta, (double)k);"),
    "ssdm_velocity_decay": ("const double bq = pow(beta, (double)q);", "const double bq = pow(beta, (double)(q - 1));"),
    "ssdm_no_velocity_readout": ("Y_AT(t0 + i, p) += ei * ch + mv[i] * cv;", "Y_AT(t0 + i, p) += ei * ch;"),
}


def _ssdm_pins(lib):
    from tests import test_oracle_ssd_momentum_pins as mp
    return mp.chunked_failures(lib=lib)


def _bwd_pins(lib):
    """Finite-difference pins of tests/test_oracle_bwd_pins.py run against `lib`."""
    from tests import test_oracle_bwd_pins as bp
    return bp.fd_failures("momentum_h0v0", lib=lib) + bp.fd_failures("gated_softplus", lib=lib)


def _gated_pins(lib):
    """Pins of tests/test_oracle_gated_pins.py run against `lib`."""
    from tests import test_oracle_gated_pins as gp
    failed = []
    g = json.load(open(GOLDEN))["selective_fig2"]
    A = math.log(0.5)
    for case in g["cases"]:
        bias = math.log(math.expm1(case["delta"]))
        y, h, _ = gp._one_step_gated([g["h_prev"]], [A], 0.0, [g["B"]], g["u"], [g["C"]],
                                     delta_bias=bias, softplus=True, lib=lib)
        if abs(h[0] - case["new_state_derived"]) > 1e-6 * case["new_state_derived"]:
            failed.append("fig2_softplus")
            break
    for case in g["cases"]:
        y, h, _ = gp._one_step_gated([g["h_prev"]], [A], 0.25 * case["delta"], [g["B"]], g["u"], [g["C"]],
                                     delta_bias=0.75 * case["delta"], softplus=False, lib=lib)
        if abs(h[0] - case["new_state_derived"]) > 1e-6 * case["new_state_derived"]:
            failed.append("fig2_bias")
            break
    y, _, _ = gp._one_step_gated([0.0], [-1.0], 0.1, [1.0], 3.0, [0.0], D=2.0, z=1.0, lib=lib)
    if abs(y - 6.0 * gp.SIGMA1) > 1e-12:
        failed.append("skip_then_gate")
    y, _, _ = gp._one_step_gated([0.0], [-1.0], 0.1, [1.0], 3.0, [0.0], D=2.0, z=2.0, lib=lib)
    if abs(y - 6.0 * gp.SILU2) > 1e-12:
        failed.append("silu2")
    y, _, _ = gp._one_step_gated([0.0], [-1.0], 0.1, [1.0], 3.0, [0.0], D=2.0, lib=lib)
    if y != 6.0:
        failed.append("skip_C0")
    return failed


def _ssd_pins(lib):
    """Chunked SSD against the sequential definition (tiny, several chunks)."""
    rng = np.random.default_rng(4)
    Bsz, L, H, P, N, G = 1, 20, 2, 2, 3, 1
    x = rng.standard_normal((Bsz, L, H, P)).astype(np.float32)
    delta = np.exp(rng.uniform(np.log(1e-2), np.log(0.3), (Bsz, L, H))).astype(np.float32)
    A = (-rng.uniform(1.0, 4.0, H)).astype(np.float32)
    Bm = rng.standard_normal((Bsz, L, G, N)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, G, N)).astype(np.float32)
    h0 = rng.standard_normal((Bsz, H, P, N))
    ys, hs, _ = oracle.ssd_seq(x, delta, A, Bm, Cm, h0=h0, beta=0.0, alpha=1.0)
    yc, hc = oracle.ssd_chunked(x, delta, A, Bm, Cm, h0=h0, alpha=1.0, chunk=6, lib=lib)
    ok = np.allclose(yc.transpose(0, 2, 3, 1).reshape(-1, L), ys, rtol=1e-10, atol=1e-11) and \
        np.allclose(hc.reshape(-1, N), hs, rtol=1e-10, atol=1e-12)
    return [] if ok else ["ssd_chunked_vs_seq"]


def _pins(lib):
    """Run a few pins against `lib`; return the names of those that fail."""
    failed = []
    g = json.load(open(GOLDEN))
    # Figure 5 of the selective-SSM tutorial
    f5 = g["selective_fig5"]
    A = [math.log(0.5), math.log(0.8)]
    for case in f5["cases"]:
        y, h, _ = oracle.scan_seq(
            np.array([[[f5["u"]]]], np.float32), np.array([[[case["delta"]]]], np.float32),
            np.array([A], np.float32), np.array(case["B"], np.float32).reshape(1, 2, 1),
            np.array(case["C"], np.float32).reshape(1, 2, 1),
            h0=np.array(f5["h_prev"], np.float64).reshape(1, 1, 2), beta=0.0, alpha=1.0, lib=lib)
        if not (np.allclose(h[0], case["new_state"], rtol=1e-6) and abs(y[0, 0] - case["y"]) < 1e-5):
            failed.append("fig5")
            break
    # brute-force matrix with momentum, alpha != 1 and an initial state
    rng = np.random.default_rng(11)
    Bsz, D, L, N = 2, 3, 9, 3
    x = rng.standard_normal((Bsz, D, L)).astype(np.float32)
    delta = np.exp(rng.uniform(np.log(1e-2), np.log(0.5), (Bsz, D, L))).astype(np.float32)
    Am = (-rng.uniform(0.5, 3.0, (D, N))).astype(np.float32)
    Bm = rng.standard_normal((Bsz, N, L)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, N, L)).astype(np.float32)
    h0 = rng.standard_normal((Bsz, D, N))
    v0 = rng.standard_normal((Bsz, D, N))
    y, _, _ = oracle.scan_seq(x, delta, Am, Bm, Cm, h0=h0, v0=v0, beta=0.6, alpha=1.7, lib=lib)
    ref = _brute_force_scan(x, delta, Am, Bm, Cm, h0, v0, 0.6, 1.7)
    if not np.allclose(y.reshape(Bsz, D, L), ref, rtol=1e-10, atol=1e-11):
        failed.append("brute_force")
    return failed


def test_real_oracle_passes_the_mutant_pins():
    assert _pins(oracle.load()) == []
    assert _ssd_pins(oracle.load()) == []
    assert _gated_pins(oracle.load()) == []


@pytest.mark.parametrize("name", sorted(MUTANTS) + sorted(SSD_MUTANTS) + sorted(GATED_MUTANTS)
                         + sorted(BWD_MUTANTS) + sorted(SSDM_MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = (MUTANTS.get(name) or SSD_MUTANTS.get(name) or GATED_MUTANTS.get(name)
                or BWD_MUTANTS.get(name) or SSDM_MUTANTS[name])
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mut_src = tmp_path / "mm_oracle.c"
    mut_src.write_text(src.replace(old, new, 1))
    import subprocess
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared",
                    "-fPIC", "-std=c11", "-o", str(so), str(mut_src), "-lm"], check=True)
    lib = oracle.load(str(so))
    pins = (_pins if name in MUTANTS else _ssd_pins if name in SSD_MUTANTS
            else _gated_pins if name in GATED_MUTANTS else _bwd_pins if name in BWD_MUTANTS
            else _ssdm_pins)
    assert pins(lib), f"no pin caught the planted mistake '{name}'"
