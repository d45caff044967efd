"""The oracle's pins have teeth: each plausible slip, planted in a copy of the
oracle's C source (on the CPU), must make at least one pin in
test_oracle_pins.py fail.  The real oracle is not touched."""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ss_oracle.c")

# (name, original text, mutated text)
MUTANTS = [
    ("B_bar without Delta", ": dt * b_t;", ": b_t;"),
    ("sign of A", "exp(dt * (double)J->A[d * N + n])", "exp(-dt * (double)J->A[d * N + n])"),
    ("B and C swapped", "const double b_t = widen(J->B,", "const double b_t = widen(J->C,"),
    ("bias outside the softplus",
     "const double dt = J->softplus_flag ? softplus64(x) : x;",
     "const double dt = J->softplus_flag ? softplus64(x - bias) + bias : x;"),
    ("readout before the update",
     "h[n] = a_bar * h[n] + b_bar * ut;\n      s += c_t * h[n];",
     "s += c_t * h[n];\n      h[n] = a_bar * h[n] + b_bar * ut;"),
    ("gate misses the skip term",
     "    s += Dd * ut;\n    if (J->z) s *= silu64(widen(J->z, J->dtype, row + t));",
     "    if (J->z) s *= silu64(widen(J->z, J->dtype, row + t));\n    s += Dd * ut;"),
    ("A indexed [n][d]", "J->A[d * N + n]", "J->A[n * J->dim + d]"),
    ("state not carried", "h[n] = a_bar * h[n] + b_bar * ut;", "h[n] = a_bar * 0.0 + b_bar * ut;"),
    ("initial state ignored", "h[n] = J->h0 ? J->h0[flat * N + n] : 0.0;", "h[n] = 0.0;"),
    ("initial state indexed [b][n][d]", "J->h0[flat * N + n]", "J->h0[(b * N + n) * J->dim + d]"),
    ("initial state indexed [n][b][d]", "J->h0[flat * N + n]", "J->h0[n * J->batch * J->dim + flat]"),
    ("conv taps reversed", "J->conv_w[d * W + k]", "J->conv_w[d * W + (W - 1 - k)]"),
    ("conv taps indexed [k][d]", "J->conv_w[d * W + k]", "J->conv_w[k * J->dim + d]"),
    ("conv window shifted", "const int64_t s = t - (W - 1) + k;", "const int64_t s = t - W + k;"),
    ("conv bias dropped", "double acc = J->conv_b ? (double)J->conv_b[d] : 0.0;", "double acc = 0.0;"),
    ("conv output without SiLU", "  return silu64(acc);", "  return acc;"),
    ("zoh through exp - 1", "expm1(dt * an)", "(exp(dt * an) - 1.0)"),
    ("zoh without the division by A", "expm1(dt * an) / an * b_t", "expm1(dt * an) * b_t"),
    ("zoh with Delta twice", "expm1(dt * an) / an * b_t", "expm1(dt * an) / an * dt * b_t"),
    ("zoh sign of A", "expm1(dt * an) / an * b_t", "expm1(-dt * an) / an * b_t"),
    ("bwd carry not decayed", "g[n] = a * gt;", "g[n] = gt;"),
    ("bwd dDelta misses the decay term", "ddt += gt * (bt * ut + an * a * prev);", "ddt += gt * bt * ut;"),
    ("bwd dz with the sigmoid only", "q * sg * (1.0 + zt * (1.0 - sg));", "q * sg;"),
    ("bwd dC from the previous state", "dC[bc + (int64_t)n * L + t] += dq * hs[t * N + n];",
     "dC[bc + (int64_t)n * L + t] += dq * prev;"),
    ("bwd softplus derivative dropped", "ddt * sigmoid64(x) : ddt", "ddt : ddt"),
    ("bwd dA without Delta", "gt * dt * a * prev", "gt * a * prev"),
    ("bwd du misses the skip", "du = dq * Dd;", "du = 0.0;"),
]

PIN_CALLS = [
    lambda: pins.test_lti_closed_form(False),
    lambda: pins.test_lti_closed_form(True),
    pins.test_tree_fold_equals_serial_oracle,
    pins.test_hold_limit_exact_zero_delta,
    pins.test_hold_limit_softplus_with_bias,
    pins.test_reset_limit,
    lambda: pins.test_bruteforce_unrolled(5),
    pins.test_prefix_sum_special_case,
    pins.test_index_plumbing_single_impulse,
    pins.test_initial_state_free_decay_closed_form,
    lambda: pins.test_initial_state_bruteforce(3),
    lambda: pins.test_conv_prologue_matches_numpy_convolution(4),
    pins.test_conv_prologue_impulse_taps,
    pins.test_zoh_matches_ode_integration,
    pins.test_zoh_small_delta_series,
    lambda: pins.test_backward_matches_finite_differences(True, True, True),
]


def _build_mutant(tmp_path, old, new):
    text = open(SRC).read()
    assert old in text, f"mutation target not found: {old!r}"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new, 1))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                           "-ffp-contract=off", "-o", str(lib), str(src), "-lm", "-lpthread"])
    return str(lib)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, monkeypatch, name, old, new):
    path = _build_mutant(tmp_path, old, new)
    real = oracle._load()
    lib = ctypes.CDLL(path)
    for fn in ("oracle_scan_fwd", "oracle_scan_bwd", "oracle_softplus", "oracle_silu"):
        f = getattr(lib, fn)
        f.argtypes = getattr(real, fn).argtypes
        f.restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = []
    for call in PIN_CALLS:
        try:
            call()
        except AssertionError:
            failed.append(call)
    assert failed, f"no pin caught the mutant '{name}'"
