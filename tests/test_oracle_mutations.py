"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
never in the CUDA path), builds it, and runs the pin suite against that build
in a subprocess: the suite must fail.  The unmodified source must pass.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lq_oracle.c")

MUTATIONS = {
    "drop_compensator_rows": (
        "Sh[(size_t)row * dk + j] += (double)comp_val[(size_t)c * dk + j];", ";"),
    "wrong_sign_update": ("u[i] = vt[i] - acc;", "u[i] = vt[i] + acc;"),
    "decay_off_by_one": (
        "for (int j = 0; j < dk; ++j) x[j] = decay(L, gdim, t - 1, 0, j) * bt[j];",
        "for (int j = 0; j < dk; ++j) x[j] = decay(L, gdim, t, 0, j) * bt[j];"),
    "output_drops_own_token": ("for (int m = 1; m <= t; ++m) {", "for (int m = 1; m < t; ++m) {"),
    "rebuild_drops_last_record": ("for (int m = 1; m <= n; ++m)", "for (int m = 1; m < n; ++m)"),
    "gate_index_transposed": (
        "Sh[(size_t)i * dk + j] = Sh[(size_t)i * dk + j] * dt[j] + u[i] * kk[j];",
        "Sh[(size_t)i * dk + j] = Sh[(size_t)i * dk + j] * dt[i % dk] + u[i] * kk[j];"),
    "ties_to_larger_row": ("norm[i] > norm[best]", "norm[i] >= norm[best]"),
    "smoothing_without_sqrt": ("(float)sqrt(m) : 1.0f", "(float)m : 1.0f"),
    "round_half_away": ("qv = rint(f32(", "qv = round(f32("),
    "inverse_scale_product": ("qv = rint(f32(R[(size_t)i * dk + j] / sigma));",
                              "qv = rint(f32(R[(size_t)i * dk + j] * f32(1.0 / sigma)));"),
    "inverse_smoothing_product": (
        "R[(size_t)i * dk + j] = f32(R[(size_t)i * dk + j] / (double)c[j]);",
        "R[(size_t)i * dk + j] = f32(R[(size_t)i * dk + j] * f32(1.0 / (double)c[j]));"),
    "scale_255": ("double sigma = f32(mx / qmax);", "double sigma = f32(mx / (2.0 * qmax + 1.0));"),
    "code_range_one_too_wide": ("const double qmax = (double)((1 << (bits - 1)) - 1);",
                                "const double qmax = (double)(1 << (bits - 1));"),
    "svd_compensators_dropped": ("Sh[(size_t)i * dk + j] += (double)comp_u[(size_t)c * dv + i] *",
                                 "Sh[(size_t)i * dk + j] += 0.0 * comp_u[(size_t)c * dv + i] *"),
    "svd_compensator_transposed": ("(double)comp_val[(size_t)c * dk + j];\n            continue;",
                                   "(double)comp_val[(size_t)c * dk + (j + 1) % dk];\n            continue;"),
    "bf16_truncates": ("return ldexp(rint(ldexp(m, 8)), e - 8);",
                       "return ldexp(trunc(ldexp(m, 8)), e - 8);"),
    "bf16_keeps_9_bits": ("return ldexp(rint(ldexp(m, 8)), e - 8);",
                          "return ldexp(rint(ldexp(m, 9)), e - 9);"),
    "code_width_fixed_at_8": ("const double qmax = (double)((1 << (bits - 1)) - 1);",
                              "const double qmax = 127.0;"),
}


def _build(src_text, out_dir):
    c = os.path.join(out_dir, "lq_oracle.c")
    so = os.path.join(out_dir, "liblq_oracle.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                    "-o", so, c, "-lm"], check=True)
    return so


def _run_pins(so):
    env = dict(os.environ, LQ_ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    with tempfile.TemporaryDirectory() as d:
        so = _build(src.replace(old, new), d)
        assert _run_pins(so) != 0, f"pins did not catch mutation {name}"


def test_unmutated_oracle_passes_pins():
    with tempfile.TemporaryDirectory() as d:
        assert _run_pins(_build(open(SRC).read(), d)) == 0
