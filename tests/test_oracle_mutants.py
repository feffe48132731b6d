"""Planted mistakes in the oracle must fail its pins (CPU only).

Each case copies the oracle's C source, changes one line to a plausible slip,
compiles the copy to a temporary library and runs the pin suite against it in
a child process.  The suite must fail for every mutant; the unmodified source
must pass (covered by test_oracle_pins itself).
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "grinqh_oracle.c")

MUTANTS = {
    "phi_applied_at_full_width":
        ("phi[k] = (b < b_max) ? ldexp(1.0, b_max - b - 1) : 0.0;",
         "phi[k] = ldexp(1.0, b_max - b - 1);"),
    "phi_dropped":
        ("return sv * (Q + phi[b / 2]) + zv;", "return sv * Q + zv;"),
    "zero_point_dropped":
        ("return sv * (Q + phi[b / 2]) + zv;", "return sv * (Q + phi[b / 2]);"),
    "plane_order_reversed_in_pack":
        ("int src = 2 * (P - 1 - p) + bit; /* bit of the code */",
         "int src = 2 * p + bit; /* bit of the code */"),
    "plane_significance_reversed":
        ("Q += (double)slice * ldexp(1.0, 2 * (P - 1 - p));",
         "Q += (double)slice * ldexp(1.0, 2 * p);"),
    "reads_one_plane_too_many":
        ("for (int p = 0; p < b / 2; p++) {", "for (int p = 0; p < b / 2 + (b < 2 * P); p++) {"),
    "ties_take_lower_level":
        ("if ((double)theta[k] <= a) count++;", "if ((double)theta[k] < a) count++;"),
    "nan_takes_full_width":
        ("if ((double)theta[k] <= a) count++;", "if (!((double)theta[k] > a)) count++;"),
    "skipped_rows_contribute_z":
        ("if (b[i] == 0) continue; /* R8: skipped row, no load */", ""),
    "group_index_ignored":
        ("int g = i / ORACLE_GROUP;\n    double sv", "int g = 0;\n    double sv"),
    "sign_flipped":
        ("acc += xv * w;\n            acc_abs += fabs(w) * fabs(xv);\n        }\n        y[k] = acc;\n        bound[k] = acc_abs;\n    }\n}\n\n/* ---- Dense",
         "acc -= xv * w;\n            acc_abs += fabs(w) * fabs(xv);\n        }\n        y[k] = acc;\n        bound[k] = acc_abs;\n    }\n}\n\n/* ---- Dense"),
    "field_position_shifted":
        ("int dst = 2 * t + bit;           /* bit of the word */",
         "int dst = (2 * t + bit + 2) % 32; /* bit of the word */"),
    "list_membership_off_by_one":
        ("if (b[i] > 2 * p) {", "if (b[i] >= 2 * p) {"),
    "f16_exponent_bias":
        ("v = ldexp((double)(1024 + f), e - 25);", "v = ldexp((double)(1024 + f), e - 24);"),
    "f16_subnormal_scale":
        ("v = ldexp((double)f, -24);", "v = ldexp((double)f, -25);"),
    "dense4_nibble_order":
        ("if ((code >> bit) & 1) word |= (uint32_t)1 << (4 * t + bit);",
         "if ((code >> bit) & 1) word |= (uint32_t)1 << (4 * (7 - t) + bit);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/found"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(old, new))
    lib = oracle.compile_source(str(mut_src), str(tmp_path / "libmutant.so"))
    env = dict(os.environ, GRINQH_ORACLE_LIB_OVERRIDE=lib)
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
         os.path.join(ROOT, "tests", "test_oracle_pins.py")],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout, r.stdout[-2000:]
