"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of the oracle's C source (on the CPU),
builds it, and runs the pin suite against the copy in a subprocess: the run
must fail. This shows that a dropped term, a wrong sign, a wrong index or a
reversed traversal in the oracle cannot pass the pins unnoticed.
"""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "mala_oracle.c")

MUTATIONS = {
    "forward test drops ln l": ("const double lhs = mt[r] - m[r] - log(l[r]);",
                                "const double lhs = mt[r] - m[r];"),
    "threshold sign of ln Lq": ("return log(tau) - log(Lq);", "return log(tau) + log(Lq);"),
    "forward drops rescale": ("for (int k = 0; k < d; ++k) a[k] *= alpha;\n        double lsum = l[r] * alpha;\n        for (int c = c0; c < c1; ++c) {\n          const double p = exp(s[(size_t)r * T + (c - c0)] - mnew);\n          lsum += p;\n          const double *vc",
                              "double lsum = l[r] * alpha;\n        for (int c = c0; c < c1; ++c) {\n          const double p = exp(s[(size_t)r * T + (c - c0)] - mnew);\n          lsum += p;\n          const double *vc"),
    "forward traversal reversed": ("for (int j = i; j >= 0; --j) {\n      const int c0 = j * T;\n      /* scores",
                                   "for (int j = 0; j <= i; ++j) {\n      const int c0 = j * T;\n      /* scores"),
    "backward D sign": ("const double ds = p * (dp - D[row]);\n          for (int k = 0; k < d; ++k) {",
                        "const double ds = p * (dp + D[row]);\n          for (int k = 0; k < d; ++k) {"),
    "backward dK transposed operand": ("dK[(size_t)c * d + k] += scale * ds * Q[(size_t)row * d + k];",
                                       "dK[(size_t)c * d + k] += scale * ds * K[(size_t)row * d + k];"),
    "backward forces the diagonal tile": ("if (force_first && j == i) { *mu_out = INFINITY; return 1; }",
                                          "if (j == i) { *mu_out = INFINITY; return 1; }"),
    "backward test uses row max of wrong row": ("const double crit = (mx - LSE[row]) - log_threshold(tau, (double)(row + 1));",
                                                "const double crit = (mx - LSE[r0]) - log_threshold(tau, (double)(row + 1));"),
    "decode threshold length": ("const double lthr = log_threshold(tau, (double)Lc);",
                                "const double lthr = log_threshold(tau, (double)T);"),
    "decode group test reads the first head only": (
        "for (int r = 0; r < rows; ++r) {\n          const double crit = (mt[r] - m[r] - log(l[r])) - lthr;",
        "for (int r = 0; r < 1; ++r) {\n          const double crit = (mt[r] - m[r] - log(l[r])) - lthr;"),
    "decode group test needs every head": (
        "kept = 0;\n        for (int r = 0; r < rows; ++r) {\n          const double crit = (mt[r] - m[r] - log(l[r])) - lthr;\n          if (crit > mu) mu = crit;\n          if (crit >= 0.0) kept = 1;",
        "kept = 1;\n        for (int r = 0; r < rows; ++r) {\n          const double crit = (mt[r] - m[r] - log(l[r])) - lthr;\n          if (crit > mu) mu = crit;\n          if (crit < 0.0) kept = 0;"),
    "decode traversal oldest first": ("for (int t = nt - 1; t >= 0; --t) {\n      const int c0 = t * T, c1 = imin(Lc, (t + 1) * T);",
                                      "for (int t = 0; t < nt; ++t) {\n      const int c0 = t * T, c1 = imin(Lc, (t + 1) * T);"),
    "decode scores use the group's first head": (
        "const double v = scale * dot(q + (size_t)(h0 + r) * d, Kg + (size_t)c * d, d);",
        "const double v = scale * dot(q + (size_t)h0 * d, Kg + (size_t)c * d, d);"),
    "chunk threshold ignores the cache": (
        "const double crit = lhs - log_threshold(tau, (double)(off + r0 + r + 1));",
        "const double crit = lhs - log_threshold(tau, (double)(r0 + r + 1));"),
    "chunk key tiles not aligned to the blocks": (
        "const int p0 = off + T * (k - koff);", "const int p0 = T * (k - koff);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    # a formula shared by the prefill forward and its chunk variant is
    # mutated in both (the same mistake made twice)
    assert src.count(old) >= 1, "mutation anchor not found"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(mutated),
                    "-o", str(lib), "-lm"], check=True)
    env = dict(os.environ, MALA_ORACLE_LIB=str(lib), OMP_NUM_THREADS="4")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins passed with mutation '{name}'"
