"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a private copy of ``oracle/carve_oracle.c``
(CPU only), builds it, and runs the pin suite against it in a subprocess;
the suite must fail.  The unmodified oracle passes the same suite
(``test_oracle_pins.py``).
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "carve_oracle.c")

MUTANTS = {
    # erase ignores the gate b (value-blind erase of the plain delta rule)
    "erase_without_gate": ("-e[v] * (erase ? k[j] : b[j] * k[j])",
                           "-e[v] * (erase ? k[j] : k[j])"),
    # erase with the wrong sign
    "erase_sign": ("-e[v] * (erase ? k[j] : b[j] * k[j]) + w",
                   "e[v] * (erase ? k[j] : b[j] * k[j]) + w"),
    # decay applied on the value axis instead of the key axis
    "decay_on_value_axis": ("S[(size_t)v * DK + j] *= alpha[j];",
                            "S[(size_t)v * DK + j] *= alpha[v % DK];"),
    # write gate dropped
    "no_write_gate": ("+ w * vv[v] * k[j]", "+ vv[v] * k[j]"),
    # chunk mean divides by the tokens present instead of L
    "mean_divisor": ("m[vv] = msum[vv] / (double)L;\n  }\n  if (S_T)",
                     "m[vv] = msum[vv] / (double)(t1 - t0);\n  }\n  if (S_T)"),
    # U_up read transposed
    "u_up_transposed": ("acc += u_up[(size_t)j * R + r] * h[r];",
                        "acc += u_up[(size_t)r * DK + j] * h[r];"),
    # gate derivative of the sigmoid dropped in the reverse pass
    "bwd_sigmoid_derivative": ("db * b[j] * (1.0 - b[j])", "db * b[j]"),
    # chunk-mean share of the upstream gradient not divided by L
    "bwd_mean_share": ("dm_next[vv] / (double)L;", "dm_next[vv];"),
    # other erase form: the state read with the ungated key
    "erase1_ungated_read": ("(erase ? b[j] * k[j] : k[j])",
                            "(erase ? k[j] : k[j])"),
    # other erase form: reverse pass with the wrong sign on the written key
    "erase1_bwd_sign": ("dk[(size_t)t * DK + j] -= acc;",
                        "dk[(size_t)t * DK + j] += acc;"),
    # reverse pass forgets the decay on the carried state gradient
    "bwd_decay": ("dS[(size_t)vv * DK + j] * alpha[j] + dot[vv] * qt[j]",
                  "dS[(size_t)vv * DK + j] + dot[vv] * qt[j]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not unique: " + name
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared",
                           "-o", str(lib), str(mutant), "-lm"])
    env = dict(os.environ, CARVE_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x",
                        "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True)
    assert r.returncode != 0, "pins did not catch mutant " + name
