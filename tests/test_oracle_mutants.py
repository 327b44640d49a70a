"""The pins must catch plausible mistakes in the oracle. Each case plants one mistake in a
copy of oracle/gdn2_ref.c (on the CPU, in a temporary directory), builds it, and runs the
pin suite against the mutant; the suite has to fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn2_ref.c")

MUTANTS = {
    "no_decay": ("exp((double)log_alpha[kd_base + i])", "1.0"),
    "erase_with_write_gate": ("elem(b, kd_base + i, dtype)", "elem(w, vd_base + i, dtype)"),
    "erase_sign": ("-= ei * r[j]", "+= ei * r[j]"),
    "write_without_gate": ("ki * (elem(w, vd_base + j, dtype) * elem(v, vd_base + j, dtype))",
                           "ki * elem(v, vd_base + j, dtype)"),
    "transposed_key_read": ("r[j] += ki * S[(size_t)i * dv + j]", "r[j] += ki * S[(size_t)j * dv + i]"),
    "query_reads_with_key": ("acc += elem(q, qk_base + i, dtype)", "acc += elem(k, qk_base + i, dtype)"),
    "wrong_head_group": ("const int g = h / group;", "const int g = h % h_qk;"),
    "decay_by_value_index": ("S[(size_t)i * dv + j] *= alpha", "S[(size_t)j * dv + i] *= alpha"),
    "erase_uses_query": ("* elem(k, qk_base + i, dtype);\n", "* elem(q, qk_base + i, dtype);\n"),
    "no_state_reset": ("S[i] = S0 ? (double)S0[((size_t)n * h_v + h) * dk * dv + i] : 0.0;",
                       "if (t0 == 0) S[i] = S0 ? (double)S0[((size_t)n * h_v + h) * dk * dv + i] : 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mut = src.replace(old, new)
    c = tmp_path / "gdn2_ref.c"
    c.write_text(mut.replace('#include "../include/gdn2_ref.h"',
                             f'#include "{os.path.join(ROOT, "include", "gdn2_ref.h")}"'))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c), "-lm"],
                   check=True)
    env = dict(os.environ, GDN2_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
