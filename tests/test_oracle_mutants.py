"""The pins must catch plausible mistakes in the oracle.

Each case copies ``oracle/gdn2_oracle.c`` to a temporary directory, plants one
mistake by text substitution (a dropped term, a wrong sign, a swapped
operand), compiles it with gcc and checks that the brute-force / worked-example
pins reject it.  Mistakes are planted only in these CPU copies.
"""
import json
import os
import subprocess

import numpy as np
import pytest

import oracle
from test_oracle_pins import HERE, brute_force_head, head, rand_inputs, rel_err

MUTANTS = {
    "write_sign": ("row[j] += ki * u[j];", "row[j] -= ki * u[j];"),
    "erase_sign": ("u[j] = (double)wt[j] * (double)vt[j] - r[j];",
                   "u[j] = (double)wt[j] * (double)vt[j] + r[j];"),
    "erase_gate_dropped": ("const double bk = (double)bt[i] * (double)kt[i];",
                           "const double bk = (double)kt[i];"),
    "decay_dropped": ("const double a = exp((double)lat[i]);", "const double a = 1.0;"),
    "decay_inverted": ("const double a = exp((double)lat[i]);",
                       "const double a = exp(-(double)lat[i]);"),
    "write_gate_dropped": ("u[j] = (double)wt[j] * (double)vt[j] - r[j];",
                           "u[j] = (double)vt[j] - r[j];"),
    "query_is_key": ("const double qi = (double)qt[i];", "const double qi = (double)kt[i];"),
    "erase_on_query": ("const double bk = (double)bt[i] * (double)kt[i];",
                       "const double bk = (double)bt[i] * (double)qt[i];"),
}


def _pins_pass(lib) -> bool:
    rng = np.random.default_rng(101)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 2, 17, 2, 5, 4)
    o, ST = oracle.forward(q, k, v, la, b, w, S0=S0, lib=lib)
    for bi in range(2):
        for hi in range(2):
            ob, Sb = brute_force_head(*(head(x, bi, hi) for x in (q, k, v, la, b, w)), S0[bi, hi])
            if rel_err(o[bi * 2 + hi], ob) > 1e-12 or rel_err(ST[bi * 2 + hi], Sb) > 1e-12:
                return False
    with open(os.path.join(HERE, "golden", "worked_example_dk2_dv1.json")) as f:
        g = json.load(f)
    inp = g["inputs"]
    sh = lambda x: np.asarray(x, dtype=np.float64)[None, :, None, :]
    o, ST = oracle.forward(sh(inp["q"]), sh(inp["k"]), sh(inp["v"]),
                           sh(np.log(np.asarray(inp["alpha"]))), sh(inp["b"]), sh(inp["w"]),
                           S0=np.asarray(inp["S0"])[None, None], lib=lib)
    return bool(np.allclose(o[0], g["expected"]["o"], atol=1e-7)
                and np.allclose(ST[0], g["expected"]["S_T"], atol=1e-7))


def _compile(src_text: str, tmp_path, name: str):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src_text)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    return oracle.open_library(str(so))


@pytest.fixture(scope="module")
def oracle_source():
    with open(os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")) as f:
        return f.read()


def test_unmutated_copy_passes(oracle_source, tmp_path):
    assert _pins_pass(_compile(oracle_source, tmp_path, "clean"))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(oracle_source, tmp_path, name):
    old, new = MUTANTS[name]
    assert oracle_source.count(old) == 1, f"mutation site for {name} not found"
    lib = _compile(oracle_source.replace(old, new), tmp_path, name)
    assert not _pins_pass(lib), f"pins did not catch mutant {name}"
