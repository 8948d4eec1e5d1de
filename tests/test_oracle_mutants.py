"""The pins must catch plausible mistakes in the oracle.

Each case copies ``oracle/gdn2_oracle.c`` to a temporary directory, plants one
mistake by text substitution (a dropped term, a wrong sign, a swapped
operand), compiles it with gcc and checks that the brute-force / worked-example
pins reject it (the input-prep and epilogue mistakes against the fused pins).
Mistakes are planted only in these CPU copies.
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
    "erase_sign": ("u[j] = wd[j] * (double)vt[j] - r[j];", "u[j] = wd[j] * (double)vt[j] + r[j];"),
    "erase_gate_dropped": ("const double bk = bd[i] * kd[i];", "const double bk = kd[i];"),
    "decay_dropped": ("const double a = exp((double)lat[i]);", "const double a = 1.0;"),
    "decay_inverted": ("const double a = exp((double)lat[i]);",
                       "const double a = exp(-(double)lat[i]);"),
    "write_gate_dropped": ("u[j] = wd[j] * (double)vt[j] - r[j];", "u[j] = (double)vt[j] - r[j];"),
    "query_is_key": ("const double qi = qd[i];", "const double qi = kd[i];"),
    "erase_on_query": ("const double bk = bd[i] * kd[i];", "const double bk = bd[i] * qd[i];"),
}

# mistakes in the optional input prep and output epilogue
FUSED_MUTANTS = {
    "l2_without_sqrt": ("const double nq = sqrt(sq + f->l2_eps), nk = sqrt(sk + f->l2_eps);",
                        "const double nq = sq + f->l2_eps, nk = sk + f->l2_eps;"),
    "l2_key_skipped": ("kd[i] *= ik;", "kd[i] *= 1.0;"),
    "logistic_sign": ("static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }",
                      "static double sigmoid(double x) { return 1.0 / (1.0 + exp(x)); }"),
    "neg_eigval_ignored": ("(f->neg_eigval ? 2.0 : 1.0)", "(1.0)"),
    "write_gate_left_raw": ("for (long j = 0; j < dv; ++j) wd[j] = sigmoid(wd[j]);", ""),
    "rms_sum_not_mean": ("sqrt(ms / (double)dv + f->norm_eps)", "sqrt(ms + f->norm_eps)"),
    "silu_is_sigmoid": ("(gj * sigmoid(gj))", "sigmoid(gj)"),
    "norm_weight_dropped": ("ot[j] * inv * f->weight[j] * ", "ot[j] * inv * "),
}


# mistakes in the second, query-derived erase (forward_qed)
QED_MUTANTS = {
    "qed_erase_sign": ("row[j] -= ui * r2[j];", "row[j] += ui * r2[j];"),
    "qed_not_orthogonal": ("const double coef = kk > 0.0 ? qk / kk : 0.0;", "const double coef = 0.0;"),
    "qed_not_normalised": ("const double inr = nr > 0.0 ? 1.0 / nr : 0.0;", "const double inr = 1.0;"),
    "qed_gate_on_key": ("const double cu = cd[i] * ud[i];", "const double cu = cd[i] * kd[i];"),
    "qed_gate_left_raw": ("cd[i] = f->prep ? sigmoid((double)ct[i]) : (double)ct[i];", "cd[i] = (double)ct[i];"),
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


def _fused_pins_pass(lib) -> bool:
    import test_oracle_fused_pins as fp

    class _Mod:   # the oracle module's forward, bound to this library
        @staticmethod
        def forward(*a, **kw):
            return oracle.forward(*a, lib=lib, **kw)

    checks = [lambda: fp.test_input_prep_worked_example(_Mod, "plain"),
              lambda: fp.test_input_prep_worked_example(_Mod, "neg_eigval"),
              lambda: fp.test_output_epilogue_worked_example(_Mod),
              lambda: fp.test_prep_is_scale_invariant_in_q_and_k(_Mod),
              lambda: fp.test_epilogue_constant_row_and_zero_gate(_Mod)]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def _qed_pins_pass(lib) -> bool:
    import test_oracle_qed_pins as qp

    class _Mod:   # the oracle module's functions, bound to this library
        @staticmethod
        def forward(*a, **kw):
            return oracle.forward(*a, lib=lib, **kw)

        @staticmethod
        def forward_qed(*a, **kw):
            return oracle.forward_qed(*a, lib=lib, **kw)

    checks = [lambda: qp.test_qed_brute_force_matrix_form(_Mod, 2, 21, 2, 6, 5, 1e-6),
              lambda: qp.test_qed_full_erase_read_sees_only_the_key_part(_Mod),
              lambda: qp.test_qed_prep_gates_c_with_the_logistic(_Mod)]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


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
    lib = _compile(oracle_source, tmp_path, "clean")
    assert _pins_pass(lib) and _fused_pins_pass(lib) and _qed_pins_pass(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(oracle_source, tmp_path, name):
    old, new = MUTANTS[name]
    assert oracle_source.count(old) == 1, f"mutation site for {name} not found"
    lib = _compile(oracle_source.replace(old, new), tmp_path, name)
    assert not _pins_pass(lib), f"pins did not catch mutant {name}"


@pytest.mark.parametrize("name", sorted(FUSED_MUTANTS))
def test_fused_mutant_is_caught(oracle_source, tmp_path, name):
    old, new = FUSED_MUTANTS[name]
    assert oracle_source.count(old) == 1, f"mutation site for {name} not found"
    lib = _compile(oracle_source.replace(old, new), tmp_path, name)
    assert not _fused_pins_pass(lib), f"fused pins did not catch mutant {name}"


@pytest.mark.parametrize("name", sorted(QED_MUTANTS))
def test_qed_mutant_is_caught(oracle_source, tmp_path, name):
    old, new = QED_MUTANTS[name]
    assert oracle_source.count(old) == 1, f"mutation site for {name} not found"
    lib = _compile(oracle_source.replace(old, new), tmp_path, name)
    assert not _qed_pins_pass(lib), f"QED pins did not catch mutant {name}"
