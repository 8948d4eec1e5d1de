"""Pins for the oracle's optional input prep and output epilogue.

The burn-gdn2 README ("Architecture") draws an L2-Norm of q and k before the
mixer and a SiLU-gated RMS norm after it; "Configuration" gives
``allow_neg_eigval`` (b x 2) and ``norm_eps``.  These tests pin the oracle's
versions of both steps against hand-worked examples (``tests/golden/``) and
against properties the definitions fix: scale invariance of the L2 norm, the
logistic function's values at 0 and +-ln 3, scale and sign behaviour of the
RMS norm, and silu(0) = 0.
"""
import json
import math
import os

import numpy as np
import pytest

from test_oracle_pins import HERE, rand_inputs, rel_err

LN3 = math.log(3.0)


def _num(x):
    return {"ln3": LN3, "-ln3": -LN3, "0": 0.0}[x] if isinstance(x, str) else float(x)


def _closed(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"sqrt": math.sqrt, "ln3": LN3}))


def _sh(x):
    """[T, d] -> [1, T, 1, d]"""
    return np.asarray([[_num(e) for e in row] for row in x], dtype=np.float64)[None, :, None, :]


def _golden(name):
    with open(os.path.join(HERE, "golden", name)) as f:
        return json.load(f)


@pytest.mark.parametrize("case", ["plain", "neg_eigval"])
def test_input_prep_worked_example(oracle_mod, case):
    g = _golden("input_prep_example_dk4_dv1.json")
    inp = g["inputs"]
    o, ST = oracle_mod.forward(_sh(inp["q_raw"]), _sh(inp["k_raw"]), _sh(inp["v"]),
                               np.log(_sh(inp["alpha"])), _sh(inp["b_raw"]), _sh(inp["w_raw"]),
                               S0=np.asarray(inp["S0"])[None, None], prep=True,
                               allow_neg_eigval=(case == "neg_eigval"), l2_eps=g["l2_eps"])
    exp = g["expected"][case]
    # the raw gates pass through float32 (ln 3 is not exact there): 1e-7 relative
    np.testing.assert_allclose(o[0], exp["o"], rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(ST[0], exp["S_T"], rtol=1e-6, atol=1e-7)


def test_output_epilogue_worked_example(oracle_mod):
    g = _golden("output_epilogue_example_dk1_dv2.json")
    inp = g["inputs"]
    y, ST = oracle_mod.forward(_sh(inp["q"]), _sh(inp["k"]), _sh(inp["v"]), np.log(_sh(inp["alpha"])),
                               _sh(inp["b"]), _sh(inp["w"]), S0=np.asarray(inp["S0"])[None, None],
                               gate=_sh(inp["gate"]), norm_weight=np.asarray(inp["weight"]),
                               norm_eps=g["norm_eps"])
    want_y = [[_closed(e) for e in row] for row in g["expected_closed_form"]["y"]]
    want_s = [[_closed(e) for e in row] for row in g["expected_closed_form"]["S_T"]]
    np.testing.assert_allclose(y[0], want_y, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(ST[0], want_s, rtol=0, atol=1e-12)


def _raw_inputs(rng, B, T, H, dk, dv):
    q, k, v, la, b, w, S0 = rand_inputs(rng, B, T, H, dk, dv)
    # raw projections: unnormalised q, k; gate logits for b, w
    return (rng.standard_normal((B, T, H, dk)) * 3, rng.standard_normal((B, T, H, dk)) * 0.5, v, la,
            rng.standard_normal((B, T, H, dk)), rng.standard_normal((B, T, H, dv)), S0)


def test_prep_is_scale_invariant_in_q_and_k(oracle_mod):
    rng = np.random.default_rng(31)
    q, k, v, la, b, w, S0 = _raw_inputs(rng, 1, 40, 2, 8, 5)
    lam = rng.uniform(0.25, 4.0, size=(1, 40, 2, 1))
    o1, S1 = oracle_mod.forward(q, k, v, la, b, w, S0=S0, prep=True, l2_eps=0.0)
    o2, S2 = oracle_mod.forward(q * lam, k * lam[:, ::-1], v, la, b, w, S0=S0, prep=True, l2_eps=0.0)
    # the float32 pass of the scaled raw values is the only difference
    assert rel_err(o1, o2) < 1e-6 and rel_err(S1, S2) < 1e-6


def test_prep_equals_recurrence_on_prepared_inputs(oracle_mod):
    """prep=True on (q_raw, k_raw, logit(b), logit(w)) is the plain recurrence on
    (q_raw/|q_raw|, k_raw/|k_raw|, b, w): the logistic function inverts the logit."""
    rng = np.random.default_rng(32)
    q, k, v, la, _, _, S0 = _raw_inputs(rng, 2, 24, 2, 6, 4)
    bq = rng.uniform(0.05, 0.95, size=(2, 24, 2, 6))
    wq = rng.uniform(0.05, 0.95, size=(2, 24, 2, 4))
    for neg in (False, True):
        braw = np.log(bq / (1 - bq))
        o1, S1 = oracle_mod.forward(q, k, v, la, braw, np.log(wq / (1 - wq)), S0=S0, prep=True,
                                    allow_neg_eigval=neg, l2_eps=0.0)
        qn = q / np.linalg.norm(q, axis=-1, keepdims=True)
        kn = k / np.linalg.norm(k, axis=-1, keepdims=True)
        o2, S2 = oracle_mod.forward(qn, kn, v, la, bq * (2 if neg else 1), wq, S0=S0)
        assert rel_err(o1, o2) < 1e-5 and rel_err(S1, S2) < 1e-5


def test_prep_zero_query_is_finite(oracle_mod):
    rng = np.random.default_rng(33)
    q, k, v, la, b, w, S0 = _raw_inputs(rng, 1, 8, 1, 4, 3)
    q[0, 3] = 0.0
    o, _ = oracle_mod.forward(q, k, v, la, b, w, S0=S0, prep=True, l2_eps=1e-6)
    assert np.all(np.isfinite(o)) and np.all(o[0, 3] == 0.0)


@pytest.mark.parametrize("lam", [0.5, 3.0, -2.0])
def test_epilogue_scale_and_sign(oracle_mod, lam):
    """With S0 = 0 the map v -> o is linear, and RMSNorm(lam o) = sign(lam) RMSNorm(o)
    when eps = 0."""
    rng = np.random.default_rng(34)
    q, k, v, la, b, w, _ = rand_inputs(rng, 1, 30, 2, 6, 5)
    gate = rng.standard_normal((1, 30, 2, 5))
    wt = rng.standard_normal(5)
    y1, _ = oracle_mod.forward(q, k, v, la, b, w, gate=gate, norm_weight=wt, norm_eps=0.0)
    y2, _ = oracle_mod.forward(q, k, v * lam, la, b, w, gate=gate, norm_weight=wt, norm_eps=0.0)
    assert rel_err(y2, np.sign(lam) * y1) < 1e-6


def test_epilogue_constant_row_and_zero_gate(oracle_mod):
    """d_k = 1, q = k = 1, b = 0, alpha = 1, S0 = 0: o_t = sum_{s<=t} w_s v_s.  With v
    constant across d_v the row is constant c, so y_j = sign(c) weight_j silu(g_j);
    silu(0) = 0 zeroes the entry."""
    T, dv = 5, 4
    ones = np.ones((1, T, 1, 1))
    v = np.broadcast_to(np.array([2.0, -1.0, -3.0, 0.5, 4.0])[None, :, None, None], (1, T, 1, dv)).copy()
    gate = np.tile(np.array([0.0, LN3, -LN3, 1.0])[None, None, None, :], (1, T, 1, 1))
    wt = np.array([1.5, -2.0, 0.5, 1.0])
    y, _ = oracle_mod.forward(ones, ones, v, np.zeros((1, T, 1, 1)), np.zeros((1, T, 1, 1)),
                              np.ones((1, T, 1, dv)), gate=gate, norm_weight=wt, norm_eps=0.0)
    c = np.cumsum(v[0, :, 0, 0])
    silu = np.array([0.0, 0.75 * LN3, -0.25 * LN3, 1.0 / (1.0 + math.exp(-1.0))])
    # the gate passes through float32 (ln 3 is not exact there)
    np.testing.assert_allclose(y[0], np.sign(c)[:, None] * (wt * silu)[None, :], rtol=1e-7, atol=1e-12)


def test_decode_steps_with_prep_and_epilogue_match_forward(oracle_mod):
    rng = np.random.default_rng(35)
    q, k, v, la, b, w, S0 = _raw_inputs(rng, 2, 6, 2, 4, 3)
    gate = rng.standard_normal((2, 6, 2, 3))
    wt = rng.standard_normal(3)
    kw = dict(prep=True, allow_neg_eigval=True, gate=gate, norm_weight=wt)
    o1, S1 = oracle_mod.forward(q, k, v, la, b, w, S0=S0, **kw)
    tb = lambda x: np.swapaxes(x, 0, 1)
    kw["gate"] = tb(gate)
    o2, S2 = oracle_mod.decode_steps(tb(q), tb(k), tb(v), tb(la), tb(b), tb(w), S0, **kw)
    assert rel_err(o1, o2) < 1e-14 and rel_err(S1, S2) < 1e-14


def test_fused_arguments_are_checked(oracle_mod):
    rng = np.random.default_rng(36)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 1, 4, 1, 2, 2)
    with pytest.raises(AssertionError):
        oracle_mod.forward(q, k, v, la, b, w, gate=np.zeros((1, 4, 1, 2)))   # no weight
    with pytest.raises(ValueError):
        oracle_mod.forward(q, k, v, la, b, w, prep=True, l2_eps=-1.0)
