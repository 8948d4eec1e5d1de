"""Pins for the fp64 oracle: checks against things the pages and mathematics fix.

The oracle (``oracle/gdn2_oracle.c``) writes the burn-gdn2 README recurrence
("Architecture" section) token by token with the erase applied as a rank-1
update.  Everything below computes the expected result a different way:

* an explicit d_k x d_k transition matrix per token (brute force);
* closed forms of special cases -- b = 0 with alpha = 1 is causal linear
  attention, b = 0 alone is gated linear attention with per-channel decay;
* the collapses stated by the asapai.co.kr article on Gated DeltaNet-2 (the
  decay/gate comparison table): b = w = one scalar beta gives KDA, and a scalar
  decay on top gives Gated DeltaNet; each is written out here as its own
  recurrence;
* the scalar case d_k = d_v = 1, a first-order linear recurrence with a
  product-sum closed form (covers b in (0, 2), the "b x 2" negative-eigenvalue
  setting of the README configuration table);
* a hand-derived worked example (tests/golden);
* invariants: the delta-write identity, state split, linearity, w/v symmetry.
"""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_inputs(rng, B, T, H, dk, dv, *, b_scale=1.0, lo=0.8, hi=0.999, s0=True):
    q = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, dk))
    k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    la = np.log(rng.uniform(lo, hi, (B, T, H, dk))).astype(np.float32)
    b = (b_scale / (1 + np.exp(-rng.standard_normal((B, T, H, dk))))).astype(np.float32)
    w = (1 / (1 + np.exp(-rng.standard_normal((B, T, H, dv))))).astype(np.float32)
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5 if s0 else None
    return q, k, v, la, b, w, S0


def head(x, bi, hi):
    return np.asarray(x, dtype=np.float64)[bi, :, hi, :]


def brute_force_head(q, k, v, la, b, w, S0):
    """Explicit matrices: S <- (I - k (b.k)^T) diag(alpha) S + k (w.v)^T."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.copy()
    o = np.zeros((T, dv))
    for t in range(T):
        erase = np.eye(dk) - np.outer(k[t], b[t] * k[t])
        M = erase @ np.diag(np.exp(la[t]))
        S = M @ S + np.outer(k[t], w[t] * v[t])
        o[t] = S.T @ q[t]
    return o, S


def rel_err(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# --------------------------------------------------------------------------
# brute force on tiny inputs, several heads and batches (also pins indexing)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("B,T,H,dk,dv,bs", [(1, 7, 1, 3, 2, 1.0), (2, 19, 3, 5, 4, 1.0),
                                             (2, 33, 2, 8, 16, 2.0), (1, 64, 2, 16, 8, 2.0)])
def test_brute_force_matrix_form(oracle_mod, B, T, H, dk, dv, bs):
    rng = np.random.default_rng(10 + T)
    q, k, v, la, b, w, S0 = rand_inputs(rng, B, T, H, dk, dv, b_scale=bs)
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    for bi in range(B):
        for hi in range(H):
            n = bi * H + hi
            ob, Sb = brute_force_head(*(head(x, bi, hi) for x in (q, k, v, la, b, w)), S0[bi, hi])
            assert rel_err(o[n], ob) < 1e-12
            assert rel_err(ST[n], Sb) < 1e-12


def test_head_subset_and_order(oracle_mod):
    rng = np.random.default_rng(3)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 3, 11, 4, 6, 5)
    o_all, S_all = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    sel = [7, 0, 11, 5]
    o_s, S_s = oracle_mod.forward(q, k, v, la, b, w, S0=S0, heads=sel)
    for i, n in enumerate(sel):
        np.testing.assert_array_equal(o_s[i], o_all[n])
        np.testing.assert_array_equal(S_s[i], S_all[n])


def test_zero_state_default(oracle_mod):
    rng = np.random.default_rng(4)
    q, k, v, la, b, w, _ = rand_inputs(rng, 1, 9, 2, 4, 3, s0=False)
    o1, S1 = oracle_mod.forward(q, k, v, la, b, w, S0=None)
    o2, S2 = oracle_mod.forward(q, k, v, la, b, w, S0=np.zeros((1, 2, 4, 3)))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


# --------------------------------------------------------------------------
# worked example derived by hand
# --------------------------------------------------------------------------
def test_hand_worked_example(oracle_mod):
    with open(os.path.join(HERE, "golden", "worked_example_dk2_dv1.json")) as f:
        g = json.load(f)
    inp = g["inputs"]
    sh = lambda x: np.asarray(x, dtype=np.float64)[None, :, None, :]
    la = np.log(np.asarray(inp["alpha"]))
    o, ST = oracle_mod.forward(sh(inp["q"]), sh(inp["k"]), sh(inp["v"]), sh(la), sh(inp["b"]),
                               sh(inp["w"]), S0=np.asarray(inp["S0"])[None, None])
    np.testing.assert_allclose(o[0], np.asarray(g["expected"]["o"]), rtol=1e-7, atol=1e-7)
    np.testing.assert_allclose(ST[0], np.asarray(g["expected"]["S_T"]), rtol=1e-7, atol=1e-7)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------
def test_linear_attention_closed_form(oracle_mod):
    """b = 0, alpha = 1: o_t = S0^T q_t + sum_{i<=t} (q_t . k_i) (w_i . v_i)."""
    rng = np.random.default_rng(5)
    B, T, H, dk, dv = 2, 40, 2, 8, 6
    q, k, v, la, b, w, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la[:] = 0.0
    b[:] = 0.0
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    mask = np.tril(np.ones((T, T)))
    for bi in range(B):
        for hi in range(H):
            Q, K, V, W = (head(x, bi, hi) for x in (q, k, v, w))
            ref = (mask * (Q @ K.T)) @ (W * V) + Q @ S0[bi, hi]
            assert rel_err(o[bi * H + hi], ref) < 1e-12
            assert rel_err(ST[bi * H + hi], S0[bi, hi] + K.T @ (W * V)) < 1e-12


def test_gated_linear_attention_closed_form(oracle_mod):
    """b = 0: o_t = S0^T (e^{G_t} . q_t) + sum_{i<=t} sum_c q_tc k_ic e^{G_tc - G_ic} (w_i . v_i)."""
    rng = np.random.default_rng(6)
    B, T, H, dk, dv = 1, 30, 3, 5, 4
    q, k, v, la, b, w, S0 = rand_inputs(rng, B, T, H, dk, dv, lo=0.5, hi=0.99)
    b[:] = 0.0
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    for hi in range(H):
        Q, K, V, W, LA = (head(x, 0, hi) for x in (q, k, v, w, la))
        G = np.cumsum(LA, axis=0)
        ref = np.zeros((T, dv))
        for t in range(T):
            ref[t] = S0[0, hi].T @ (np.exp(G[t]) * Q[t])
            for i in range(t + 1):
                ref[t] += np.sum(Q[t] * K[i] * np.exp(G[t] - G[i])) * (W[i] * V[i])
        assert rel_err(o[hi], ref) < 1e-12
        Sref = np.exp(G[-1])[:, None] * S0[0, hi] + sum(
            np.outer(np.exp(G[-1] - G[i]) * K[i], W[i] * V[i]) for i in range(T))
        assert rel_err(ST[hi], Sref) < 1e-12


@pytest.mark.parametrize("bs", [1.0, 2.0])
def test_scalar_recurrence_closed_form(oracle_mod, bs):
    """d_k = d_v = 1: S_t = lambda_t S_{t-1} + k_t w_t v_t, lambda_t = (1 - b_t k_t^2) alpha_t.

    Closed form S_T = (prod_t lambda_t) S0 + sum_i (prod_{s>i} lambda_s) k_i w_i v_i.
    With bs = 2 the erase factor (1 - b k^2) is negative for b > 1 (|k| = 1).
    """
    rng = np.random.default_rng(7)
    T = 50
    q, k, v, la, b, w, S0 = rand_inputs(rng, 1, T, 1, 1, 1, b_scale=bs, lo=0.7, hi=1.0)
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    K, Q, V, W, LA, Bg = (head(x, 0, 0)[:, 0] for x in (k, q, v, w, la, b))
    lam = (1 - Bg * K * K) * np.exp(LA)
    if bs == 2.0:
        assert np.any(lam < 0)
    S = np.empty(T)
    for t in range(T):
        tail = np.prod(lam[:t + 1])
        S[t] = tail * S0[0, 0, 0, 0] + sum(np.prod(lam[i + 1:t + 1]) * K[i] * W[i] * V[i]
                                           for i in range(t + 1))
    assert rel_err(o[0, :, 0], Q * S) < 1e-12
    assert rel_err(ST[0, 0, 0], np.array(S[-1])) < 1e-12


# --------------------------------------------------------------------------
# KDA and Gated DeltaNet collapses
# --------------------------------------------------------------------------
def kda_head(q, k, v, la, beta, S0):
    """KDA: S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T."""
    T, dk = q.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        S = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ (np.exp(la[t])[:, None] * S) \
            + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def gdn_head(q, k, v, a, beta, S0):
    """Gated DeltaNet: S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, scalar a_t."""
    T, dk = q.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        S = a[t] * (S - beta[t] * np.outer(k[t], k[t] @ S)) + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


@pytest.mark.parametrize("bs", [1.0, 2.0])
def test_kda_collapse(oracle_mod, bs):
    rng = np.random.default_rng(8)
    B, T, H, dk, dv = 2, 25, 2, 6, 10
    q, k, v, la, _, _, S0 = rand_inputs(rng, B, T, H, dk, dv)
    beta = (bs / (1 + np.exp(-rng.standard_normal((B, T, H, 1))))).astype(np.float32)
    b = np.broadcast_to(beta, (B, T, H, dk)).copy()
    w = np.broadcast_to(beta, (B, T, H, dv)).copy()
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    for bi in range(B):
        for hi in range(H):
            ref_o, ref_S = kda_head(*(head(x, bi, hi) for x in (q, k, v, la)),
                                    head(beta, bi, hi)[:, 0], S0[bi, hi])
            assert rel_err(o[bi * H + hi], ref_o) < 1e-12
            assert rel_err(ST[bi * H + hi], ref_S) < 1e-12


def test_gdn_collapse(oracle_mod):
    rng = np.random.default_rng(9)
    B, T, H, dk, dv = 1, 40, 3, 7, 5
    q, k, v, la, _, _, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la_s = la[..., :1]
    la = np.broadcast_to(la_s, la.shape).copy()
    beta = (1 / (1 + np.exp(-rng.standard_normal((B, T, H, 1))))).astype(np.float32)
    b = np.broadcast_to(beta, (B, T, H, dk)).copy()
    w = np.broadcast_to(beta, (B, T, H, dv)).copy()
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    for hi in range(H):
        a = np.exp(head(la_s, 0, hi)[:, 0])
        ref_o, ref_S = gdn_head(*(head(x, 0, hi) for x in (q, k, v)), a,
                                head(beta, 0, hi)[:, 0], S0[0, hi])
        assert rel_err(o[hi], ref_o) < 1e-12
        assert rel_err(ST[hi], ref_S) < 1e-12


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------
def test_delta_write_invariant(oracle_mod):
    """k_t^T S_t = (k_t - |k_t|^2 (b_t . k_t))^T diag(alpha_t) S_{t-1} + |k_t|^2 (w_t . v_t).

    With |k_t| = 1 and b_t = 1 this is k_t^T S_t = w_t . v_t: the erase acts
    along the key axis and the write gate along the value axis (d_k != d_v here).
    """
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 1, 12, 2, 9, 4
    q, k, v, la, b, w, S0 = rand_inputs(rng, B, T, H, dk, dv)
    _, S_prev = oracle_mod.forward(*(x[:, :T - 1] for x in (q, k, v, la, b, w)), S0=S0)
    _, S_t = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    for hi in range(H):
        kt, bt, lat, vt, wt = (head(x, 0, hi)[T - 1] for x in (k, b, la, v, w))
        kk = kt @ kt
        lhs = kt @ S_t[hi]
        rhs = (kt - kk * bt * kt) @ (np.exp(lat)[:, None] * S_prev[hi]) + kk * wt * vt
        assert rel_err(lhs, rhs) < 1e-12
    # b = 1 and unit k (renormalised in fp64): k^T S_t = w . v exactly
    b1 = np.ones_like(b)
    _, S_prev = oracle_mod.forward(*(x[:, :T - 1] for x in (q, k, v, la, b1, w)), S0=S0)
    _, S_t = oracle_mod.forward(q, k, v, la, b1, w, S0=S0)
    for hi in range(H):
        kt = head(k, 0, hi)[T - 1]
        wv = head(w, 0, hi)[T - 1] * head(v, 0, hi)[T - 1]
        kk = kt @ kt
        lhs = kt @ S_t[hi]
        rhs = (1 - kk) * kt @ (np.exp(head(la, 0, hi)[T - 1])[:, None] * S_prev[hi]) + kk * wv
        assert rel_err(lhs, rhs) < 1e-12
        assert abs(kk - 1) < 1e-6 and rel_err(lhs, wv) < 1e-5


def test_state_split(oracle_mod):
    rng = np.random.default_rng(12)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 2, 70, 2, 6, 5, b_scale=2.0)
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    T1 = 29
    o1, S1 = oracle_mod.forward(*(x[:, :T1] for x in (q, k, v, la, b, w)), S0=S0)
    o2, S2 = oracle_mod.forward(*(x[:, T1:] for x in (q, k, v, la, b, w)),
                                S0=S1.reshape(2, 2, 6, 5))
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S2, ST, rtol=1e-12, atol=1e-12)


def test_linearity_in_state_and_value(oracle_mod):
    rng = np.random.default_rng(13)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 1, 30, 2, 5, 6)
    _, _, v2, _, _, _, S02 = rand_inputs(rng, 1, 30, 2, 5, 6)
    a, c = 2.0, -0.5            # powers of two: the fp32 inputs stay exact
    oA, SA = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    oB, SB = oracle_mod.forward(q, k, v2, la, b, w, S0=S02)
    vc = (a * v.astype(np.float64) + c * v2.astype(np.float64))
    oC, SC = oracle_mod.forward(q, k, vc.astype(np.float32), la, b, w, S0=a * S0 + c * S02)
    tol = 1e-6   # the combined v is rounded to fp32 once
    assert rel_err(oC, a * oA + c * oB) < tol
    assert rel_err(SC, a * SA + c * SB) < tol
    oD, SD = oracle_mod.forward(q, k, (a * v).astype(np.float32), la, b, w, S0=a * S0)
    assert rel_err(oD, a * oA) < 1e-14 and rel_err(SD, a * SA) < 1e-14


def test_write_gate_value_symmetry(oracle_mod):
    rng = np.random.default_rng(14)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 2, 20, 2, 4, 7)
    o1, S1 = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    o2, S2 = oracle_mod.forward(q, k, w, la, b, v, S0=S0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


def test_decode_steps_matches_forward(oracle_mod):
    rng = np.random.default_rng(15)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 3, 6, 2, 4, 4)
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    sw = lambda x: np.swapaxes(x, 0, 1)
    od, Sd = oracle_mod.decode_steps(*(sw(x) for x in (q, k, v, la, b, w)), S0=S0)
    np.testing.assert_array_equal(o, od)
    np.testing.assert_array_equal(ST, Sd)


def test_state_growth_is_reported(oracle_mod):
    rng = np.random.default_rng(16)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 1, 40, 1, 4, 3, b_scale=2.0)
    o, ST, smax = oracle_mod.forward(q, k, v, la, b, w, S0=S0, want_smax=True)
    assert smax[0] >= np.max(np.abs(ST[0])) > 0


def test_rejects_bad_arguments(oracle_mod):
    rng = np.random.default_rng(17)
    q, k, v, la, b, w, S0 = rand_inputs(rng, 1, 4, 2, 3, 3)
    with pytest.raises(ValueError):
        oracle_mod.forward(q, k, v, la, b, w, S0=S0, heads=[0, 5])
