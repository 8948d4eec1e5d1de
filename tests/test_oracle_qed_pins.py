"""Pins for the oracle's second, query-derived erase direction (``forward_qed``).

The "Query Knows What to Forget" page (mlsanity 2608.13668, abstract) adds to
GDN-2 an erase direction taken from the query and orthogonal to the key, which
cancels what the old state holds along the query; a key-directed edit cannot
reach the key-orthogonal part of a read.  The page prints no formula; the
oracle's reading is

    u_t = r_t / sqrt(r_t . r_t + eps),  r_t = q_t - (q_t.k_t / k_t.k_t) k_t
    S_t = (I - k_t (b_t . k_t)^T - u_t (c_t . u_t)^T) diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T

These tests pin that reading by an explicit d_k x d_k matrix brute force, by the
property the abstract states (with a full second erase and nothing else, a
read along q_t sees only the key-directed part: o_t = (q_t.k_t / k_t.k_t) k_t^T S_{t-1},
and k^T S is untouched), and by the cases that reduce to GDN-2 (c = 0; q
parallel to k, where no second direction exists).
"""
import numpy as np
import pytest

from test_oracle_pins import rand_inputs, rel_err


def qed_direction(q, k, eps):
    """u = r / sqrt(r.r + eps) with r the part of q orthogonal to k."""
    kk = float(k @ k)
    r = q - (float(q @ k) / kk) * k if kk > 0 else q.copy()
    n = np.sqrt(float(r @ r) + eps)
    return r / n if n > 0 else np.zeros_like(r)


def brute_force_qed_head(q, k, v, la, b, c, w, S0, eps):
    """Explicit matrices: S <- (I - k (b.k)^T - u (c.u)^T) diag(alpha) S + k (w.v)^T."""
    T, dk = q.shape
    S = np.zeros((dk, v.shape[1])) if S0 is None else S0.copy()
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        u = qed_direction(q[t], k[t], eps)
        erase = np.eye(dk) - np.outer(k[t], b[t] * k[t]) - np.outer(u, c[t] * u)
        S = erase @ np.diag(np.exp(la[t])) @ S + np.outer(k[t], w[t] * v[t])
        o[t] = S.T @ q[t]
    return o, S


def _qed_inputs(rng, B, T, H, dk, dv):
    q, k, v, la, b, w, S0 = rand_inputs(rng, B, T, H, dk, dv)
    c = (1 / (1 + np.exp(-rng.standard_normal((B, T, H, dk))))).astype(np.float32)
    return q, k, v, la, b, c, w, S0


def f64(x):
    return np.asarray(x, dtype=np.float64)


@pytest.mark.parametrize("B,T,H,dk,dv,eps", [(1, 9, 1, 3, 2, 0.0), (2, 21, 2, 6, 5, 1e-6),
                                             (1, 40, 3, 16, 8, 1e-3)])
def test_qed_brute_force_matrix_form(oracle_mod, B, T, H, dk, dv, eps):
    rng = np.random.default_rng(200 + T)
    q, k, v, la, b, c, w, S0 = _qed_inputs(rng, B, T, H, dk, dv)
    o, ST = oracle_mod.forward_qed(q, k, v, la, b, c, w, S0=S0, qed_eps=eps)
    for bi in range(B):
        for hi in range(H):
            hd = lambda x: f64(x)[bi, :, hi, :]
            ob, Sb = brute_force_qed_head(hd(q), hd(k), hd(v), hd(la), hd(b), hd(c), hd(w), S0[bi, hi], eps)
            assert rel_err(o[bi * H + hi], ob) < 1e-12
            assert rel_err(ST[bi * H + hi], Sb) < 1e-12


def test_qed_full_erase_read_sees_only_the_key_part(oracle_mod):
    """b = 0, w = 0, alpha = 1, c = 1, eps = 0: the step is the projection I - u u^T, so
    o_t = S_t^T q_t = (q_t . k_t / k_t . k_t) k_t^T S_{t-1} (the query-orthogonal part of the
    read is cancelled) and k_t^T S_t = k_t^T S_{t-1} (the key-directed part is untouched)."""
    rng = np.random.default_rng(210)
    B, T, H, dk, dv = 1, 12, 1, 7, 4
    q, k, v, _, _, _, _, S0 = _qed_inputs(rng, B, T, H, dk, dv)
    zeros_k = np.zeros((B, T, H, dk), np.float32)
    ones_k = np.ones((B, T, H, dk), np.float32)
    zeros_v = np.zeros((B, T, H, dv), np.float32)
    o, _ = oracle_mod.forward_qed(q, k, v, zeros_k, zeros_k, ones_k, zeros_v, S0=S0, qed_eps=0.0)
    for t in range(T):
        # the state before token t from the same oracle on the first t tokens (state split)
        if t == 0:
            Sprev = S0[0, 0]
        else:
            sl = lambda x: x[:, :t]
            _, Sp = oracle_mod.forward_qed(sl(q), sl(k), sl(v), sl(zeros_k), sl(zeros_k), sl(ones_k),
                                           sl(zeros_v), S0=S0, qed_eps=0.0)
            Sprev = Sp[0]
        qt, kt = f64(q)[0, t, 0], f64(k)[0, t, 0]
        expect = float(qt @ kt) / float(kt @ kt) * (kt @ Sprev)
        assert rel_err(o[0, t], expect) < 1e-11
        _, Snow = oracle_mod.forward_qed(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], zeros_k[:, :t + 1],
                                         zeros_k[:, :t + 1], ones_k[:, :t + 1], zeros_v[:, :t + 1],
                                         S0=S0, qed_eps=0.0)
        assert rel_err(kt @ Snow[0], kt @ Sprev) < 1e-11


def test_qed_zero_gate_is_gdn2(oracle_mod):
    rng = np.random.default_rng(220)
    q, k, v, la, b, c, w, S0 = _qed_inputs(rng, 2, 30, 2, 8, 6)
    o1, S1 = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    o2, S2 = oracle_mod.forward_qed(q, k, v, la, b, np.zeros_like(c), w, S0=S0)
    assert rel_err(o2, o1) < 1e-15 and rel_err(S2, S1) < 1e-15


def test_qed_query_parallel_to_key_is_gdn2(oracle_mod):
    """q = lambda k: no direction orthogonal to the key exists, so any c leaves GDN-2."""
    rng = np.random.default_rng(230)
    _, k, v, la, b, c, w, S0 = _qed_inputs(rng, 1, 25, 2, 6, 5)
    lam = rng.uniform(-2, 2, size=(1, 25, 2, 1)).astype(np.float32)
    q = (k * lam).astype(np.float32)
    o1, S1 = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    o2, S2 = oracle_mod.forward_qed(q, k, v, la, b, c, w, S0=S0, qed_eps=1e-6)
    # q, k pass through float32; r = q - (q.k/k.k) k is zero up to that rounding
    assert rel_err(o2, o1) < 1e-5 and rel_err(S2, S1) < 1e-5


def test_qed_prep_gates_c_with_the_logistic(oracle_mod):
    """Under the input prep c is a logit: prep=True with logit(c) equals prep on the other
    inputs and the gate c itself."""
    rng = np.random.default_rng(240)
    q, k, v, la, b, c, w, S0 = _qed_inputs(rng, 1, 16, 1, 5, 3)
    braw = np.log(b / (1 - b)).astype(np.float32)
    wraw = np.log(w / (1 - w)).astype(np.float32)
    craw = np.log(c / (1 - c)).astype(np.float32)
    o1, S1 = oracle_mod.forward_qed(q, k, v, la, braw, craw, wraw, S0=S0, prep=True, l2_eps=0.0)
    qn = q / np.linalg.norm(f64(q), axis=-1, keepdims=True)
    kn = k / np.linalg.norm(f64(k), axis=-1, keepdims=True)
    o2, S2 = oracle_mod.forward_qed(qn, kn, v, la, b, c, w, S0=S0)
    assert rel_err(o1, o2) < 1e-5 and rel_err(S1, S2) < 1e-5


def test_qed_decode_steps_match_forward(oracle_mod):
    rng = np.random.default_rng(250)
    q, k, v, la, b, c, w, S0 = _qed_inputs(rng, 2, 7, 2, 4, 3)
    o1, S1 = oracle_mod.forward_qed(q, k, v, la, b, c, w, S0=S0)
    tb = lambda x: np.swapaxes(x, 0, 1)
    o2, S2 = oracle_mod.decode_steps_qed(tb(q), tb(k), tb(v), tb(la), tb(b), tb(c), tb(w), S0)
    assert rel_err(o1, o2) < 1e-14 and rel_err(S1, S2) < 1e-14
