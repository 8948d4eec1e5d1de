"""The chunk (WY) regrouping used by both GPU kernels, written in fp64 numpy,
must reproduce the token recurrence (the oracle) to rounding.

This checks the algebra, not a kernel: per chunk of C tokens with
chunk-start state S,
    g = cumsum(log_alpha), gamma = exp(g)
    Q~ = Q.gamma, K~ = K/gamma, E = B.K.gamma
    A = strict_lower(E K~^T), P = lower(Q~ K~^T), T = (I + A)^{-1}
    U = T (W.V) - (T E) S
    O = Q~ S + P U
    S' = diag(gamma_C) (S + K~^T U)
"""
import numpy as np
import pytest

from test_oracle_pins import head, rand_inputs, rel_err


def chunk_model_head(q, k, v, la, b, w, S0, C):
    T, dk = q.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for t0 in range(0, T, C):
        sl = slice(t0, t0 + C)
        g = np.cumsum(la[sl], axis=0)
        gam = np.exp(g)
        Qt, Kt, E = q[sl] * gam, k[sl] / gam, b[sl] * k[sl] * gam
        A = np.tril(E @ Kt.T, -1)
        P = np.tril(Qt @ Kt.T)
        Tm = np.linalg.inv(np.eye(len(g)) + A)
        U = Tm @ (w[sl] * v[sl]) - (Tm @ E) @ S
        o[sl] = Qt @ S + P @ U
        S = gam[-1][:, None] * (S + Kt.T @ U)
    return o, S


@pytest.mark.parametrize("C", [4, 16, 64])
@pytest.mark.parametrize("bs", [1.0, 2.0])
def test_chunk_form_matches_recurrence(oracle_mod, C, bs):
    rng = np.random.default_rng(21 + C)
    B, T, H, dk, dv = 1, 128, 2, 8, 6
    q, k, v, la, b, w, S0 = rand_inputs(rng, B, T, H, dk, dv, b_scale=bs)
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    for hi in range(H):
        om, Sm = chunk_model_head(*(head(x, 0, hi) for x in (q, k, v, la, b, w)), S0[0, hi], C)
        assert rel_err(om, o[hi]) < 1e-10
        assert rel_err(Sm, ST[hi]) < 1e-10


def test_blocked_unit_lower_inverse():
    """The 16x16-blocked forward substitution of the tensor-core kernel:
    diagonal blocks by substitution, then T_ib = -D_ib sum_k A_ib,k T_k."""
    rng = np.random.default_rng(3)
    A = np.tril(rng.standard_normal((64, 64)) * 0.3, -1)
    Tb = A.copy()
    for blk in range(4):
        R = 16 * blk
        D = np.linalg.inv(np.eye(16) + A[R:R + 16, R:R + 16])
        Tb[R:R + 16, R:R + 16] = D
    for ib in range(1, 4):
        n = 16 * ib
        Wm = A[n:n + 16, :n] @ Tb[:n, :n]
        Tb[n:n + 16, :n] = -Tb[n:n + 16, n:n + 16] @ Wm
    np.testing.assert_allclose(Tb, np.linalg.inv(np.eye(64) + A), rtol=1e-10, atol=1e-10)
