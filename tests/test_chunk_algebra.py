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


def test_doubling_unit_lower_inverse():
    """The in-place inverse of the tensor-core kernel, step by step:
    16x16 diagonal blocks by right-looking substitution, then
    T_{2p+1,2p} = -D_{2p+1} A_{2p+1,2p} D_{2p}, then T_ba = -T_b A_ba T_a."""
    rng = np.random.default_rng(3)
    A = np.tril(rng.standard_normal((64, 64)) * 0.3, -1)
    M = A.copy()
    for blk in range(4):
        R = 16 * blk
        X = np.zeros((16, 16))
        for j in range(16):
            s = np.eye(16)[:, j].copy()
            x = np.zeros(16)
            for i in range(16):
                x[i] = s[i]
                s[i + 1:] -= A[R + i + 1:R + 16, R + i] * x[i]
            X[:, j] = x
        M[R:R + 16, R:R + 16] = X
    for p in range(2):
        R = 32 * p
        Y = M[R + 16:R + 32, R:R + 16] @ M[R:R + 16, R:R + 16]
        M[R + 16:R + 32, R:R + 16] = -M[R + 16:R + 32, R + 16:R + 32] @ Y
    Y = M[32:, :32] @ M[:32, :32]
    M[32:, :32] = -M[32:, 32:] @ Y
    np.testing.assert_allclose(M, np.linalg.inv(np.eye(64) + A), rtol=1e-10, atol=1e-10)
