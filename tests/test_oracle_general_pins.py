"""Pins for the oracle's packed variable-length sequences and value heads
(burn-gdn2 README, "Configuration": num_v_heads; the chunked mode's batches of
sequences).  Each is checked against the explicit d_k x d_k transition-matrix
brute force of ``test_oracle_pins`` applied to the head's own token slice,
and planted mistakes in the head and sequence indexing are caught.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from test_oracle_pins import brute_force_head, rel_err


def _inputs(rng, T, H, HV, dk, dv, n_seq=None):
    q = rng.standard_normal((1, T, H, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((1, T, H, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    la = np.log(rng.uniform(0.8, 0.999, (1, T, H, dk)))
    b = rng.uniform(0.0, 2.0, (1, T, H, dk))
    v = rng.standard_normal((1, T, HV, dv))
    w = rng.uniform(0.0, 1.0, (1, T, HV, dv))
    S0 = rng.standard_normal((n_seq or 1, HV, dk, dv)) * 0.3
    return [x.astype(np.float32) for x in (q, k, v, la, b, w)] + [S0]


def _brute(q, k, v, la, b, w, S0, t0, t1, hk, hv):
    sl = lambda x, h: x[0, t0:t1, h].astype(np.float64)
    return brute_force_head(sl(q, hk), sl(k, hk), sl(v, hv), sl(la, hk), sl(b, hk), sl(w, hv), S0)


@pytest.mark.parametrize("HV", [2, 6])
def test_packed_sequences_and_value_heads_brute_force(oracle_mod, HV):
    rng = np.random.default_rng(41 + HV)
    H, dk, dv = 2, 5, 3
    lens = [7, 0, 1, 13, 4]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v, la, b, w, S0 = _inputs(rng, T, H, HV, dk, dv, n_seq=len(lens))
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0, cu_seqlens=cu)
    G = HV // H
    for n in range(len(lens)):
        for hv in range(HV):
            i = n * HV + hv
            ob, Sb = _brute(q, k, v, la, b, w, S0[n, hv], cu[n], cu[n + 1], hv // G, hv)
            assert o[i].shape == (lens[n], dv)
            assert rel_err(ST[i], Sb) < 1e-12
            if lens[n]:
                assert rel_err(o[i], ob) < 1e-12


def test_value_heads_without_packing(oracle_mod):
    """B sequences of equal length with HV = 2H equal the brute force per value head."""
    rng = np.random.default_rng(43)
    B, T, H, HV, dk, dv = 2, 9, 2, 4, 4, 3
    parts = [_inputs(rng, T, H, HV, dk, dv) for _ in range(B)]
    q, k, v, la, b, w = (np.concatenate([p[j] for p in parts]) for j in range(6))
    S0 = np.concatenate([p[6] for p in parts])
    o, ST = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    for bi in range(B):
        for hv in range(HV):
            ob, Sb = brute_force_head(*(x[bi, :, h].astype(np.float64) for x, h in
                                        ((q, hv // 2), (k, hv // 2), (v, hv), (la, hv // 2), (b, hv // 2), (w, hv))),
                                      S0[bi, hv])
            assert rel_err(o[bi * HV + hv], ob) < 1e-12 and rel_err(ST[bi * HV + hv], Sb) < 1e-12


def test_packed_equals_equal_length_batches(oracle_mod):
    """Packing B equal-length sequences reproduces the [B, T] layout exactly."""
    rng = np.random.default_rng(44)
    B, T, H, dk, dv = 3, 11, 2, 4, 4
    parts = [_inputs(rng, T, H, H, dk, dv) for _ in range(B)]
    q, k, v, la, b, w = (np.concatenate([p[j] for p in parts]) for j in range(6))
    S0 = np.concatenate([p[6] for p in parts])
    o1, S1 = oracle_mod.forward(q, k, v, la, b, w, S0=S0)
    pk = lambda x: x.reshape(1, B * T, *x.shape[2:])
    o2, S2 = oracle_mod.forward(pk(q), pk(k), pk(v), pk(la), pk(b), pk(w), S0=S0,
                                cu_seqlens=np.arange(B + 1) * T)
    assert np.array_equal(np.stack(o2), o1) and np.array_equal(S2, S1)


def test_bad_packing_is_rejected(oracle_mod):
    rng = np.random.default_rng(45)
    q, k, v, la, b, w, S0 = _inputs(rng, 10, 1, 1, 2, 2, n_seq=2)
    for cu in ([0, 4, 9], [1, 4, 10], [0, 6, 4, 10][:3]):
        with pytest.raises(ValueError):
            oracle_mod.forward(q, k, v, la, b, w, S0=S0[: len(cu) - 1], cu_seqlens=cu)
    with pytest.raises(AssertionError):   # HV not a multiple of H
        oracle_mod.forward(np.zeros((1, 4, 2, 2)), np.zeros((1, 4, 2, 2)), np.zeros((1, 4, 3, 2)),
                           np.zeros((1, 4, 2, 2)), np.zeros((1, 4, 2, 2)), np.zeros((1, 4, 3, 2)))


MUTANTS = {
    "key_head_modulo": ("const long bi = bh / HV, hv = bh % HV, hk = hv / G;",
                        "const long bi = bh / HV, hv = bh % HV, hk = hv % H;"),
    "sequence_start_off_by_one": ("const long t0 = cu ? (long)cu[bi] : bi * (long)T;",
                                  "const long t0 = cu ? (long)cu[bi] + (bi > 0) : bi * (long)T;"),
    "value_stride_uses_key_heads": ("const long sk = H * dk, sv = HV * dv;", "const long sk = H * dk, sv = H * dv;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_indexing_mutant_is_caught(tmp_path, name):
    with open(os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")) as f:
        src = f.read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    c, so = tmp_path / "m.c", tmp_path / "m.so"
    c.write_text(src.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    lib = oracle.open_library(str(so))

    class _M:
        @staticmethod
        def forward(*a, **kw):
            return oracle.forward(*a, lib=lib, **kw)
    with pytest.raises(AssertionError):
        test_packed_sequences_and_value_heads_brute_force(_M, 6)
