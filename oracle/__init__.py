"""fp64 CPU oracle for the Gated DeltaNet-2 recurrence (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``gated_delta_rule_92_b200`` and its binding) never imports it, and this
package never imports the product path.

The arithmetic lives in ``gdn2_oracle.c``: the per-token recurrence of the
burn-gdn2 README, section "Architecture",
``S_t = (I - k_t (b_t . k_t)^T) diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T``,
``o_t = S_t^T q_t``, evaluated in double precision.  This module only
compiles it (gcc, OpenMP) and marshals numpy arrays into it.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
an explicit d_k x d_k matrix brute force, the linear-attention and
gated-linear-attention closed forms, separately written KDA and Gated DeltaNet
recurrences, a hand-derived worked example, and invariants (delta-write,
state split, linearity, w/v symmetry).  The optional input prep and output
epilogue are pinned in ``tests/test_oracle_fused_pins.py`` (hand-worked
values, closed forms of sigmoid and SiLU, scale and sign invariances).  The
second, query-derived erase (``forward_qed``) is pinned in
``tests/test_oracle_qed_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn2_oracle.c`` into ``liboracle.so`` next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def open_library(path: str):
    """Open a compiled oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.gdn2_oracle_forward.argtypes = [P, P, P, P, P, P, P, P, P, P,
                                        I, I, I, I, I, P, I, I]
    lib.gdn2_oracle_forward.restype = I
    D = ctypes.c_double
    lib.gdn2_oracle_forward_ex.argtypes = [P, P, P, P, P, P, P, P, P, P,
                                           I, I, I, I, I, I, P, P, I, I,
                                           I, D, P, P, D]
    lib.gdn2_oracle_forward_ex.restype = I
    lib.gdn2_oracle_forward_qed.argtypes = [P, P, P, P, P, P, P, P, P, P, P,
                                            I, I, I, I, I, P, I, I, I, D, D]
    lib.gdn2_oracle_forward_qed.restype = I
    lib.gdn2_oracle_max_threads.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = open_library(_LIB)
    return _lib


def max_threads() -> int:
    return int(_load().gdn2_oracle_max_threads())


def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):            # a torch tensor (bf16 has no numpy dtype)
        x = x.detach().float().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(q, k, v, log_alpha, b, w, S0=None, heads=None, n_threads: int = 0,
            want_state: bool = True, want_smax: bool = False, lib=None, *,
            prep: bool = False, allow_neg_eigval: bool = False, l2_eps: float = 1e-6,
            gate=None, norm_weight=None, norm_eps: float = 1e-5, cu_seqlens=None):
    """Run the recurrence in fp64.

    q, k, log_alpha, b : [B, T, H, d_k];  v, w : [B, T, H, d_v] (any float
    dtype; values are taken as float32, which holds bf16 values exactly).
    S0 : [B, H, d_k, d_v] or None (zeros).  heads : iterable of flat b*H+h
    indices, or None for all.  Returns (o, S_T[, smax]) with
    o : [n_heads, T, d_v] and S_T : [n_heads, d_k, d_v] (float64), heads in
    the order requested.

    prep=True takes q, k, b, w as raw: q and k are L2-normalised over d_k
    (x / sqrt(sum x^2 + l2_eps)), b = sigmoid(b) (2 sigmoid(b) with
    allow_neg_eigval) and w = sigmoid(w), all in double (burn-gdn2 README,
    "Architecture" L2-Norm; "Configuration" allow_neg_eigval).  gate
    [B, T, H, d_v] with norm_weight [d_v] returns the gated RMS norm
    o / sqrt(mean(o^2) + norm_eps) * norm_weight * silu(gate) per (token, head)
    instead of o (README "Architecture": Gated RMS Norm <- SiLU Gate).

    Value heads: v, w (and gate) may have HV = G H heads (README
    "Configuration", num_v_heads); value head hv then reads key head hv // G,
    and heads / S0 / S_T index the B * HV value heads.  cu_seqlens ([N + 1],
    cu[0] = 0, non-decreasing, cu[N] = T): N sequences packed along the token
    axis of [1, T, H, d] inputs; o is then a list with one [len, d_v] array per
    requested head, S0 / S_T are [N, HV, d_k, d_v].
    """
    q, k, v, la, b, w = (_f32(x) for x in (q, k, v, log_alpha, b, w))
    Bt, T, H, dk = q.shape
    HV, dv = v.shape[-2], v.shape[-1]
    for x in (k, la, b):
        assert x.shape == (Bt, T, H, dk), x.shape
    for x in (v, w):
        assert x.shape == (Bt, T, HV, dv), x.shape
    assert HV % H == 0, (H, HV)
    cu = None
    if cu_seqlens is not None:
        assert Bt == 1, "packed sequences take [1, T, H, d] inputs"
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        B = int(cu.size) - 1
    else:
        B = Bt
    s0 = None
    if S0 is not None:
        if hasattr(S0, "detach"):
            S0 = S0.detach().double().cpu().numpy()
        s0 = np.ascontiguousarray(np.asarray(S0, dtype=np.float64))
        assert s0.shape == (B, HV, dk, dv), s0.shape
    if heads is None:
        hl = None
        nh = B * HV
    else:
        hl = np.ascontiguousarray(np.asarray(list(heads), dtype=np.int32))
        nh = int(hl.size)
    hidx = range(B * HV) if hl is None else [int(x) for x in hl]
    lens = [(int(cu[x // HV + 1] - cu[x // HV]) if 0 <= x < B * HV else 0) if cu is not None else T
            for x in hidx]
    o = np.empty((max(1, sum(lens)), dv), dtype=np.float64)
    st = np.empty((nh, dk, dv), dtype=np.float64) if want_state else None
    sm = np.empty((nh,), dtype=np.float64) if want_smax else None
    g = None
    wt = None
    if gate is not None:
        g = _f32(gate)
        assert g.shape == (Bt, T, HV, dv), g.shape
        assert norm_weight is not None, "the epilogue needs norm_weight"
        if hasattr(norm_weight, "detach"):
            norm_weight = norm_weight.detach().double().cpu().numpy()
        wt = np.ascontiguousarray(np.asarray(norm_weight, dtype=np.float64))
        assert wt.shape == (dv,), wt.shape
    pflag = (1 | (2 if allow_neg_eigval else 0)) if prep else 0
    rc = (lib or _load()).gdn2_oracle_forward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(w),
                                        _ptr(s0), _ptr(o), _ptr(st), _ptr(sm),
                                        B, T, H, HV, dk, dv, _ptr(cu), _ptr(hl), nh, int(n_threads),
                                        pflag, float(l2_eps), _ptr(g), _ptr(wt), float(norm_eps))
    if rc != 0:
        raise ValueError("gdn2 oracle rejected its arguments")
    if cu is not None:
        offs = np.cumsum([0] + lens)
        o = [o[offs[i]:offs[i + 1]] for i in range(nh)]
    else:
        o = o[:nh * T].reshape(nh, T, dv)
    if want_smax:
        return o, st, sm
    return o, st


def decode_steps(q, k, v, log_alpha, b, w, S0, heads=None, n_threads: int = 0, *,
                 prep: bool = False, allow_neg_eigval: bool = False, l2_eps: float = 1e-6,
                 gate=None, norm_weight=None, norm_eps: float = 1e-5):
    """Token-by-token decode over a step axis.

    Inputs are [steps, B, H, d] (one token per step and sequence), S0 is
    [B, H, d_k, d_v].  Returns (o [n_heads, steps, d_v], S [n_heads, d_k, d_v]).
    Decode is the same recurrence run one token at a time, so this is the
    forward pass with the step axis taken as time (prep and epilogue as in
    ``forward``).
    """
    def tb(x):
        return np.ascontiguousarray(np.swapaxes(_f32(x), 0, 1))
    return forward(tb(q), tb(k), tb(v), tb(log_alpha), tb(b), tb(w), S0=S0,
                   heads=heads, n_threads=n_threads, prep=prep, allow_neg_eigval=allow_neg_eigval,
                   l2_eps=l2_eps, gate=None if gate is None else tb(gate), norm_weight=norm_weight,
                   norm_eps=norm_eps)


def forward_qed(q, k, v, log_alpha, b, c, w, S0=None, heads=None, n_threads: int = 0, *,
                prep: bool = False, allow_neg_eigval: bool = False, l2_eps: float = 1e-6,
                qed_eps: float = 1e-6, want_smax: bool = False, lib=None):
    """The recurrence with the second, query-derived erase direction.

    u_t = r_t / sqrt(r_t . r_t + qed_eps) with r_t = q_t - (q_t.k_t / k_t.k_t) k_t,
    S_t = (I - k_t (b_t . k_t)^T - u_t (c_t . u_t)^T) diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T,
    o_t = S_t^T q_t.  c : [B, T, H, d_k] is the second erase gate (a logit under
    prep).  Shapes, heads and returns as in ``forward`` (equal-length sequences,
    value heads = key heads).
    """
    q, k, v, la, b, c, w = (_f32(x) for x in (q, k, v, log_alpha, b, c, w))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for x in (k, la, b, c):
        assert x.shape == (B, T, H, dk), x.shape
    for x in (v, w):
        assert x.shape == (B, T, H, dv), x.shape
    s0 = None
    if S0 is not None:
        if hasattr(S0, "detach"):
            S0 = S0.detach().double().cpu().numpy()
        s0 = np.ascontiguousarray(np.asarray(S0, dtype=np.float64))
        assert s0.shape == (B, H, dk, dv), s0.shape
    hl = None if heads is None else np.ascontiguousarray(np.asarray(list(heads), dtype=np.int32))
    nh = B * H if hl is None else int(hl.size)
    o = np.empty((max(1, nh * T), dv), dtype=np.float64)
    st = np.empty((nh, dk, dv), dtype=np.float64)
    sm = np.empty((nh,), dtype=np.float64) if want_smax else None
    pflag = (1 | (2 if allow_neg_eigval else 0)) if prep else 0
    rc = (lib or _load()).gdn2_oracle_forward_qed(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(c),
                                                  _ptr(w), _ptr(s0), _ptr(o), _ptr(st), _ptr(sm),
                                                  B, T, H, dk, dv, _ptr(hl), nh, int(n_threads),
                                                  pflag, float(l2_eps), float(qed_eps))
    if rc != 0:
        raise ValueError("gdn2 oracle rejected its arguments")
    o = o[:nh * T].reshape(nh, T, dv)
    return (o, st, sm) if want_smax else (o, st)


def decode_steps_qed(q, k, v, log_alpha, b, c, w, S0, heads=None, n_threads: int = 0, **kw):
    """``forward_qed`` over a step axis: inputs [steps, B, H, d], S0 [B, H, d_k, d_v]."""
    def tb(x):
        return np.ascontiguousarray(np.swapaxes(_f32(x), 0, 1))
    return forward_qed(tb(q), tb(k), tb(v), tb(log_alpha), tb(b), tb(c), tb(w), S0=S0, heads=heads,
                       n_threads=n_threads, **kw)
