"""CPU-side checks of the C ABI: the library builds, loads and exports every
symbol include/gdn2.h declares; status strings; host-side argument checks
that return before any CUDA call."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_92_b200 as g
from gated_delta_rule_92_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return g._open(g.LIB_PATH)   # the release library, whatever GDN2_DEBUG_BOUNDS selects


def declared_functions():
    with open(os.path.join(ROOT, "include", "gdn2.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn2_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    assert names == sorted(g.EXPORTED)


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {g.LIB_PATH}").read()
    exported = set(re.findall(r" T (gdn2_[a-z0-9_]+)", out))
    assert set(declared_functions()) <= exported


def test_status_strings(L):
    for code, name in g.STATUS_NAMES.items():
        assert g.status_string(code) == name
    assert g.status_string(99) == "GDN2_ERR_UNKNOWN"
    assert L.gdn2_version() >= 100


def _chunk_call(L, ptr=16, B=1, T=64, H=1, dk=64, dv=64, chunk=64, io=1, o=16, s0=None, st=None):
    P = ctypes.c_void_p
    p = P(ptr) if ptr is not None else None
    return L.gdn2_chunk_fwd(p, p, p, p, p, p, P(s0) if s0 else None, P(o) if o else None,
                            P(st) if st else None, B, T, H, dk, dv, chunk, io, None)


def test_chunk_argument_validation_on_host(L):
    # these return before touching the device
    assert _chunk_call(L, ptr=None) == 1                 # null input
    assert _chunk_call(L, ptr=None, T=0, o=None) == 0    # empty sequence, no state: no-op
    assert _chunk_call(L, B=0) == 1
    assert _chunk_call(L, T=-1) == 1
    assert _chunk_call(L, io=7) == 1
    assert _chunk_call(L, ptr=24) == 3                   # misaligned
    assert _chunk_call(L, o=40) == 3
    assert _chunk_call(L, chunk=48) == 2                 # chunk 16, 32 and 64 are built
    assert _chunk_call(L, chunk=128) == 2
    assert _chunk_call(L, dk=96) == 2
    assert _chunk_call(L, dv=96) == 2
    assert _chunk_call(L, dv=1024) == 2
    assert _chunk_call(L, B=70000) == 2


def test_decode_argument_validation_on_host(L):
    P = ctypes.c_void_p
    p = P(16)
    assert L.gdn2_decode_step(p, p, p, p, p, p, None, p, 1, 1, 64, 64, 1, None) == 1
    assert L.gdn2_decode_step(p, p, p, p, p, p, p, p, 0, 1, 64, 64, 1, None) == 1
    assert L.gdn2_decode_step(p, p, p, p, p, p, P(8), p, 1, 1, 64, 64, 1, None) == 3
    assert L.gdn2_decode_step(p, p, p, p, p, p, p, p, 1, 1, 32, 64, 1, None) == 2
    assert L.gdn2_decode_step(p, p, p, p, p, p, p, p, 1, 1, 64, 80, 1, None) == 2
    assert L.gdn2_selftest_wait_timeout(0, None) == 1


def test_product_path_does_not_touch_oracle():
    """The binding and the CUDA sources never reference the oracle."""
    pkg = os.path.join(ROOT, "gated_delta_rule_92_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, fn)) as f:
                    assert "oracle" not in f.read().lower(), fn


def test_fused_argument_validation_on_host(L):
    """The _ex calls check their fusion arguments before touching the device."""
    P, F = ctypes.c_void_p, ctypes.c_float
    p, w = P(16), P(32)

    def chunk_ex(flags=0, l2=1e-6, gate=None, weight=None, eps=1e-5, T=64):
        return L.gdn2_chunk_fwd_ex(p, p, p, p, p, p, None, p, None, 1, T, 1, 1, 64, 64, 64, 1, None,
                                   flags, F(l2), gate, weight, F(eps), None)

    def decode_ex(flags=0, l2=1e-6, gate=None, weight=None, eps=1e-5):
        return L.gdn2_decode_step_ex(p, p, p, p, p, p, p, p, 1, 1, 1, 64, 64, 1,
                                     flags, F(l2), gate, weight, F(eps), None)

    for call in (chunk_ex, decode_ex):
        assert call(flags=8) == 1                     # unknown flag
        assert call(flags=2) == 1                     # negative eigenvalues without the prep
        assert call(flags=1, l2=-1.0) == 1            # negative L2 epsilon
        assert call(gate=p) == 1                      # gate without norm_weight
        assert call(gate=p, weight=w, eps=-1.0) == 1  # negative norm epsilon
        assert call(gate=P(18), weight=w) == 3        # misaligned gate
        assert call(gate=p, weight=P(20)) == 3        # misaligned weight
    assert chunk_ex(flags=3, T=0, gate=p, weight=w) == 0   # empty sequence: nothing to do
    assert chunk_ex(weight=w) == 1                         # weight without gate


def test_value_heads_and_packing_validation_on_host(L):
    """HV must be a multiple of H; cu_seqlens must be 4-byte aligned; HV = 0 means H."""
    P, F = ctypes.c_void_p, ctypes.c_float
    p = P(16)

    def chunk_ex(H=2, HV=4, cu=None, T=64, B=1):
        return L.gdn2_chunk_fwd_ex(p, p, p, p, p, p, None, p, None, B, T, H, HV, 64, 64, 64, 1, cu,
                                   0, F(1e-6), None, None, F(1e-5), None)

    def decode_ex(H=2, HV=4, B=1):
        return L.gdn2_decode_step_ex(p, p, p, p, p, p, p, p, B, H, HV, 64, 64, 1,
                                     0, F(1e-6), None, None, F(1e-5), None)

    assert chunk_ex(HV=3) == 1            # not a multiple of H
    assert chunk_ex(HV=-2) == 1
    assert decode_ex(HV=3) == 1
    assert decode_ex(HV=-1) == 1
    assert chunk_ex(cu=P(18)) == 3        # misaligned offsets
    assert chunk_ex(T=0, cu=P(16)) == 0   # no tokens at all, no state: nothing to do
    assert chunk_ex(T=0, HV=0) == 0
    assert chunk_ex(HV=70000, H=1) == 2   # beyond the grid's y extent


def test_qed_argument_validation_on_host(L):
    """The second-erase entry points check their arguments before touching the device."""
    P, F = ctypes.c_void_p, ctypes.c_float
    p = P(16)

    def chunk_qed(c=p, eps=1e-6, T=64, dk=64, dv=64, ptr=p):
        return L.gdn2_chunk_fwd_qed(ptr, p, p, p, p, c, p, None, p, None, 1, T, 1, dk, dv, 1, F(eps), None)

    def decode_qed(c=p, eps=1e-6, dk=64, dv=64):
        return L.gdn2_decode_step_qed(p, p, p, p, p, c, p, p, p, 1, 1, dk, dv, 1, F(eps), None)

    for call in (chunk_qed, decode_qed):
        assert call(c=None) == 1            # no second gate
        assert call(eps=-1.0) == 1          # negative epsilon
        assert call(c=P(20)) == 3           # misaligned gate
        assert call(dk=96) == 2
        assert call(dv=96) == 2
    assert chunk_qed(T=0, ptr=None, c=None) == 0   # empty sequence, no state: nothing to do


def test_host_entry_workspace_and_validation_on_host(L):
    """The host-buffer entry: workspace sizing (pure host arithmetic) and the
    argument errors it returns before any copy or launch."""
    n = ctypes.c_size_t(0)
    # headline shape: one sequence per slice, two slice buffers of
    # 4 key tensors + v, w, o (16 MiB each) + S0, S_T (1 MiB each)
    assert L.gdn2_chunk_fwd_host_workspace(8, 4096, 16, 128, 128, 1, ctypes.byref(n)) == 0
    assert n.value == 2 * (7 * 16 * 2 ** 20 + 2 * 2 ** 20)
    assert L.gdn2_chunk_fwd_host_workspace(1, 100, 2, 64, 64, 0, ctypes.byref(n)) == 0
    one = 7 * (100 * 2 * 64 * 4) + 2 * (2 * 64 * 64 * 4)
    assert n.value == one                                  # one slice: one buffer
    assert L.gdn2_chunk_fwd_host_workspace(0, 64, 1, 64, 64, 1, ctypes.byref(n)) == 1
    assert L.gdn2_chunk_fwd_host_workspace(1, 64, 1, 64, 64, 7, ctypes.byref(n)) == 1
    assert L.gdn2_chunk_fwd_host_workspace(1, 64, 1, 64, 64, 1, None) == 1
    P = ctypes.c_void_p
    p = P(16)

    def call(ws, ws_bytes, B=1, T=64, dk=64):
        return L.gdn2_chunk_fwd_host(p, p, p, p, p, p, None, p, None, B, T, 1, dk, 64, 64, 1,
                                     P(ws) if ws else None, ctypes.c_size_t(ws_bytes), None)
    assert call(None, 0) == 1                              # no workspace
    assert call(4096, 16) == 1                             # too small
    assert call(16, 1 << 30) == 3                          # not 256-byte aligned
    assert call(256, 1 << 30, dk=96) == 2                  # unsupported shape, as gdn2_chunk_fwd
    assert call(256, 1 << 30, B=0) == 1


def test_host_binding_rejects_bad_tensors_before_any_copy():
    """chunk_fwd_host checks its CPU tensors in Python before it touches a device."""
    import pytest
    import torch
    B, T, H, dk, dv = 1, 8, 1, 64, 64
    q = torch.zeros(B, T, H, dk, dtype=torch.bfloat16)
    v = torch.zeros(B, T, H, dv, dtype=torch.bfloat16)
    with pytest.raises(ValueError):   # v with the wrong width
        g.chunk_fwd_host(q, q, v[..., :32], q, q, v)
    q_strided = torch.zeros(B, T, H, 2 * dk, dtype=torch.bfloat16)[..., ::2]
    assert q_strided.shape == q.shape and not q_strided.is_contiguous()
    with pytest.raises(ValueError):   # non-contiguous input
        g.chunk_fwd_host(q_strided, q, v, q, q, v)
    with pytest.raises(ValueError):   # state of the wrong shape
        g.chunk_fwd_host(q, q, v, q, q, v, torch.zeros(B, H, dk, dv + 1))
    with pytest.raises(ValueError):   # mixed dtypes
        g.chunk_fwd_host(q, q.float(), v, q, q, v)


@pytest.fixture(scope="module")
def LD():
    gbuild.build()
    return g._open(g.DEBUG_LIB_PATH)


def test_debug_build_exports_every_declared_symbol(LD):
    for name in declared_functions():
        assert hasattr(LD, name), name
    out = os.popen(f"nm -D --defined-only {g.DEBUG_LIB_PATH}").read()
    exported = set(re.findall(r" T (gdn2_[a-z0-9_]+)", out))
    assert set(declared_functions()) <= exported


def test_debug_bounds_entry_points_on_host(L, LD):
    P, I = ctypes.c_void_p, ctypes.c_int
    a, b = I(7), I(7)
    # the release library has no range checks: both calls say so before any CUDA call
    assert L.gdn2_debug_bounds_site(ctypes.byref(a), ctypes.byref(b), None) == 2
    assert (a.value, b.value) == (-1, 0)
    assert L.gdn2_selftest_bounds(None) == 2
    # null outputs are argument errors in either build
    assert L.gdn2_debug_bounds_site(None, ctypes.byref(b), None) == 1
    assert LD.gdn2_debug_bounds_site(ctypes.byref(a), None, None) == 1
    assert LD.gdn2_status_string(6) == b"GDN2_ERR_OUT_OF_BOUNDS"
    # the debug build validates arguments on the host exactly as the release one
    for kw in ({"ptr": None}, {"B": 0}, {"ptr": 24}, {"chunk": 48}, {"dk": 96}):
        assert _chunk_call(LD, **kw) == _chunk_call(L, **kw)


@pytest.mark.skipif(os.environ.get("GDN2_DEBUG_BOUNDS") == "1", reason="the debug build is already selected")
def test_debug_bounds_context_switches_library():
    release = g.lib()
    with g.debug_bounds() as LD:
        assert g.lib() is LD and LD is not release
        assert LD._name.endswith("libgdn2_debug.so")
    assert g.lib() is release


def test_testing_fail_launches_arguments(L):
    assert L.gdn2_testing_fail_launches(-1, 1) == 1
    assert L.gdn2_testing_fail_launches(0, -1) == 1
    assert L.gdn2_testing_fail_launches(3, 2) == 0
    assert L.gdn2_testing_fail_launches(0, 0) == 0   # disarmed again
