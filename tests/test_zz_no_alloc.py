"""The no-alloc host entry (gdn2_chunk_fwd_host_noalloc) against the host
entry with a caller workspace (gdn2_chunk_fwd_host).

The no-alloc entry exists for callers that cannot allocate device memory
(for example a plug-in that only receives host buffers and a CUDA context it
does not own): the library stages the data in its own fixed device array
instead.  Both entries run the same kernels on the same sequences, so o and
S_T must agree bit for bit, which is the bar the host-entry tests use.  Two
calls are made in a row on one stream, with different shapes and inputs and
the second without S0, so that the array's left-over contents from the first
call cannot leak into the second.

This file runs last (conftest orders test_zz_* files after the others).
"""
import ctypes

import pytest
import torch

import workloads as W


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_92_b200 as g
    g.lib()
    return g


NAMES = ("q", "k", "v", "log_alpha", "b", "w")


def _pinned(inp):
    return {n: inp[n].pin_memory() for n in NAMES}


@pytest.mark.gpu
def test_noalloc_matches_host_entry_two_calls_in_a_row(g):
    a = W.draw(3, 130, 2, 128, 128, seed=9701, dtype=torch.bfloat16, s0_std=0.05)
    b = W.draw(2, 200, 2, 64, 128, seed=9702, dtype=torch.bfloat16, b_scale=2.0)
    ha, hb = _pinned(a), _pinned(b)
    s0a = a["S0"].pin_memory()
    oa = torch.empty(a["v"].shape, dtype=torch.bfloat16).pin_memory()
    sa = torch.empty(3, 2, 128, 128, dtype=torch.float32).pin_memory()
    ob = torch.empty(b["v"].shape, dtype=torch.bfloat16).pin_memory()
    sb = torch.empty(2, 2, 64, 128, dtype=torch.float32).pin_memory()
    stream = torch.cuda.Stream()
    # two calls in a row on one stream, no synchronisation in between
    g.chunk_fwd_host_noalloc(*(ha[n] for n in NAMES), s0a, oa, sa, stream=stream)
    g.chunk_fwd_host_noalloc(*(hb[n] for n in NAMES), None, ob, sb, stream=stream)
    stream.synchronize()
    assert g.device_status() == 0
    # the existing entry with its own workspace, on the same inputs
    ra_o, ra_s = g.chunk_fwd_host(*(ha[n] for n in NAMES), s0a, stream=stream)
    rb_o, rb_s = g.chunk_fwd_host(*(hb[n] for n in NAMES), None, stream=stream)
    stream.synchronize()
    assert torch.equal(oa, ra_o) and torch.equal(sa, ra_s)
    assert torch.equal(ob, rb_o) and torch.equal(sb, rb_s)


def test_noalloc_rejects_shapes_beyond_its_workspace(g):
    """Host-side checks only: nothing reaches the device."""
    L = g.lib()
    P = ctypes.c_void_p
    p = P(16)
    # B8 T4096 H16 d128 bf16 needs two ~119 MB slice buffers, above the 64 MiB array
    assert L.gdn2_chunk_fwd_host_noalloc(p, p, p, p, p, p, None, p, None, 8, 4096, 16, 128, 128, 64, 1,
                                         None) == 2
    assert L.gdn2_chunk_fwd_host_noalloc(p, p, p, p, p, p, None, p, None, 0, 64, 1, 64, 64, 64, 1, None) == 1
    inp = W.draw(1, 4096, 16, 128, 128, seed=1, dtype=torch.bfloat16)
    o = torch.empty(inp["v"].shape, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="no-alloc"):
        g.chunk_fwd_host_noalloc(*(inp[n] for n in NAMES), None, o)
