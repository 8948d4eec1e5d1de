"""The debug build (libgdn2_debug.so, -DGDN2_DEBUG_BOUNDS) on the GPU.

Every per-thread global load and store of its kernels is checked against the
extent of the argument buffer it belongs to, with the extents published by the
host entry points from the call's pointers and sizes.  On valid calls of every
kernel path -- tensor-core chunk (plain, fused, packed, value heads, d_v split,
token tail), CUDA-core chunk (fp32, chunk 16/32, per-chunk token steps), the
query-derived erase direction, decode (plain, fused with its cluster epilogue,
value heads) and the host-buffer entries -- no check may fail, and the results
must equal the release library's bit for bit (the checks change no
arithmetic).  The check itself is exercised by gdn2_selftest_bounds on
addresses alone: nothing here makes an out-of-range access.
"""
import pytest
import torch

import workloads as W
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_92_b200 as g
    g.lib()
    return g


def _both(g, run):
    """Run `run(g)` through the release library, then the debug build; return
    both results (tuples of tensors) after checking the debug run's status."""
    rel = run(g)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    with g.debug_bounds():
        dbg = run(g)
        torch.cuda.synchronize()
        st = g.device_status()
        site = g.debug_bounds_site()
    assert st == 0 and site is None, f"status {st}, first failed check at {site}"
    return rel, dbg


def _same(rel, dbg):
    for a, b in zip(rel, dbg):
        if a is None:
            assert b is None
            continue
        assert torch.equal(a, b), f"max diff {(a.float() - b.float()).abs().max().item():.3e}"


def test_selftest_reports_out_of_bounds(g):
    with g.debug_bounds():
        assert g.device_status() == 0
        assert g.selftest_bounds() == g.OUT_OF_BOUNDS
        site = g.debug_bounds_site()
        assert site is not None and site[0] == "q" and site[1] > 0
        assert g.device_status() == 0 and g.debug_bounds_site() is None   # both read and cleared


def _chunk_case(B, T, H, dk, dv, dtype, *, chunk=64, s0=True, decay=None, seed=0):
    inp = W.draw(B, T, H, dk, dv, seed=seed, dtype=dtype, s0_std=0.05 if s0 else None)
    if decay == "mixed":
        inp = W.with_mixed_decay(inp, seed + 1)
    elif decay == "burst":
        inp = W.with_decay_burst(inp, 70, 80, -12.0)
    return to_dev(inp)


CHUNK_CASES = [  # B, T, H, d_k, d_v, dtype, chunk, decay
    (2, 200, 2, 128, 128, torch.bfloat16, 64, None),      # tensor cores, ragged tail
    (1, 130, 2, 64, 64, torch.bfloat16, 64, None),
    (1, 150, 1, 128, 256, torch.bfloat16, 64, None),      # two CTAs per head
    (1, 200, 2, 128, 128, torch.bfloat16, 64, "burst"),   # chunked, then the token tail
    (1, 130, 1, 128, 128, torch.bfloat16, 64, "mixed"),   # token tail from chunk 0
    (1, 100, 2, 64, 64, torch.float32, 64, None),         # CUDA cores
    (1, 100, 1, 128, 128, torch.float32, 64, "mixed"),    # CUDA cores, per-chunk token steps
    (1, 90, 2, 128, 64, torch.bfloat16, 16, None),
    (1, 90, 1, 64, 128, torch.bfloat16, 32, None),
]


@pytest.mark.parametrize("B,T,H,dk,dv,dtype,chunk,decay", CHUNK_CASES)
def test_chunk_debug_equals_release(g, B, T, H, dk, dv, dtype, chunk, decay):
    d = _chunk_case(B, T, H, dk, dv, dtype, chunk=chunk, decay=decay)
    rel, dbg = _both(g, lambda g: g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"],
                                              chunk=chunk))
    _same(rel, dbg)


@pytest.mark.parametrize("dv,decay", [(128, None), (256, None), (128, "burst")])
def test_fused_chunk_debug_equals_release(g, dv, decay):
    d = to_dev(W.draw_raw(1, 170, 2, 128, dv, seed=5, qk_scale=2.0, s0_std=0.05))
    if decay == "burst":
        d = W.with_decay_burst(d, 70, 80, -12.0)

    def run(g):
        return g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], prep=True,
                              gate=d["gate"], norm_weight=d["norm_weight"])
    _same(*_both(g, run))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_packed_value_heads_debug_equals_release(g, dtype):
    lengths = [70, 0, 129, 33, 64]
    cu = W.cu_seqlens_of(lengths).cuda()
    d = to_dev(W.draw(1, sum(lengths), 2, 128, 128, seed=9, dtype=dtype, HV=4))
    S0 = 0.05 * torch.randn(len(lengths), 4, 128, 128, device="cuda")

    def run(g):
        return g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0, cu_seqlens=cu)
    _same(*_both(g, run))


@pytest.mark.parametrize("dtype,decay", [(torch.bfloat16, None), (torch.bfloat16, "burst"), (torch.float32, None)])
def test_qed_chunk_debug_equals_release(g, dtype, decay):
    d = _chunk_case(1, 150, 2, 128, 128, dtype, decay=decay, seed=3)
    c = W.draw_qed_gate((1, 150, 2), 128, seed=4, dtype=dtype).cuda()
    rel, dbg = _both(g, lambda g: g.chunk_fwd_qed(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], c, d["w"],
                                                  d["S0"]))
    _same(rel, dbg)


def test_host_entries_debug_equal_release(g):
    d = W.draw(3, 150, 2, 128, 128, seed=12, s0_std=0.05)
    hp = {n: (t.pin_memory() if t is not None else None) for n, t in d.items()}

    def run(g):
        o1, s1 = g.chunk_fwd_host(hp["q"], hp["k"], hp["v"], hp["log_alpha"], hp["b"], hp["w"], hp["S0"])
        o2 = torch.empty_like(hp["v"]).pin_memory()
        s2 = torch.empty_like(hp["S0"]).pin_memory()
        g.chunk_fwd_host_noalloc(hp["q"], hp["k"], hp["v"], hp["log_alpha"], hp["b"], hp["w"], hp["S0"], o2, s2)
        torch.cuda.synchronize()
        return o1.clone(), s1.clone(), o2.clone(), s2.clone()
    _same(*_both(g, run))


DECODE_CASES = [  # B, H, HV, d_k, d_v, dtype, fused
    (4, 2, 2, 128, 128, torch.bfloat16, False),
    (3, 2, 4, 64, 192, torch.bfloat16, False),
    (2, 2, 2, 128, 64, torch.float32, False),
    (4, 2, 2, 128, 256, torch.bfloat16, True),    # the epilogue's cluster over two blocks
    (2, 2, 2, 64, 128, torch.float32, True),
]


@pytest.mark.parametrize("B,H,HV,dk,dv,dtype,fused", DECODE_CASES)
def test_decode_debug_equals_release(g, B, H, HV, dk, dv, dtype, fused):
    d = to_dev(W.draw_raw(B, None, H, dk, dv, seed=21, dtype=dtype, steps=3, HV=HV, s0_std=0.05))

    def run(g):
        S = d["S0"].clone()
        outs = []
        for t in range(3):
            if fused:
                outs.append(g.decode_step_ex(d["q"][t], d["k"][t], d["v"][t], d["log_alpha"][t], d["b"][t],
                                             d["w"][t], S, prep=True, gate=d["gate"][t],
                                             norm_weight=d["norm_weight"]))
            else:
                outs.append(g.decode_step_ex(d["q"][t], d["k"][t], d["v"][t], d["log_alpha"][t], d["b"][t],
                                             d["w"][t], S))
        return tuple(outs) + (S,)
    _same(*_both(g, run))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_qed_decode_debug_equals_release(g, dtype):
    d = to_dev(W.draw(3, 1, 2, 128, 128, seed=31, dtype=dtype, s0_std=0.05))
    c = W.draw_qed_gate((3, 2), 128, seed=32, dtype=dtype).cuda()
    sq = {n: d[n][:, 0].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")}

    def run(g):
        S = d["S0"].clone()
        o = g.decode_step_qed(sq["q"], sq["k"], sq["v"], sq["log_alpha"], sq["b"], c, sq["w"], S)
        return o, S
    _same(*_both(g, run))
