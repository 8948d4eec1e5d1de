"""GPU parity of packed variable-length sequences (cu_seqlens) and value
heads (HV = G * H, value head hv reading key head hv // G) through the _ex
entry points, against the fp64 oracle on the same seeded inputs.

Bar as for the plain path, per output: max |gpu - oracle| <= tol * max |oracle|,
tol = 1e-4 (fp32 I/O, CUDA-core kernel), 2e-2 (bf16 I/O, tensor-core kernel).
A packed sequence must also come out exactly as the same sequence run alone.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import TOL, rel_inf, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_92_b200 as g
    g.lib()
    return g


def _run_ex(g, d, cu=None, **kw):
    o, S_T = g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"],
                            cu_seqlens=cu, **kw)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    return o, S_T


def _oracle_kw(inp, prep, epi):
    return dict(prep=prep, gate=inp["gate"] if epi else None,
                norm_weight=inp["norm_weight"] if epi else None, norm_eps=1e-5)


def _gpu_kw(d, prep, epi):
    return dict(prep=prep, gate=d["gate"] if epi else None,
                norm_weight=d["norm_weight"] if epi else None, norm_eps=1e-5)


def _inputs(T, H, HV, dk, dv, dt, seed, prep, B=1):
    inp = W.draw_raw(B, T, H, dk, dv, seed=seed, dtype=dt, qk_scale=2.0, s0_std=0.05, HV=HV)
    if not prep:   # prepared q, k, b, w (the epilogue may still be on)
        inp.update({n: t for n, t in W.draw(B, T, H, dk, dv, seed=seed + 1, dtype=dt, HV=HV).items()
                    if n != "S0"})
    return inp


def _packed_check(g, lens, H, HV, dk, dv, dt, seed, prep=False, epi=False):
    """Packed sequences of `lens` tokens; per (sequence, value head) against the oracle."""
    N = len(lens)
    cu = W.cu_seqlens_of(lens)
    T = int(cu[-1])
    inp = _inputs(T, H, HV, dk, dv, dt, seed, prep)
    inp["S0"] = 0.05 * torch.randn(N, HV, dk, dv, generator=torch.Generator().manual_seed(seed + 2))
    d = to_dev(inp)
    o, S_T = _run_ex(g, d, cu.cuda(), **_gpu_kw(d, prep, epi))
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                            S0=inp["S0"], cu_seqlens=cu.numpy(), **_oracle_kw(inp, prep, epi))
    tol = TOL[dt]
    got = [o[0, int(cu[x // HV]):int(cu[x // HV + 1]), x % HV].float().cpu().numpy() for x in range(N * HV)]
    scale = max(float(np.max(np.abs(r))) for r in ro if r.size)
    eo = max((float(np.max(np.abs(a - r))) for a, r in zip(got, ro) if r.size), default=0.0) / scale
    es = rel_inf(S_T.double().cpu().numpy().reshape(N * HV, dk, dv), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S_T err {es:.3e} (tol {tol})"
    return inp, d, cu, o, S_T


# lengths: empty, single token, chunk-1, chunk, chunk+1, several chunks, ragged
LENS = [0, 1, 63, 64, 65, 200, 130, 7]
PACKED = [  # H, HV, d_k, d_v, dtype
    (2, 2, 128, 128, torch.bfloat16),
    (2, 4, 64, 64, torch.bfloat16),
    (1, 2, 128, 256, torch.bfloat16),
    (2, 4, 64, 64, torch.float32),
    (2, 2, 128, 128, torch.float32),
]


@pytest.mark.parametrize("case", PACKED, ids=lambda c: f"H{c[0]}HV{c[1]}dk{c[2]}dv{c[3]}{str(c[4])[6:]}")
def test_packed_sequences(g, case):
    H, HV, dk, dv, dt = case
    _packed_check(g, LENS, H, HV, dk, dv, dt, seed=6000 + dk + dv)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("mode", [(True, False), (True, True), (False, True)], ids=["prep", "prep_epi", "epi"])
def test_packed_sequences_fused(g, dt, mode):
    prep, epi = mode
    _packed_check(g, [70, 0, 129, 5, 64], 2, 4, 128, 128, dt, seed=6100, prep=prep, epi=epi)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_packed_sequence_equals_separate_call(g, dt):
    """A sequence packed between others gives exactly the output and state of the same
    sequence run alone (the neighbours' tokens never enter its chunks)."""
    lens = [100, 77, 192, 1]
    inp, d, cu, o, S_T = _packed_check(g, lens, 2, 4, 128, 128, dt, seed=6200)
    for i, n in enumerate(lens):
        a, e = int(cu[i]), int(cu[i + 1])
        one = {k: d[k][:, a:e].contiguous() for k in ("q", "k", "v", "log_alpha", "b", "w")}
        one["S0"] = d["S0"][i:i + 1].contiguous()
        o1, S1 = _run_ex(g, one)
        assert torch.equal(o1[0], o[0, a:e]), f"sequence {i}: o differs from the packed run"
        assert torch.equal(S1[0], S_T[i]), f"sequence {i}: S_T differs from the packed run"


def test_packed_many_short_sequences(g):
    """Many short sequences drawn from a length mix (several per chunk width)."""
    lens = W.packed_lengths(48, 40, seed=6300)
    _packed_check(g, lens, 2, 2, 128, 128, torch.bfloat16, seed=6301)


def test_packed_all_empty_but_one_state_passthrough(g):
    """Empty sequences leave S_T = S0 exactly and write no o rows."""
    lens = [0, 0, 96, 0]
    inp, d, cu, o, S_T = _packed_check(g, lens, 1, 1, 64, 64, torch.bfloat16, seed=6400)
    for i in (0, 1, 3):
        assert torch.equal(S_T[i], d["S0"][i])


HEADS = [  # B, T, H, HV, d_k, d_v, dtype
    (2, 150, 2, 6, 128, 128, torch.bfloat16),    # G = 3
    (1, 130, 2, 4, 64, 64, torch.bfloat16),
    (1, 100, 1, 2, 128, 256, torch.bfloat16),
    (1, 90, 2, 4, 64, 192, torch.bfloat16),
    (2, 96, 2, 6, 128, 128, torch.float32),
    (1, 70, 1, 4, 64, 64, torch.float32),
]


@pytest.mark.parametrize("case", HEADS, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}HV{c[3]}dk{c[4]}dv{c[5]}{str(c[6])[6:]}")
@pytest.mark.parametrize("mode", [(False, False), (True, True)], ids=["plain", "prep_epi"])
def test_value_heads(g, case, mode):
    B, T, H, HV, dk, dv, dt = case
    prep, epi = mode
    inp = _inputs(T, H, HV, dk, dv, dt, 6500 + T + HV, prep, B=B)
    d = to_dev(inp)
    o, S_T = _run_ex(g, d, **_gpu_kw(d, prep, epi))
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                            S0=inp["S0"], **_oracle_kw(inp, prep, epi))
    got = np.stack([o[x // HV, :, x % HV].float().cpu().numpy() for x in range(B * HV)])
    tol = TOL[dt]
    eo = rel_inf(got, ro)
    es = rel_inf(S_T.double().cpu().numpy().reshape(B * HV, dk, dv), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S_T err {es:.3e} (tol {tol})"


def test_value_heads_equal_repeated_key_heads(g):
    """HV = G H gives exactly what H' = HV key heads give with each key-side tensor
    repeated G times along the head axis (the sharing is a pure index map)."""
    B, T, H, HV, dk, dv = 1, 140, 2, 6, 128, 128
    inp = _inputs(T, H, HV, dk, dv, torch.bfloat16, 6600, False, B=B)
    d = to_dev(inp)
    o1, S1 = _run_ex(g, d)
    rep = dict(d)
    for n in ("q", "k", "log_alpha", "b"):
        rep[n] = d[n].repeat_interleave(HV // H, dim=2).contiguous()
    o2, S2 = _run_ex(g, rep)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("dv", [64, 128, 256], ids=lambda x: f"dv{x}")
@pytest.mark.parametrize("mode", [(False, False), (True, True)], ids=["plain", "prep_epi"])
def test_decode_value_heads(g, dt, dv, mode):
    prep, epi = mode
    B, H, HV, dk, steps = 3, 2, 4, 128, 5
    inp = W.draw_raw(B, None, H, dk, dv, seed=6700 + dv, dtype=dt, qk_scale=2.0, s0_std=0.05,
                     steps=steps, HV=HV)
    if not prep:
        p = W.draw(steps, B, H, dk, dv, seed=6800 + dv, dtype=dt, HV=HV)   # [steps, B, heads, d]
        for n in ("q", "k", "b", "w"):
            inp[n] = p[n]
    d = to_dev(inp)
    S = d["S0"].clone()
    outs = []
    for s in range(steps):
        outs.append(g.decode_step_ex(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s],
                                     d["w"][s], S, prep=prep, gate=d["gate"][s] if epi else None,
                                     norm_weight=d["norm_weight"] if epi else None))
    torch.cuda.synchronize()
    assert g.device_status() == 0
    o = torch.stack(outs)   # [steps, B, HV, d_v]
    ro, rS = oracle.decode_steps(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                                 inp["S0"], prep=prep, gate=inp["gate"] if epi else None,
                                 norm_weight=inp["norm_weight"] if epi else None)
    got = np.stack([o[:, x // HV, x % HV].float().cpu().numpy() for x in range(B * HV)])
    tol = TOL[dt]
    eo = rel_inf(got, ro)
    es = rel_inf(S.double().cpu().numpy().reshape(B * HV, dk, dv), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S err {es:.3e} (tol {tol})"


def test_malformed_offsets_are_reported_not_read(g):
    """Decreasing offsets: that sequence is skipped and the status word says so."""
    H, dk, dv = 1, 64, 64
    inp = W.draw(1, 128, H, dk, dv, seed=6900, dtype=torch.bfloat16, s0_std=0.05)
    d = to_dev(inp)
    d["S0"] = torch.zeros(2, H, dk, dv, device="cuda")
    cu = torch.tensor([0, 100, 90], dtype=torch.int32, device="cuda")
    o, S_T = g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"],
                            cu_seqlens=cu)
    assert g.device_status() == 1   # GDN2_ERR_INVALID_ARG recorded by the skipped sequence
    assert g.device_status() == 0   # and cleared by the read


CHUNKS = [  # B, T, H, d_k, d_v, dtype
    (1, 150, 2, 64, 64, torch.float32),
    (2, 97, 2, 128, 128, torch.float32),
    (1, 150, 2, 128, 128, torch.bfloat16),
    (1, 77, 2, 64, 192, torch.bfloat16),
]


@pytest.mark.parametrize("case", CHUNKS, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}dk{c[3]}dv{c[4]}{str(c[5])[6:]}")
@pytest.mark.parametrize("chunk", [16, 32], ids=lambda c: f"chunk{c}")
def test_chunk_lengths(g, case, chunk):
    """chunk_size 16 and 32 (CUDA-core kernel) against the oracle, which has no chunks."""
    B, T, H, dk, dv, dt = case
    inp = W.draw(B, T, H, dk, dv, seed=7000 + T + dk, dtype=dt, s0_std=0.05)
    d = to_dev(inp)
    o, S_T = g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], chunk=chunk)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], S0=inp["S0"])
    got = np.stack([o[x // H, :, x % H].float().cpu().numpy() for x in range(B * H)])
    tol = TOL[dt]
    eo = rel_inf(got, ro)
    es = rel_inf(S_T.double().cpu().numpy().reshape(B * H, dk, dv), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S_T err {es:.3e} (tol {tol})"


def test_chunk_length_invariance_fp32(g):
    """The chunk form is an exact regrouping: chunk 16, 32 and 64 agree to fp32 rounding."""
    inp = W.draw(2, 300, 2, 128, 128, seed=7100, dtype=torch.float32, s0_std=0.05)
    d = to_dev(inp)
    outs = [g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], chunk=c)
            for c in (16, 32, 64)]
    torch.cuda.synchronize()
    o64, S64 = outs[-1]
    for o, S in outs[:-1]:
        assert float((o - o64).abs().max()) <= 2e-5 * float(o64.abs().max())
        assert float((S - S64).abs().max()) <= 2e-5 * float(S64.abs().max())


def test_chunk32_packed_value_heads_fused(g):
    """chunk 32 with packed sequences, value heads, prep and epilogue together."""
    lens = [33, 0, 96, 5]
    cu = W.cu_seqlens_of(lens)
    T, H, HV, dk, dv = int(cu[-1]), 2, 4, 128, 128
    inp = _inputs(T, H, HV, dk, dv, torch.bfloat16, 7200, True)
    inp["S0"] = 0.05 * torch.randn(len(lens), HV, dk, dv, generator=torch.Generator().manual_seed(7201))
    d = to_dev(inp)
    o, S_T = _run_ex(g, d, cu.cuda(), chunk=32, **_gpu_kw(d, True, True))
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                            S0=inp["S0"], cu_seqlens=cu.numpy(), **_oracle_kw(inp, True, True))
    got = [o[0, int(cu[x // HV]):int(cu[x // HV + 1]), x % HV].float().cpu().numpy()
           for x in range(len(lens) * HV)]
    scale = max(float(np.max(np.abs(r))) for r in ro if r.size)
    eo = max(float(np.max(np.abs(a - r))) for a, r in zip(got, ro) if r.size) / scale
    es = rel_inf(S_T.double().cpu().numpy().reshape(len(lens) * HV, dk, dv), rS)
    assert eo <= 2e-2 and es <= 2e-2, f"o err {eo:.3e}, S_T err {es:.3e}"


def test_packed_equal_lengths_ties(g):
    """Equal lengths (rank ties broken by index) and a mix around one chunk."""
    _packed_check(g, [64, 64, 30, 64, 30, 0, 64, 30], 2, 2, 128, 128, torch.bfloat16, seed=7300)


def test_packed_more_sequences_than_ranked(g):
    """1100 short sequences: more than the kernel ranks, so slot z runs sequence z."""
    rng = np.random.default_rng(7400)
    lens = [int(x) for x in rng.integers(0, 6, size=1100)]
    _packed_check(g, lens, 1, 1, 64, 64, torch.bfloat16, seed=7401)
