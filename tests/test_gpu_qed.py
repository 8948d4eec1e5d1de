"""GPU parity of the second, query-derived erase direction (gdn2_chunk_fwd_qed,
gdn2_decode_step_qed) against the fp64 oracle's forward_qed on the same seeded
inputs.

Bar: max |gpu - oracle| <= tol * max |oracle| for o and for the final state;
tol = 1e-4 for fp32 I/O and 2e-2 for bf16 I/O (both kernels compute with fp32
products; bf16 I/O rounds the inputs and o).
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


def _inputs(B, T, H, dk, dv, dt, seed):
    inp = W.draw(B, T, H, dk, dv, seed=seed, dtype=dt, s0_std=0.05)
    inp["c"] = W.draw_qed_gate((B, T, H), dk, seed=seed + 1, dtype=dt)
    return inp


def _run_chunk(g, d, eps=1e-6):
    o, S = g.chunk_fwd_qed(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["c"], d["w"], d["S0"], qed_eps=eps)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    return o, S


def _check_chunk(g, B, T, H, dk, dv, dt, seed, heads=None, eps=1e-6):
    inp = _inputs(B, T, H, dk, dv, dt, seed)
    o, S = _run_chunk(g, to_dev(inp), eps)
    heads = list(range(B * H)) if heads is None else heads
    ro, rS = oracle.forward_qed(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["c"], inp["w"],
                                S0=inp["S0"], heads=heads, qed_eps=eps)
    got = np.stack([o[x // H, :, x % H].float().cpu().numpy() for x in heads])
    gS = np.stack([S[x // H, x % H].double().cpu().numpy() for x in heads])
    tol = TOL[dt]
    eo, es = rel_inf(got, ro), rel_inf(gS, rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S err {es:.3e} (tol {tol})"


CASES = [  # B, T, H, d_k, d_v, dtype (T % 32 != 0: a partial last chunk)
    (1, 100, 2, 64, 64, torch.float32),
    (2, 70, 1, 128, 128, torch.float32),
    (1, 150, 2, 128, 128, torch.bfloat16),
    (1, 33, 1, 64, 192, torch.bfloat16),
    (1, 1, 1, 128, 64, torch.float32),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}dk{c[3]}dv{c[4]}{str(c[5])[6:]}")
def test_chunk_qed(g, case):
    B, T, H, dk, dv, dt = case
    _check_chunk(g, B, T, H, dk, dv, dt, seed=8000 + T + dk + dv)


def test_chunk_qed_zero_epsilon(g):
    _check_chunk(g, 1, 64, 2, 64, 64, torch.float32, seed=8100, eps=0.0)


def test_chunk_qed_headline_size_sampled(g):
    """B8 T4096 H16 d128 bf16 (the tensor-core kernel), 8 heads over every batch row."""
    _check_chunk(g, 8, 4096, 16, 128, 128, torch.bfloat16, seed=8200, heads=[0, 15, 16, 45, 64, 90, 111, 127])


# bf16 I/O runs the tensor-core kernel: 32 tokens (64 pseudo-rows) a chunk
TC_CASES = [  # B, T, H, d_k, d_v
    (2, 200, 2, 128, 256),   # two 128-column slices, partial last chunk
    (1, 97, 2, 64, 128),     # 3 chunks + 1 token
    (1, 32, 1, 128, 128),    # exactly one chunk
    (1, 1, 1, 128, 64),      # a single token
    (3, 64, 1, 64, 64),
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: "B%dT%dH%dk%dv%d" % c)
def test_chunk_qed_tensor_core(g, case):
    B, T, H, dk, dv = case
    _check_chunk(g, B, T, H, dk, dv, torch.bfloat16, seed=8250 + T + dv)


def test_chunk_qed_tensor_core_zero_gate_matches_gdn2(g):
    """c = 0 leaves GDN-2: the tensor-core QED kernel (32-token chunks) and the
    GDN-2 tensor-core kernel (64-token chunks) agree within the bf16 bar."""
    inp = to_dev(_inputs(2, 300, 2, 128, 128, torch.bfloat16, 8410))
    inp["c"] = torch.zeros_like(inp["c"])
    o1, S1 = _run_chunk(g, inp)
    o2, S2 = g.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], inp["S0"])
    torch.cuda.synchronize()
    assert float((o1.float() - o2.float()).abs().max()) <= 2e-2 * float(o2.float().abs().max())
    assert float((S1 - S2).abs().max()) <= 2e-2 * float(S2.abs().max())


def test_chunk_qed_tensor_core_state_split_resume(g):
    """A run resumed from S_T at a chunk boundary equals the whole run bit for bit."""
    inp = to_dev(_inputs(1, 256, 2, 128, 128, torch.bfloat16, 8420))
    names = ("q", "k", "v", "log_alpha", "b", "c", "w")
    part = lambda sl: {**{n: inp[n][:, sl].contiguous() for n in names}}
    o, S = g.chunk_fwd_qed(*(inp[n] for n in ("q", "k", "v", "log_alpha", "b", "c", "w")), inp["S0"])
    a, b = part(slice(0, 96)), part(slice(96, 256))
    o1, S1 = g.chunk_fwd_qed(*(a[n] for n in ("q", "k", "v", "log_alpha", "b", "c", "w")), inp["S0"])
    o2, S2 = g.chunk_fwd_qed(*(b[n] for n in ("q", "k", "v", "log_alpha", "b", "c", "w")), S1)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([o1, o2], 1), o)
    assert torch.equal(S2, S)


def test_chunk_qed_empty_sequence(g):
    inp = to_dev(_inputs(1, 1, 2, 64, 64, torch.float32, 8300))
    e = {n: (t[:, :0].contiguous() if n not in ("S0",) else t) for n, t in inp.items()}
    o, S = _run_chunk(g, e)
    assert o.numel() == 0 and torch.equal(S, inp["S0"])


def test_chunk_qed_zero_gate_matches_gdn2(g):
    """c = 0 leaves GDN-2: the QED kernel and the GDN-2 CUDA-core kernel agree to fp32 rounding."""
    inp = to_dev(_inputs(2, 130, 2, 128, 128, torch.float32, 8400))
    inp["c"] = torch.zeros_like(inp["c"])
    o1, S1 = _run_chunk(g, inp)
    o2, S2 = g.chunk_fwd_cuda_core(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], inp["S0"])
    torch.cuda.synchronize()
    assert float((o1 - o2).abs().max()) <= 2e-5 * float(o2.abs().max())
    assert float((S1 - S2).abs().max()) <= 2e-5 * float(S2.abs().max())


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 128, 256], ids=lambda x: f"dv{x}")
def test_decode_qed(g, dt, dv):
    B, H, dk, steps = 3, 2, 128, 6
    inp = W.draw(steps, B, H, dk, dv, seed=8500 + dv, dtype=dt)   # [steps, B, H, d]
    c = W.draw_qed_gate((steps, B, H), dk, seed=8600 + dv, dtype=dt)
    S0 = 0.05 * torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(8700 + dv))
    d = to_dev(inp)
    dc, S = c.cuda(), S0.cuda().clone()
    outs = [g.decode_step_qed(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s], dc[s], d["w"][s], S)
            for s in range(steps)]
    torch.cuda.synchronize()
    assert g.device_status() == 0
    o = torch.stack(outs)
    ro, rS = oracle.decode_steps_qed(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], c, inp["w"], S0)
    got = np.stack([o[:, x // H, x % H].float().cpu().numpy() for x in range(B * H)])
    tol = TOL[dt]
    eo = rel_inf(got, ro)
    es = rel_inf(S.double().cpu().numpy().reshape(B * H, dk, dv), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S err {es:.3e} (tol {tol})"


def test_chunk_qed_equals_decode_steps(g):
    """The chunk form and T decode steps compute the same recurrence (fp32)."""
    B, T, H, dk, dv = 1, 45, 2, 64, 128
    inp = to_dev(_inputs(B, T, H, dk, dv, torch.float32, 8800))
    o1, S1 = _run_chunk(g, inp)
    S = inp["S0"].clone()
    outs = []
    for t in range(T):
        sl = lambda n: inp[n][:, t].contiguous()
        outs.append(g.decode_step_qed(sl("q"), sl("k"), sl("v"), sl("log_alpha"), sl("b"), sl("c"), sl("w"), S))
    torch.cuda.synchronize()
    o2 = torch.stack(outs, dim=1)
    assert float((o1 - o2).abs().max()) <= 2e-5 * float(o2.abs().max())
    assert float((S1 - S).abs().max()) <= 2e-5 * float(S.abs().max())
