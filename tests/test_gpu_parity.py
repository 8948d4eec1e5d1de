"""GPU parity: the CUDA kernels, called through the C ABI, against the fp64
oracle on the same seeded inputs.

Bar (stated per output, o and the final state separately):
    max |gpu - oracle| <= tol * max |oracle|,  tol = 1e-4 (fp32 I/O), 2e-2 (bf16 I/O).
Small cases are compared element by element on every head; the full-size
workloads on a sample of heads (all T tokens, all d_v columns of each).
"""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_util import TOL, heads_of, oracle_chunk, rel_inf, state_heads, to_dev

pytestmark = pytest.mark.gpu

cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_92_b200 as g
    g.lib()
    return g


def _run_chunk(g, fn, inp):
    d = to_dev(inp)
    o, S_T = fn(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    torch.cuda.synchronize()
    assert g.device_status() == 0
    return o, S_T


def _check_chunk(g, fn, inp, heads=None, tol=None):
    B, T, H, _ = inp["q"].shape
    heads = list(range(B * H)) if heads is None else heads
    o, S_T = _run_chunk(g, fn, inp)
    ro, rS = oracle_chunk(inp, heads)
    tol = TOL[inp["q"].dtype] if tol is None else tol
    eo = rel_inf(heads_of(o, heads, H), ro)
    es = rel_inf(state_heads(S_T, heads, H), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S_T err {es:.3e} (tol {tol})"
    return eo, es


# ------------------------------------------------------------------ small
SMALL = [  # B, T, H, d_k, d_v, dtype, b_scale, s0
    (1, 64, 1, 64, 64, torch.bfloat16, 1.0, None),
    (2, 192, 3, 64, 64, torch.bfloat16, 1.0, 0.02),
    (1, 128, 2, 128, 128, torch.bfloat16, 1.0, 0.02),
    (2, 256, 2, 128, 64, torch.bfloat16, 2.0, 0.02),
    (1, 320, 2, 128, 256, torch.bfloat16, 2.0, 0.5),
    (1, 128, 2, 64, 192, torch.bfloat16, 1.0, 0.02),
    (1, 256, 2, 64, 64, torch.float32, 1.0, None),
    (2, 128, 2, 128, 128, torch.float32, 2.0, 0.02),
]


@cuda
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}k{c[3]}v{c[4]}{str(c[5])[6:]}")
def test_chunk_small_all_heads(g, case):
    B, T, H, dk, dv, dt, bs, s0 = case
    inp = W.draw(B, T, H, dk, dv, seed=7 + T + dk + dv, dtype=dt, b_scale=bs, s0_std=s0)
    _check_chunk(g, g.chunk_fwd, inp)


@cuda
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}k{c[3]}v{c[4]}{str(c[5])[6:]}")
def test_chunk_cuda_core_small_all_heads(g, case):
    B, T, H, dk, dv, dt, bs, s0 = case
    inp = W.draw(B, T, H, dk, dv, seed=7 + T + dk + dv, dtype=dt, b_scale=bs, s0_std=s0)
    _check_chunk(g, g.chunk_fwd_cuda_core, inp)


# ------------------------------------------- partial last chunk (T % 64 != 0)
TAILS = [  # B, T, H, d_k, d_v, dtype
    (2, 100, 2, 128, 128, torch.bfloat16),
    (1, 1, 2, 128, 256, torch.bfloat16),
    (3, 65, 1, 64, 64, torch.bfloat16),
    (1, 191, 2, 128, 64, torch.bfloat16),
    (2, 37, 2, 64, 128, torch.float32),
    (1, 130, 1, 128, 128, torch.float32),
]


@cuda
@pytest.mark.parametrize("case", TAILS, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}k{c[3]}v{c[4]}{str(c[5])[6:]}")
@pytest.mark.parametrize("impl", ["chunk_fwd", "chunk_fwd_cuda_core"])
def test_chunk_partial_last_chunk(g, case, impl):
    B, T, H, dk, dv, dt = case
    inp = W.draw(B, T, H, dk, dv, seed=40 + T, dtype=dt, b_scale=2.0, s0_std=0.1)
    _check_chunk(g, getattr(g, impl), inp)


@cuda
def test_partial_chunk_writes_nothing_past_T(g):
    """Batch rows are contiguous: the padded rows of row b's last chunk are
    row b+1's first tokens, which must be neither read as padding nor written."""
    B, T, H, dk, dv = 3, 70, 2, 128, 128
    inp = W.draw(B, T, H, dk, dv, seed=8, dtype=torch.bfloat16)
    d = to_dev(inp)
    o = torch.full((B, T, H, dv), 3.0, dtype=torch.bfloat16, device="cuda")
    g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], None, o=o)
    torch.cuda.synchronize()
    ro, _ = oracle_chunk(inp)
    assert rel_inf(heads_of(o, range(B * H), H), ro) <= TOL[torch.bfloat16]


# ------------------------------------------------------- named workloads
@cuda
def test_workload_chunk_f32_small(g):
    wl = W.BY_NAME["chunk_f32_small"]
    _check_chunk(g, g.chunk_fwd, W.make_chunk_inputs(wl))


@cuda
def test_workload_chunk_bf16_small(g):
    wl = W.BY_NAME["chunk_bf16_small"]
    _check_chunk(g, g.chunk_fwd, W.make_chunk_inputs(wl))


# Sampled heads of the full-size workloads (flat b * H + h): spread over every
# batch row, first and last head of a row, the very last head included.
H2048_HEADS = [0, 15, 16, 37, 64, 90, 111, 127]       # B8 x H16
NEGEIG_HEADS = [0, 15, 17, 30, 33, 47, 50, 63]        # B4 x H16


@cuda
def test_workload_chunk_bf16_h2048_sampled_heads(g):
    wl = W.BY_NAME["chunk_bf16_h2048"]
    inp = W.make_chunk_inputs(wl)
    _check_chunk(g, g.chunk_fwd, inp, heads=H2048_HEADS)


@cuda
def test_workload_chunk_bf16_negeig_sampled_heads(g):
    wl = W.BY_NAME["chunk_bf16_negeig"]
    inp = W.make_chunk_inputs(wl)
    _check_chunk(g, g.chunk_fwd, inp, heads=NEGEIG_HEADS)


@cuda
@pytest.mark.parametrize("collapse", ["kda", "gdn"])
def test_workload_negeig_collapses(g, collapse):
    """The expanded-value workload at its full size (B4 T8192 H16 d_k 128 d_v 256)
    with b = w = beta (KDA) and additionally a scalar decay per head (Gated
    DeltaNet), on sampled heads over all T tokens."""
    wl = W.BY_NAME["chunk_bf16_negeig"]
    inp = W.make_chunk_inputs(wl)
    f = W.kda_collapse if collapse == "kda" else W.gdn_collapse
    _check_chunk(g, g.chunk_fwd, f(inp, seed=77, b_scale=wl.b_scale), heads=NEGEIG_HEADS)


# ------------------------------------------------------------- decode
def _decode_run(g, inp, steps):
    d = to_dev(inp)
    S = d["S0"].clone()
    outs = []
    for s in range(steps):
        outs.append(g.decode_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s],
                                  d["w"][s], S).clone())
    torch.cuda.synchronize()
    return torch.stack(outs), S


@cuda
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 256), (64, 192)])
def test_decode_small_all_heads(g, dt, dk, dv):
    import oracle
    B, H, steps = 3, 2, 9
    inp = W.draw(B, steps, H, dk, dv, seed=31 + dk + dv, dtype=dt, s0_std=0.3, b_scale=2.0)
    for n in ("q", "k", "v", "log_alpha", "b", "w"):
        inp[n] = inp[n].transpose(0, 1).contiguous()
    o, S = _decode_run(g, inp, steps)
    ro, rS = oracle.decode_steps(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                                 inp["S0"])
    go = np.stack([o[:, n // H, n % H, :].float().cpu().numpy() for n in range(B * H)])
    tol = TOL[dt]
    assert rel_inf(go, ro) <= tol
    assert rel_inf(state_heads(S, range(B * H), H), rS) <= tol


@cuda
def test_workload_decode_all_1024_steps(g):
    """The decode workload as specified: 256 sequences x H16 x d128 for 1024
    consecutive steps from S0 ~ N(0, 0.02).  Every step's o and the final state
    of 16 sampled heads (spread over the sequences, the last head included)
    against the oracle run over the same 1024 steps.  The 6.4 GB of inputs are
    drawn on the device with the workload's recipe; the oracle reads the same
    cast values of the sampled heads."""
    import oracle
    wl = W.BY_NAME["decode_bf16"]
    steps, H = wl.decode_steps, wl.H
    heads = [0, 17, 300, 1023, 1500, 2047, 2100, 2600, 3000, 3333, 3600, 3900, 4000, 4050, 4094, 4095]
    d = W.make_decode_inputs(wl, steps, device="cuda")
    bi = torch.tensor([x // H for x in heads], device="cuda")
    hi = torch.tensor([x % H for x in heads], device="cuda")
    names = ("q", "k", "v", "log_alpha", "b", "w")
    sample = {n: d[n][:, bi, hi].unsqueeze(1).cpu() for n in names}     # [steps, 1, n, d]
    S0 = d["S0"][bi, hi].unsqueeze(0).cpu()                             # [1, n, d_k, d_v]
    S = d["S0"].clone()
    o_hist = torch.empty(steps, len(heads), wl.d_v, dtype=torch.bfloat16, device="cuda")
    for s in range(steps):
        o = g.decode_step(*(d[n][s] for n in names), S)
        o_hist[s] = o[bi, hi]
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ro, rS = oracle.decode_steps(*(sample[n] for n in names), S0)
    go = o_hist.float().cpu().numpy().transpose(1, 0, 2)               # [n, steps, d_v]
    assert rel_inf(go, ro) <= TOL[torch.bfloat16]
    assert rel_inf(S[bi, hi].double().cpu().numpy(), rS) <= TOL[torch.bfloat16]


@cuda
def test_workload_decode_sampled_heads(g):
    import oracle
    wl = W.BY_NAME["decode_bf16"]
    steps = 64
    inp = W.make_decode_inputs(wl, steps)
    o, S = _decode_run(g, inp, steps)
    heads = [0, 1234, 4095]
    ro, rS = oracle.decode_steps(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                                 inp["S0"], heads=heads)
    go = np.stack([o[:, n // wl.H, n % wl.H, :].float().cpu().numpy() for n in heads])
    assert rel_inf(go, ro) <= TOL[torch.bfloat16]
    assert rel_inf(state_heads(S, heads, wl.H), rS) <= TOL[torch.bfloat16]


# ------------------------------------------------------------ cross-path
@cuda
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_chunk_equals_consecutive_decode(g, dt):
    B, T, H, dk, dv = 2, 128, 2, 128, 128
    inp = W.draw(B, T, H, dk, dv, seed=5, dtype=dt, s0_std=0.02)
    d = to_dev(inp)
    o, S_T = g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    S = d["S0"].clone()
    od = []
    for t in range(T):
        od.append(g.decode_step(*(d[n][:, t].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")), S))
    od = torch.stack(od, dim=1)
    torch.cuda.synchronize()
    scale = od.float().abs().max().item()
    assert (o.float() - od.float()).abs().max().item() <= 2 * TOL[dt] * scale
    assert (S_T - S).abs().max().item() <= 2 * TOL[dt] * S.abs().max().item()


@cuda
def test_state_split_resume(g):
    B, T, H, dk, dv = 1, 256, 2, 128, 128
    inp = W.draw(B, T, H, dk, dv, seed=9, dtype=torch.bfloat16, s0_std=0.02)
    d = to_dev(inp)
    args = lambda sl: [d[n][:, sl].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")]
    o, S_T = g.chunk_fwd(*args(slice(0, T)), d["S0"])
    o1, S1 = g.chunk_fwd(*args(slice(0, 128)), d["S0"])
    o2, S2 = g.chunk_fwd(*args(slice(128, T)), S1)
    torch.cuda.synchronize()
    torch.testing.assert_close(torch.cat([o1, o2], 1), o, rtol=0, atol=0)
    torch.testing.assert_close(S2, S_T, rtol=0, atol=0)


# ------------------------------------------------------------ edge cases
@cuda
def test_empty_sequence_returns_initial_state(g):
    inp = W.draw(2, 0, 2, 64, 64, seed=1, dtype=torch.bfloat16, s0_std=0.1)
    d = to_dev(inp)
    o, S_T = g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    torch.cuda.synchronize()
    assert o.numel() == 0
    torch.testing.assert_close(S_T, d["S0"], rtol=0, atol=0)
    o, S_T = g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], None)
    torch.cuda.synchronize()
    assert S_T.abs().max().item() == 0.0


@cuda
def test_state_in_place_alias(g):
    inp = W.draw(1, 128, 2, 128, 128, seed=2, dtype=torch.bfloat16, s0_std=0.05)
    d = to_dev(inp)
    o_ref, S_ref = g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    S = d["S0"].clone()
    o, _ = g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S, S_T=S)
    torch.cuda.synchronize()
    torch.testing.assert_close(o, o_ref, rtol=0, atol=0)
    torch.testing.assert_close(S, S_ref, rtol=0, atol=0)


@cuda
def test_outputs_stay_in_bounds(g):
    """Canary regions around o and S_T are left untouched."""
    B, T, H, dk, dv = 1, 128, 2, 128, 128
    inp = W.draw(B, T, H, dk, dv, seed=3, dtype=torch.bfloat16)
    d = to_dev(inp)
    n_o, n_s, pad = B * T * H * dv, B * H * dk * dv, 4096
    ob = torch.full((n_o + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    sb = torch.full((n_s + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    o = ob[pad:pad + n_o].view(B, T, H, dv)
    S_T = sb[pad:pad + n_s].view(B, H, dk, dv)
    g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], None, o=o, S_T=S_T)
    torch.cuda.synchronize()
    assert torch.all(ob[:pad] == 7.0) and torch.all(ob[pad + n_o:] == 7.0)
    assert torch.all(sb[:pad] == 7.0) and torch.all(sb[pad + n_s:] == 7.0)


@cuda
def test_bounded_wait_reports_timeout(g):
    assert g.device_status() == 0
    assert g.selftest_wait_timeout(2000) == 5          # GDN2_ERR_DEVICE_TIMEOUT
    assert g.device_status() == 0                      # read-and-clear
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


@cuda
def test_unsupported_shapes_rejected_on_device_pointers(g):
    inp = to_dev(W.draw(1, 96, 1, 96, 64, seed=4, dtype=torch.bfloat16))
    with pytest.raises(g.Gdn2Error) as e:
        g.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], None)
    assert e.value.status == 2
    inp = to_dev(W.draw(1, 64, 1, 64, 64, seed=4, dtype=torch.bfloat16))
    with pytest.raises(g.Gdn2Error) as e:
        g.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], None, chunk=48)
    assert e.value.status == 2
