"""GPU parity at the edges of the built shapes: d_v = 512 (the largest), d_v = 320
(an odd number of 64-column slices), d_k = 64 with wide d_v, and the fused epilogue
over a 512-wide row (four decode CTAs in one cluster; the chunk kernel's separate
normalisation pass).  Bar as elsewhere: max |gpu - oracle| <= tol * max |oracle|,
tol = 1e-4 (fp32 I/O), 2e-2 (bf16 I/O)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import TOL, heads_of, rel_inf, state_heads, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_92_b200 as g
    g.lib()
    return g


WIDE = [  # B, T, H, d_k, d_v, dtype
    (1, 130, 2, 128, 512, torch.bfloat16),
    (1, 100, 2, 64, 512, torch.bfloat16),
    (1, 90, 1, 128, 320, torch.bfloat16),
    (1, 70, 1, 128, 512, torch.float32),
]


@pytest.mark.parametrize("case", WIDE, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}dk{c[3]}dv{c[4]}{str(c[5])[6:]}")
@pytest.mark.parametrize("impl", ["chunk_fwd", "chunk_fwd_cuda_core"])
def test_chunk_wide_value_dim(g, case, impl):
    B, T, H, dk, dv, dt = case
    inp = W.draw(B, T, H, dk, dv, seed=9000 + T + dv, dtype=dt, s0_std=0.05)
    d = to_dev(inp)
    o, S = getattr(g, impl)(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    torch.cuda.synchronize()
    assert g.device_status() == 0
    heads = list(range(B * H))
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], S0=inp["S0"])
    tol = TOL[dt]
    eo, es = rel_inf(heads_of(o, heads, H), ro), rel_inf(state_heads(S, heads, H), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S err {es:.3e} (tol {tol})"


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("dk", [64, 128])
def test_decode_wide_value_dim(g, dt, dk):
    B, H, dv, steps = 2, 2, 512, 4
    inp = W.draw(steps, B, H, dk, dv, seed=9100 + dk, dtype=dt)
    S0 = 0.05 * torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(9101))
    d = to_dev(inp)
    S = S0.cuda().clone()
    outs = [g.decode_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s], d["w"][s], S)
            for s in range(steps)]
    torch.cuda.synchronize()
    assert g.device_status() == 0
    o = torch.stack(outs)
    ro, rS = oracle.decode_steps(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], S0)
    got = np.stack([o[:, x // H, x % H].float().cpu().numpy() for x in range(B * H)])
    tol = TOL[dt]
    eo = rel_inf(got, ro)
    es = rel_inf(S.double().cpu().numpy().reshape(B * H, dk, dv), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S err {es:.3e} (tol {tol})"


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_fused_epilogue_over_512_wide_rows(g, dt):
    """Chunk (separate normalisation pass) and decode (a cluster of four CTAs) with the
    input prep and the gated RMS-norm epilogue over d_v = 512."""
    B, T, H, dk, dv = 1, 80, 2, 128, 512
    inp = W.draw_raw(B, T, H, dk, dv, seed=9200, dtype=dt, qk_scale=2.0, s0_std=0.05)
    d = to_dev(inp)
    o, S = g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], prep=True,
                          gate=d["gate"], norm_weight=d["norm_weight"])
    torch.cuda.synchronize()
    assert g.device_status() == 0
    heads = list(range(B * H))
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], S0=inp["S0"],
                            prep=True, gate=inp["gate"], norm_weight=inp["norm_weight"])
    tol = TOL[dt]
    assert rel_inf(heads_of(o, heads, H), ro) <= tol and rel_inf(state_heads(S, heads, H), rS) <= tol
    # decode: one token per sequence from the same S0
    q1 = {n: inp[n][:, 0].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w", "gate")}
    dq = to_dev(q1)
    Sd = d["S0"].clone()
    od = g.decode_step_ex(dq["q"], dq["k"], dq["v"], dq["log_alpha"], dq["b"], dq["w"], Sd, prep=True,
                          gate=dq["gate"], norm_weight=d["norm_weight"])
    torch.cuda.synchronize()
    assert g.device_status() == 0
    sb = lambda x: x[None]   # [1 step, B, H, d]
    ro2, rS2 = oracle.decode_steps(sb(q1["q"]), sb(q1["k"]), sb(q1["v"]), sb(q1["log_alpha"]), sb(q1["b"]),
                                   sb(q1["w"]), inp["S0"], prep=True, gate=sb(q1["gate"]),
                                   norm_weight=inp["norm_weight"])
    got = np.stack([od[x // H, x % H].float().cpu().numpy() for x in heads])
    assert rel_inf(got, ro2[:, 0]) <= tol
    assert rel_inf(Sd.double().cpu().numpy().reshape(B * H, dk, dv), rS2) <= tol
