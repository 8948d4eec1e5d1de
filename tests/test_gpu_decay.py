"""GPU parity under strong decay: every chunk kernel and its fused, packed
and value-head variants against the fp64 oracle when log_alpha is far from 0.

The recurrence (burn-gdn2 README, "Architecture": diag(alpha_t) with alpha a
per-channel decay) puts no lower bound on alpha, so the chunked kernels must
stay exact for any log_alpha <= 0.  Decay regimes exercised:
  * alpha ~ U[0.05, 0.5]: about 130 (log2) of decay per chunk, inside the
    tensor-core form's own range (it keeps its operands within 2^(+-100));
  * mixed channels: even key channels alpha ~ 1e-3, odd ones ~ 0.999, so every
    chunk passes that range and runs token by token, while the slow channels
    still carry information across chunks;
  * spikes: single tokens with log_alpha = -20 on every channel;
  * a burst of strong decay in the middle of a sequence, so a sequence starts
    chunked and is finished token by token from that chunk on;
  * resets: single tokens with log_alpha = -inf (alpha = 0: the state is
    cleared before the token's own write).
Bar as for the other parity tests: max |gpu - oracle| <= tol * max |oracle| for
the stored output and the final state, tol = 1e-4 (fp32 I/O), 2e-2 (bf16 I/O).
"""
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


def _decay(inp, kind, seed):
    """Apply one decay regime to drawn inputs (log_alpha only)."""
    T = inp["log_alpha"].shape[1]
    if kind == "alpha_005_05":
        u = torch.rand(inp["log_alpha"].shape, generator=torch.Generator().manual_seed(seed))
        out = dict(inp)
        out["log_alpha"] = torch.log(0.05 + 0.45 * u).to(inp["log_alpha"].dtype).contiguous()
        return out
    if kind == "mixed":
        return W.with_mixed_decay(inp, seed)
    if kind == "spikes":
        return W.with_decay_spikes(inp, seed, prob=0.03, value=-20.0)
    if kind == "reset":
        return W.with_decay_spikes(inp, seed, prob=0.02, value=float("-inf"))
    if kind == "burst":   # 10 tokens of log_alpha = -12 starting inside chunk 2 (or late in a short T)
        t0 = min(140, max(0, T - 30))
        return W.with_decay_burst(inp, t0, t0 + 10, -12.0)
    raise ValueError(kind)


DECAYS = ["alpha_005_05", "mixed", "spikes", "reset", "burst"]


def _check_plain(g, fn, inp, chunk=64):
    B, T, H, _ = inp["q"].shape
    heads = list(range(B * H))
    d = to_dev(inp)
    o, S_T = fn(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], chunk=chunk)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                            S0=inp["S0"], heads=heads)
    tol = TOL[inp["q"].dtype]
    eo = rel_inf(heads_of(o, heads, H), ro)
    es = rel_inf(state_heads(S_T, heads, H), rS)
    assert np.isfinite(eo) and np.isfinite(es)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S_T err {es:.3e} (tol {tol})"


TC_SHAPES = [  # B, T, H, d_k, d_v  (bf16, chunk 64: the tensor-core kernel)
    (2, 300, 2, 128, 128),
    (1, 256, 2, 64, 64),
    (1, 200, 1, 128, 256),
    (2, 130, 2, 64, 128),
]


@pytest.mark.parametrize("shape", TC_SHAPES, ids=lambda s: "B%dT%dH%dk%dv%d" % s)
@pytest.mark.parametrize("kind", DECAYS)
def test_tensor_core_chunk_strong_decay(g, shape, kind):
    B, T, H, dk, dv = shape
    inp = W.draw(B, T, H, dk, dv, seed=8100 + T + dk + dv, dtype=torch.bfloat16, s0_std=0.05, b_scale=2.0)
    _check_plain(g, g.chunk_fwd, _decay(inp, kind, 8200 + T))


CC_CASES = [  # B, T, H, d_k, d_v, dtype, chunk  (the CUDA-core kernel)
    (1, 256, 2, 64, 64, torch.float32, 64),
    (2, 100, 1, 128, 128, torch.float32, 64),
    (1, 150, 2, 128, 64, torch.bfloat16, 16),
    (1, 150, 2, 64, 128, torch.bfloat16, 32),
]


@pytest.mark.parametrize("case", CC_CASES, ids=lambda c: "B%dT%dH%dk%dv%d%sc%d" % (*c[:5], str(c[5])[6:], c[6]))
@pytest.mark.parametrize("kind", DECAYS)
def test_cuda_core_chunk_strong_decay(g, case, kind):
    B, T, H, dk, dv, dt, chunk = case
    inp = W.draw(B, T, H, dk, dv, seed=8300 + T + dk + dv, dtype=dt, s0_std=0.05, b_scale=2.0)
    _check_plain(g, g.chunk_fwd_cuda_core, _decay(inp, kind, 8400 + T), chunk=chunk)


@pytest.mark.parametrize("kind", DECAYS)
def test_tensor_core_handoff_positions(g, kind):
    """The token tail taking over at the first chunk, a middle one and the last one."""
    for t0 in (0, 64 * 3 + 5, 64 * 6 + 40):
        inp = W.draw(1, 64 * 7, 2, 128, 128, seed=8500 + t0, dtype=torch.bfloat16, s0_std=0.05)
        inp = W.with_decay_burst(inp, t0, t0 + 12, -15.0)
        if kind != "burst":
            inp = _decay(inp, kind, 8600 + t0)
        _check_plain(g, g.chunk_fwd, inp)


FUSED = [  # B, T, H, d_k, d_v, dtype: tensor cores (epilogue in kernel / own pass), CUDA cores
    (1, 200, 2, 128, 128, torch.bfloat16),
    (1, 150, 1, 128, 256, torch.bfloat16),
    (1, 130, 2, 64, 64, torch.bfloat16),
    (1, 160, 2, 64, 64, torch.float32),
]


@pytest.mark.parametrize("case", FUSED, ids=lambda c: "B%dT%dH%dk%dv%d%s" % (*c[:5], str(c[5])[6:]))
@pytest.mark.parametrize("kind", DECAYS)
def test_fused_strong_decay(g, case, kind):
    B, T, H, dk, dv, dt = case
    inp = _decay(W.draw_raw(B, T, H, dk, dv, seed=8700 + T + dv, dtype=dt, qk_scale=2.0, s0_std=0.05),
                 kind, 8800 + T)
    heads = list(range(B * H))
    d = to_dev(inp)
    o, S_T = g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], prep=True,
                            allow_neg_eigval=True, gate=d["gate"], norm_weight=d["norm_weight"], norm_eps=1e-5)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], S0=inp["S0"],
                            heads=heads, prep=True, allow_neg_eigval=True, gate=inp["gate"],
                            norm_weight=inp["norm_weight"], norm_eps=1e-5)
    tol = TOL[dt]
    eo, es = rel_inf(heads_of(o, heads, H), ro), rel_inf(state_heads(S_T, heads, H), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S_T err {es:.3e} (tol {tol})"


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("kind", DECAYS)
def test_packed_value_heads_strong_decay(g, dt, kind):
    """Packed sequences (lengths 0, 1, 65, 200, 130) with two value heads per key head."""
    lens = [65, 0, 200, 1, 130]
    N, H, HV, dk, dv = len(lens), 2, 4, 128, 128
    cu = W.cu_seqlens_of(lens)
    T = int(cu[-1])
    inp = _decay(W.draw(1, T, H, dk, dv, seed=8900, dtype=dt, HV=HV, b_scale=2.0), kind, 8901)
    inp["S0"] = 0.05 * torch.randn(N, HV, dk, dv, generator=torch.Generator().manual_seed(8902))
    d = to_dev(inp)
    o, S_T = g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"],
                            cu_seqlens=cu.cuda())
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ro, rS = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                            S0=inp["S0"], cu_seqlens=cu.numpy())
    got = [o[0, int(cu[x // HV]):int(cu[x // HV + 1]), x % HV].float().cpu().numpy() for x in range(N * HV)]
    scale = max(float(np.max(np.abs(r))) for r in ro if r.size)
    eo = max((float(np.max(np.abs(a - r))) for a, r in zip(got, ro) if r.size), default=0.0) / scale
    es = rel_inf(S_T.double().cpu().numpy().reshape(N * HV, dk, dv), rS)
    tol = TOL[dt]
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S_T err {es:.3e} (tol {tol})"


@pytest.mark.parametrize("case", [(1, 100, 2, 64, 64, torch.float32), (1, 150, 2, 128, 128, torch.bfloat16)],
                         ids=["f32", "bf16"])
@pytest.mark.parametrize("kind", DECAYS)
def test_qed_chunk_strong_decay(g, case, kind):
    B, T, H, dk, dv, dt = case
    inp = _decay(W.draw(B, T, H, dk, dv, seed=9000 + T, dtype=dt, s0_std=0.05), kind, 9001)
    inp["c"] = W.draw_qed_gate((B, T, H), dk, seed=9002, dtype=dt)
    d = to_dev(inp)
    o, S = g.chunk_fwd_qed(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["c"], d["w"], d["S0"])
    torch.cuda.synchronize()
    assert g.device_status() == 0
    heads = list(range(B * H))
    ro, rS = oracle.forward_qed(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["c"], inp["w"],
                                S0=inp["S0"], heads=heads)
    got = np.stack([o[x // H, :, x % H].float().cpu().numpy() for x in heads])
    gS = np.stack([S[x // H, x % H].double().cpu().numpy() for x in heads])
    tol = TOL[dt]
    eo, es = rel_inf(got, ro), rel_inf(gS, rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S err {es:.3e} (tol {tol})"


@pytest.mark.parametrize("kind", DECAYS)
def test_decode_strong_decay(g, kind):
    """The decode step applies exp(log_alpha) per token; it stays exact too."""
    B, H, steps, dk, dv = 3, 2, 40, 128, 128
    inp = _decay(W.draw(B, steps, H, dk, dv, seed=9100, dtype=torch.bfloat16, s0_std=0.3, b_scale=2.0),
                 kind, 9101)
    for n in ("q", "k", "v", "log_alpha", "b", "w"):
        inp[n] = inp[n].transpose(0, 1).contiguous()
    d = to_dev(inp)
    S = d["S0"].clone()
    outs = [g.decode_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s], d["w"][s], S).clone()
            for s in range(steps)]
    torch.cuda.synchronize()
    o = torch.stack(outs)
    ro, rS = oracle.decode_steps(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], inp["S0"])
    go = np.stack([o[:, n // H, n % H, :].float().cpu().numpy() for n in range(B * H)])
    assert rel_inf(go, ro) <= TOL[torch.bfloat16]
    assert rel_inf(state_heads(S, range(B * H), H), rS) <= TOL[torch.bfloat16]
