"""GPU parity of the fused input prep and output epilogue (the _ex entry
points) against the fp64 oracle's prep -> recurrence -> epilogue on the same
seeded raw inputs.

Bar as for the plain path, per output (the stored o -- y when the epilogue
is on -- and the final state): max |gpu - oracle| <= tol * max |oracle|,
tol = 1e-4 (fp32 I/O), 2e-2 (bf16 I/O).
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


def _oracle(inp, heads, prep, neg, epi, l2_eps):
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                          S0=inp["S0"], heads=heads, prep=prep, allow_neg_eigval=neg, l2_eps=l2_eps,
                          gate=inp["gate"] if epi else None,
                          norm_weight=inp["norm_weight"] if epi else None, norm_eps=1e-5)


def _check(g, fn, inp, *, prep, neg, epi, heads=None, l2_eps=1e-6):
    B, T, H, _ = inp["q"].shape
    heads = list(range(B * H)) if heads is None else heads
    d = to_dev(inp)
    o, S_T = fn(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], prep=prep,
                allow_neg_eigval=neg, l2_eps=l2_eps, gate=d["gate"] if epi else None,
                norm_weight=d["norm_weight"] if epi else None, norm_eps=1e-5)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ro, rS = _oracle(inp, heads, prep, neg, epi, l2_eps)
    tol = TOL[inp["q"].dtype]
    eo = rel_inf(heads_of(o, heads, H), ro)
    es = rel_inf(state_heads(S_T, heads, H), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S_T err {es:.3e} (tol {tol})"
    return eo, es


CASES = [  # B, T, H, d_k, d_v, dtype   (ragged T: a partial last chunk)
    (2, 200, 2, 128, 128, torch.bfloat16),   # tensor cores, epilogue inside the kernel
    (1, 130, 2, 64, 64, torch.bfloat16),     # tensor cores, d_v = 64 slices
    (1, 150, 2, 128, 256, torch.bfloat16),   # tensor cores, epilogue as its own pass
    (1, 100, 2, 64, 192, torch.bfloat16),    # tensor cores, mixed slices
    (1, 160, 2, 64, 64, torch.float32),      # CUDA cores (fp32 I/O)
    (2, 96, 2, 128, 128, torch.float32),
]
MODES = [  # prep, neg_eigval, epilogue
    (True, False, False),
    (True, True, True),
    (False, False, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}dk{c[3]}dv{c[4]}{str(c[5])[6:]}")
@pytest.mark.parametrize("mode", MODES, ids=lambda m: f"prep{int(m[0])}neg{int(m[1])}epi{int(m[2])}")
def test_chunk_fused(g, case, mode):
    B, T, H, dk, dv, dt = case
    prep, neg, epi = mode
    inp = W.draw_raw(B, T, H, dk, dv, seed=5000 + T + dk, dtype=dt, qk_scale=2.0, s0_std=0.05)
    if not prep:   # the epilogue alone takes prepared inputs
        inp.update(W.draw(B, T, H, dk, dv, seed=5100 + T, dtype=dt, s0_std=0.05))
    _check(g, g.chunk_fwd_ex, inp, prep=prep, neg=neg, epi=epi)


def test_chunk_fused_zero_l2_eps_and_zero_rows(g):
    """l2_eps = 0 with some all-zero q and k rows (they stay zero) and a partial last chunk."""
    inp = W.draw_raw(1, 100, 2, 128, 128, seed=5200, dtype=torch.bfloat16, s0_std=0.05)
    inp["q"][0, 7] = 0
    inp["k"][0, 70] = 0
    _check(g, g.chunk_fwd_ex, inp, prep=True, neg=False, epi=True, l2_eps=0.0)


def test_chunk_fused_flags_zero_is_plain_forward(g):
    inp = W.draw(1, 192, 2, 128, 128, seed=5300, dtype=torch.bfloat16, s0_std=0.05)
    d = to_dev(inp)
    o1, S1 = g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    o2, S2 = g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_chunk_fused_headline_size_sampled(g):
    """B8 T4096 H16 d128 with prep and epilogue, on a sample of heads."""
    inp = W.draw_raw(8, 4096, 16, 128, 128, seed=5400, dtype=torch.bfloat16, qk_scale=2.0)
    heads = [0, 37, 64, 127]
    _check(g, g.chunk_fwd_ex, inp, prep=True, neg=False, epi=True, heads=heads)


def _decode_run(g, inp, steps, prep, neg, epi):
    d = to_dev(inp)
    S = d["S0"].clone()
    outs = []
    for s in range(steps):
        outs.append(g.decode_step_ex(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s],
                                     d["w"][s], S, prep=prep, allow_neg_eigval=neg,
                                     gate=d["gate"][s] if epi else None,
                                     norm_weight=d["norm_weight"] if epi else None))
    torch.cuda.synchronize()
    assert g.device_status() == 0
    return torch.stack(outs), S


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("dv", [64, 128, 256, 192], ids=lambda x: f"dv{x}")
@pytest.mark.parametrize("mode", MODES, ids=lambda m: f"prep{int(m[0])}neg{int(m[1])}epi{int(m[2])}")
def test_decode_fused(g, dt, dv, mode):
    """d_v = 256 and 192 split the row over 2 and 3 CTAs (a thread-block cluster)."""
    prep, neg, epi = mode
    B, H, dk, steps = 3, 2, 128, 6
    inp = W.draw_raw(B, None, H, dk, dv, seed=5500 + dv, dtype=dt, qk_scale=2.0, s0_std=0.05, steps=steps)
    if not prep:
        p = W.draw(steps, B, H, dk, dv, seed=5600 + dv, dtype=dt)   # [steps, B, H, d]
        for n in ("q", "k", "b", "w"):
            inp[n] = p[n]
    o, S = _decode_run(g, inp, steps, prep, neg, epi)
    ro, rS = oracle.decode_steps(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                                 inp["S0"], prep=prep, allow_neg_eigval=neg,
                                 gate=inp["gate"] if epi else None,
                                 norm_weight=inp["norm_weight"] if epi else None)
    heads = list(range(B * H))
    got = np.stack([o[:, h // H, h % H, :].float().cpu().numpy() for h in heads])
    tol = TOL[dt]
    eo = rel_inf(got, ro)
    es = rel_inf(state_heads(S, heads, H), rS)
    assert eo <= tol and es <= tol, f"o err {eo:.3e}, S err {es:.3e} (tol {tol})"
