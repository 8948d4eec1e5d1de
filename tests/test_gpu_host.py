"""gdn2_chunk_fwd_host (host buffers, copies pipelined with the kernel by the
library) against gdn2_chunk_fwd on device copies of the same inputs.  Both
run the same kernels on the same sequences, so o and S_T must match bit for
bit; the device path itself is checked against the oracle elsewhere."""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_92_b200 as g
    g.lib()
    return g


CASES = [  # B, T, H, d_k, d_v, dtype, with S0, pinned
    (3, 130, 2, 128, 128, torch.bfloat16, True, True),
    (2, 70, 2, 64, 128, torch.float32, False, True),
    (1, 200, 1, 128, 256, torch.bfloat16, True, False),
    (70, 64, 1, 64, 64, torch.bfloat16, True, True),       # more sequences than slices
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}dk{c[3]}dv{c[4]}{str(c[5])[6:]}"
                                                        f"{'_s0' if c[6] else ''}{'_pinned' if c[7] else ''}")
def test_host_entry_matches_device_entry(g, case):
    B, T, H, dk, dv, dt, with_s0, pinned = case
    inp = W.draw(B, T, H, dk, dv, seed=9500 + B + T, dtype=dt, s0_std=0.05 if with_s0 else None)
    names = ("q", "k", "v", "log_alpha", "b", "w")
    host = {n: (inp[n].pin_memory() if pinned else inp[n].contiguous()) for n in names}
    s0 = inp["S0"]
    s0h = (s0.pin_memory() if pinned else s0) if s0 is not None else None
    stream = torch.cuda.Stream()
    oh, sh = g.chunk_fwd_host(*(host[n] for n in names), s0h, stream=stream)
    stream.synchronize()
    assert g.device_status() == 0
    d = {n: inp[n].cuda() for n in names}
    od, sd = g.chunk_fwd(*(d[n] for n in names), s0.cuda() if s0 is not None else None)
    torch.cuda.synchronize()
    assert torch.equal(oh, od.cpu())
    assert torch.equal(sh, sd.cpu())


def test_host_entry_empty_sequence(g):
    inp = W.draw(2, 1, 2, 64, 64, seed=9600, dtype=torch.bfloat16, s0_std=0.05)
    e = {n: inp[n][:, :0].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")}
    o, S = g.chunk_fwd_host(e["q"], e["k"], e["v"], e["log_alpha"], e["b"], e["w"], inp["S0"])
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(S, inp["S0"])
    o, S = g.chunk_fwd_host(e["q"], e["k"], e["v"], e["log_alpha"], e["b"], e["w"], None)
    assert torch.count_nonzero(S) == 0
