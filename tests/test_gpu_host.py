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


def _host_inputs(seed, B=2, T=130, H=2, dk=128, dv=128):
    inp = W.draw(B, T, H, dk, dv, seed=seed, dtype=torch.bfloat16, s0_std=0.05)
    names = ("q", "k", "v", "log_alpha", "b", "w")
    return {n: inp[n].pin_memory() for n in names}, inp["S0"].pin_memory(), names


def _device_ref(g, host, s0, names):
    od, sd = g.chunk_fwd(*(host[n].cuda() for n in names), s0.cuda())
    torch.cuda.synchronize()
    return od.cpu(), sd.cpu()


def test_host_entry_reuses_one_workspace(g):
    """Two calls in a row on one stream and one workspace, different inputs:
    the second must not see the first's data."""
    a, s0a, names = _host_inputs(9700)
    b, s0b, _ = _host_inputs(9701)
    ws = torch.empty(g.chunk_fwd_host_workspace_bytes(2, 130, 2, 128, 128, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    oa, sa = g.chunk_fwd_host(*(a[n] for n in names), s0a, workspace=ws, stream=stream)
    ob, sb = g.chunk_fwd_host(*(b[n] for n in names), s0b, workspace=ws, stream=stream)
    stream.synchronize()
    for (o, S), (host, s0) in (((oa, sa), (a, s0a)), ((ob, sb), (b, s0b))):
        ro, rs = _device_ref(g, host, s0, names)
        assert torch.equal(o, ro) and torch.equal(S, rs)


def test_host_entry_interleaved_streams(g):
    """Calls on two streams with two workspaces, interleaved: the helper
    streams are shared per device, the results must still be exact."""
    ins = [_host_inputs(9710 + i) for i in range(4)]
    names = ins[0][2]
    need = g.chunk_fwd_host_workspace_bytes(2, 130, 2, 128, 128, torch.bfloat16)
    wss = [torch.empty(need, dtype=torch.uint8, device="cuda") for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for i, (host, s0, _) in enumerate(ins):
        outs.append(g.chunk_fwd_host(*(host[n] for n in names), s0, workspace=wss[i % 2],
                                     stream=streams[i % 2]))
    for st in streams:
        st.synchronize()
    assert g.device_status() == 0
    for (o, S), (host, s0, _) in zip(outs, ins):
        ro, rs = _device_ref(g, host, s0, names)
        assert torch.equal(o, ro) and torch.equal(S, rs)


def test_host_entry_rejects_stream_on_other_device(g):
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two devices")
    a, s0a, names = _host_inputs(9720)
    with pytest.raises(ValueError, match="stream"):
        g.chunk_fwd_host(*(a[n] for n in names), s0a, stream=torch.cuda.Stream(device=1))
