"""Fault injection on the host (gdn2_testing_fail_launches): a kernel launch
site returns GDN2_ERR_CUDA without launching, as a launch the driver refused
would.  Nothing faults on the device.  Checked: the status reaches the caller
(Gdn2Error), nothing is left half-done that should not be (a decode state is
untouched; in the pipelined host-buffer call the slices before the failure are
complete and the later ones untouched, and the call's work stays ordered on
its stream), and the next call on the same buffers is exact to the bit.
"""
import pytest
import torch

import workloads as W
from gpu_util import to_dev

pytestmark = pytest.mark.gpu

CUDA_ERR = 4   # GDN2_ERR_CUDA


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_92_b200 as g
    g.lib()
    yield g
    g.testing_fail_launches(0, 0)


def _raises_cuda(g, fn):
    with pytest.raises(g.Gdn2Error) as e:
        fn()
    assert e.value.status == CUDA_ERR
    g.testing_fail_launches(0, 0)


@pytest.mark.parametrize("dtype,chunk", [(torch.bfloat16, 64), (torch.float32, 64), (torch.bfloat16, 32)])
def test_injected_failure_device_path(g, dtype, chunk):
    d = to_dev(W.draw(2, 130, 2, 128, 128, seed=41, dtype=dtype, s0_std=0.05))
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    o_ref, s_ref = g.chunk_fwd(*args, chunk=chunk)
    torch.cuda.synchronize()
    g.testing_fail_launches(0, 1)
    _raises_cuda(g, lambda: g.chunk_fwd(*args, chunk=chunk))
    o, s = g.chunk_fwd(*args, chunk=chunk)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)


def test_injected_failure_of_the_separate_epilogue_pass(g):
    # d_v = 256 with the gated RMS norm: the chunk kernel, then the norm as a pass of its own
    d = to_dev(W.draw_raw(1, 100, 2, 128, 256, seed=42, s0_std=0.05))
    def call():
        return g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], prep=True,
                              gate=d["gate"], norm_weight=d["norm_weight"])
    o_ref, s_ref = call()
    torch.cuda.synchronize()
    g.testing_fail_launches(1, 1)   # the chunk kernel runs, the norm pass is refused
    _raises_cuda(g, call)
    o, s = call()
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)


@pytest.mark.parametrize("fused", [False, True])
def test_injected_failure_leaves_decode_state_untouched(g, fused):
    d = to_dev(W.draw_raw(3, None, 2, 128, 128, seed=43, steps=2, s0_std=0.05))
    kw = dict(prep=True, gate=d["gate"][0], norm_weight=d["norm_weight"]) if fused else {}
    S = d["S0"].clone()
    S_before = S.clone()
    g.testing_fail_launches(0, 1)
    _raises_cuda(g, lambda: g.decode_step_ex(d["q"][0], d["k"][0], d["v"][0], d["log_alpha"][0], d["b"][0],
                                             d["w"][0], S, **kw))
    torch.cuda.synchronize()
    assert torch.equal(S, S_before)
    o = g.decode_step_ex(d["q"][0], d["k"][0], d["v"][0], d["log_alpha"][0], d["b"][0], d["w"][0], S, **kw)
    S_ref = S_before.clone()
    o_ref = g.decode_step_ex(d["q"][0], d["k"][0], d["v"][0], d["log_alpha"][0], d["b"][0], d["w"][0], S_ref, **kw)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


def test_injected_failure_qed(g):
    d = to_dev(W.draw(1, 100, 2, 128, 128, seed=44, s0_std=0.05))
    c = W.draw_qed_gate((1, 100, 2), 128, seed=45).cuda()
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["b"], c, d["w"], d["S0"])
    g.testing_fail_launches(0, 1)
    _raises_cuda(g, lambda: g.chunk_fwd_qed(*args))
    S = d["S0"].clone()
    tok = {n: d[n][:, 0].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")}
    g.testing_fail_launches(0, 1)
    _raises_cuda(g, lambda: g.decode_step_qed(tok["q"], tok["k"], tok["v"], tok["log_alpha"], tok["b"],
                                              c[:, 0].contiguous(), tok["w"], S))
    torch.cuda.synchronize()
    assert torch.equal(S, d["S0"])


def test_injected_failure_mid_host_pipeline(g):
    # four sequences: four slices of one sequence each; the third slice's launch is refused
    B, T, H = 4, 150, 2
    d = W.draw(B, T, H, 128, 128, seed=46, s0_std=0.05)
    hp = {n: t.pin_memory() for n, t in d.items()}
    args = (hp["q"], hp["k"], hp["v"], hp["log_alpha"], hp["b"], hp["w"], hp["S0"])
    ref = to_dev(d)
    o_ref, s_ref = g.chunk_fwd(ref["q"], ref["k"], ref["v"], ref["log_alpha"], ref["b"], ref["w"], ref["S0"])
    o_ref, s_ref = o_ref.cpu(), s_ref.cpu()
    ws = torch.empty(g.chunk_fwd_host_workspace_bytes(B, T, H, 128, 128, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    o = torch.zeros_like(hp["v"]).pin_memory()
    S_T = torch.zeros_like(hp["S0"]).pin_memory()
    g.testing_fail_launches(2, 1)
    _raises_cuda(g, lambda: g.chunk_fwd_host(*args, o=o, S_T=S_T, workspace=ws))
    torch.cuda.synchronize()   # the call's copies are ordered on the current stream
    assert torch.equal(o[:2], o_ref[:2]) and torch.equal(S_T[:2], s_ref[:2])   # slices before the failure
    assert not o[2:].any() and not S_T[2:].any()                                # the rest untouched
    o2, s2 = g.chunk_fwd_host(*args, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o2, o_ref) and torch.equal(s2, s_ref)
