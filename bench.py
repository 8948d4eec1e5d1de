#!/usr/bin/env python
"""Benchmark of the B200 Gated DeltaNet-2 mixer (chunk forward + decode).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one chunk-forward call over the headline workload
(B8 T4096 H16 d_k=d_v=128, chunk 64, bf16 I/O, fp32 state: the burn-gdn2
default configuration of 16 heads x head_dim 128, hidden 2048), inputs
resident in HBM (948 MB, larger than the 126 MB L2, so no flush is needed).
`value` is tokens/s over all ranks (a token = one (b, t) position through all
16 heads), timed on the device with CUDA events, max over ranks.  The same
JSON line carries:
  e2e          the same metric through the host-buffer C-ABI entry
               (gdn2_chunk_fwd_host) on pinned host buffers: every step
               copies the inputs in and o, S_T out, the library overlapping
               the copies of one slice of sequences with the kernel of the next;
  roofline     the chunk kernel's algorithmic HBM bytes / launch time vs the
               measured copy bandwidth, the tensor-pipe fraction of its useful
               FLOPs, and the attainable fraction max(t_flop, t_byte) / t;
  steady       after the K timed steps, rounds of 50 calls over at least
               0.5 s (per-call median, min, max), under the same clock sampler;
  decode       tokens/s of the decode workload (256 sequences x 16 heads x
               d128, 1024 consecutive steps) with its own HBM roofline, timed
               as plain launches and as one captured CUDA graph;
  expanded_v   the d_v=256, b in (0,2) chunk workload;
  cpu_baseline the fp64 oracle on the host cores over a bounded sample.
With torchrun (N > 1) every rank runs its own batch (weak scaling, no
collective on the data path); only the barrier and the max-over-ranks time
reduction use NCCL.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

HEADLINE = "chunk_bf16_h2048"
METRIC = "GDN-2 chunk-fwd tokens/s and decode tokens/s at 1 B200; % of roofline"


# ------------------------------------------------------------ accounting
def chunk_bytes(wl, with_s0: bool, with_st: bool = True) -> int:
    """Algorithmic HBM bytes of one chunk-forward launch: every input read
    once, o written once, the fp32 state read (S0) / written (S_T) once."""
    io = 4 if wl.io == "f32" else 2
    tok = wl.B * wl.T * wl.H * (4 * wl.d_k + 3 * wl.d_v) * io
    st = wl.B * wl.H * wl.d_k * wl.d_v * 4
    return tok + st * (int(with_s0) + int(with_st))


def chunk_flops(wl) -> float:
    """Useful FLOPs of the chunk form per launch (triangles counted half):
    per token-head C(3 d_k + 2 d_v) + C^2/3 + 6 d_k d_v."""
    C = wl.chunk
    per = C * (3 * wl.d_k + 2 * wl.d_v) + C * C / 3 + 6 * wl.d_k * wl.d_v
    return per * wl.B * wl.T * wl.H


def decode_bytes(wl) -> int:
    io = 4 if wl.io == "f32" else 2
    return wl.B * wl.H * ((4 * wl.d_k + 3 * wl.d_v) * io + 2 * wl.d_k * wl.d_v * 4)


def measured_traffic(kernel: str, batch: int):
    """DRAM bytes per launch from the committed ncu capture in
    profiles/traffic.json, scaled to `batch`; None if the kernel sources have
    changed since that capture (digest mismatch) or no capture exists."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if rec is None:
        return None
    h = hashlib.sha256()
    for src in rec["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != rec["digest"]:
        return None
    return (rec["dram_bytes_read"] + rec["dram_bytes_write"]) * batch / rec["case_batch"]


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# --------------------------------------------------------------- clocks
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""

    def __init__(self, period_s: float = 0.005):
        self.period = period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            props = torch.cuda.get_device_properties(torch.cuda.current_device())
            try:
                bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _reasons(self):
        nv = self._nv
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(nv, fn):
                return int(getattr(nv, fn)(self._h))
        return 0

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                self.reasons |= self._reasons()
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self) -> dict:
        names = sorted(n for bit, n in REASONS.items() if self.reasons & bit and n != "gpu_idle")
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------- timing
def device_time_ms(fn, steps: int, stream) -> float:
    """Time `steps` calls of fn on `stream` with CUDA events (ms total)."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Max of a per-rank scalar over all ranks (NCCL on cuda, gloo on cpu)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wl, rank: int) -> int:
    """Each rank draws its own batch of the workload (weak scaling)."""
    return wl.seed + 100 * rank


def aggregate_throughput(ms_local: float, steps: int, tokens_per_rank_step: int, world: int,
                         device: str = "cuda"):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    ms_max = max_over_ranks(ms_local, world, device)
    return tokens_per_rank_step * world * steps / (ms_max / 1e3), ms_max


# ------------------------------------------------------- our measurements
def nvtx(name: str):
    """An NVTX range around one phase of the harness (visible to nsys / ncu
    range filters; a no-op without a profiler attached)."""
    return torch.cuda.nvtx.range(name)


def steady_rounds(step, stream, min_s: float = 0.5, per_round: int = 50, max_rounds: int = 400):
    """Rounds of `per_round` back-to-back calls, each timed with CUDA events on
    `stream`, until `min_s` of device time has been covered; returns the
    per-call median, min and max over the rounds (ms) and the time covered (s)."""
    per, total = [], 0.0
    while total < min_s * 1e3 and len(per) < max_rounds:
        ms = device_time_ms(step, per_round, stream)
        per.append(ms / per_round)
        total += ms
    return {"rounds": len(per), "calls_per_round": per_round, "ms_per_call_median": statistics.median(per),
            "ms_per_call_min": min(per), "ms_per_call_max": max(per), "seconds": total / 1e3}


def bench_chunk(g, wl, steps, warmup, rank, world, stream, sampler=None, steady_s: float = 0.0):
    d = W.make_chunk_inputs(wl, seed=rank_seed(wl, rank), device="cuda")
    o = torch.empty_like(d["v"])
    S_T = torch.empty(wl.B, wl.H, wl.d_k, wl.d_v, dtype=torch.float32, device="cuda")

    def step():
        g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], o=o, S_T=S_T,
                    stream=stream)

    with nvtx("warm-up " + wl.name), torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    steady = None
    if sampler is not None:
        # the sampler covers the timed steps and the steady rounds after them
        with sampler:
            with nvtx("timed " + wl.name):
                ms = device_time_ms(step, steps, stream)
            torch.cuda.synchronize()
            barrier(world)
            if steady_s > 0:
                with nvtx("steady rounds " + wl.name):
                    steady = steady_rounds(step, stream, steady_s)
    else:
        with nvtx("timed " + wl.name):
            ms = device_time_ms(step, steps, stream)
        torch.cuda.synchronize()
        barrier(world)
    if g.device_status() != 0:
        raise RuntimeError("chunk kernel reported a device timeout")
    if sampler is not None:
        return ms, d, o, S_T, steady
    return ms, d, o, S_T


def bench_chunk_fused(g, wl, steps, warmup, rank, stream):
    """The workload's shapes from raw projections: fused input prep (L2 norm of
    q, k; sigmoid gates) and the gated RMS-norm epilogue in the same call."""
    d = W.draw_raw(wl.B, wl.T, wl.H, wl.d_k, wl.d_v, seed=rank_seed(wl, rank) + 7, dtype=wl.torch_dtype,
                   alpha_lo=wl.alpha_lo, alpha_hi=wl.alpha_hi, qk_scale=2.0, s0_std=wl.s0_std, device="cuda")
    o = torch.empty_like(d["v"])
    S_T = torch.empty(wl.B, wl.H, wl.d_k, wl.d_v, dtype=torch.float32, device="cuda")

    def step():
        g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], prep=True,
                       gate=d["gate"], norm_weight=d["norm_weight"], o=o, S_T=S_T, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    torch.cuda.synchronize()
    ms = device_time_ms(step, steps, stream)
    if g.device_status() != 0:
        raise RuntimeError("fused chunk kernel reported a device timeout")
    return ms / steps


def bench_chunk_general(g, wl, steps, rank, stream, *, H=None, HV=None, lengths=None):
    """chunk_fwd_ex on the workload's shapes with H key heads and HV value heads
    (defaults: the workload's H), optionally as packed sequences of the given
    lengths (their sum replaces B x T).  Returns (ms per call, bytes per call)."""
    H = wl.H if H is None else H
    HV = H if HV is None else HV
    if lengths is None:
        Bt, T, N = wl.B, wl.T, wl.B
        cu = None
    else:
        cu_h = W.cu_seqlens_of(lengths)
        Bt, T, N = 1, int(cu_h[-1]), len(lengths)
        cu = cu_h.to("cuda")
    d = W.draw(Bt, T, H, wl.d_k, wl.d_v, seed=rank_seed(wl, rank) + 11, dtype=wl.torch_dtype,
               alpha_lo=wl.alpha_lo, alpha_hi=wl.alpha_hi, b_scale=wl.b_scale, HV=HV, device="cuda")
    o = torch.empty_like(d["v"])
    S_T = torch.empty(N, HV, wl.d_k, wl.d_v, dtype=torch.float32, device="cuda")

    def step():
        g.chunk_fwd_ex(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], None, cu_seqlens=cu,
                       o=o, S_T=S_T, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
    torch.cuda.synchronize()
    ms = device_time_ms(step, steps, stream)
    if g.device_status() != 0:
        raise RuntimeError("chunk kernel reported a device error")
    io = 2 if wl.io == "bf16" else 4
    nbytes = Bt * T * (H * 4 * wl.d_k + HV * 3 * wl.d_v) * io + N * HV * wl.d_k * wl.d_v * 4
    return ms / steps, nbytes, Bt * T


def bench_chunk_decay(g, wl, steps, rank, stream, kind):
    """The headline shape under strong decay: alpha ~ U[0.05, 0.5] (about 130 log2
    units per chunk, still inside the tensor-core form's range) or mixed channels
    (even ones alpha ~ 1e-3: every chunk runs token by token)."""
    d = W.make_chunk_inputs(wl, seed=rank_seed(wl, rank) + 23, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(rank_seed(wl, rank) + 24)
    u = torch.rand(d["log_alpha"].shape, generator=gen, device="cuda")
    if kind == "alpha_005_05":
        la = torch.log(0.05 + 0.45 * u)
    else:
        even = (torch.arange(wl.d_k, device="cuda") % 2 == 0)
        la = torch.where(even, torch.log(5e-4 + 1.5e-3 * u), torch.log(0.99 + 0.0099 * u))
    d["log_alpha"] = la.to(d["log_alpha"].dtype).contiguous()
    o = torch.empty_like(d["v"])
    S_T = torch.empty(wl.B, wl.H, wl.d_k, wl.d_v, dtype=torch.float32, device="cuda")

    def step():
        g.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], o=o, S_T=S_T, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(2):
            step()
    torch.cuda.synchronize()
    ms = device_time_ms(step, steps, stream)
    if g.device_status() != 0:
        raise RuntimeError("chunk kernel reported a device error")
    return ms / steps


def bench_chunk_qed(g, wl, steps, rank, stream):
    """The workload's shapes through the second, query-derived erase (CUDA cores)."""
    d = W.draw(wl.B, wl.T, wl.H, wl.d_k, wl.d_v, seed=rank_seed(wl, rank) + 17, dtype=wl.torch_dtype,
               alpha_lo=wl.alpha_lo, alpha_hi=wl.alpha_hi, s0_std=wl.s0_std, device="cuda")
    c = W.draw_qed_gate((wl.B, wl.T, wl.H), wl.d_k, seed=rank_seed(wl, rank) + 18, dtype=wl.torch_dtype,
                        device="cuda")
    o = torch.empty_like(d["v"])
    S_T = torch.empty(wl.B, wl.H, wl.d_k, wl.d_v, dtype=torch.float32, device="cuda")

    def step():
        g.chunk_fwd_qed(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], c, d["w"], d["S0"], o=o, S_T=S_T,
                        stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(2):
            step()
    torch.cuda.synchronize()
    ms = device_time_ms(step, steps, stream)
    if g.device_status() != 0:
        raise RuntimeError("QED chunk kernel reported a device error")
    return ms / steps


def bench_decode_qed(g, wl, steps, rank, stream):
    d = W.draw(steps, wl.B, wl.H, wl.d_k, wl.d_v, seed=rank_seed(wl, rank) + 19, dtype=wl.torch_dtype,
               device="cuda")
    c = W.draw_qed_gate((steps, wl.B, wl.H), wl.d_k, seed=rank_seed(wl, rank) + 20, dtype=wl.torch_dtype,
                        device="cuda")
    S = (0.02 * torch.randn(wl.B, wl.H, wl.d_k, wl.d_v, device="cuda")).contiguous()
    o = torch.empty(wl.B, wl.H, wl.d_v, dtype=wl.torch_dtype, device="cuda")
    it = {"s": 0}

    def step():
        s = it["s"] % steps
        it["s"] += 1
        g.decode_step_qed(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s], c[s], d["w"][s], S, o=o,
                          stream=stream)

    for _ in range(8):
        step()
    torch.cuda.synchronize()
    it["s"] = 0
    ms = device_time_ms(step, steps, stream)
    if g.device_status() != 0:
        raise RuntimeError("QED decode kernel reported a device error")
    return ms / steps


def bench_decode_fused(g, wl, steps, rank, stream):
    d = W.draw_raw(wl.B, None, wl.H, wl.d_k, wl.d_v, seed=rank_seed(wl, rank) + 7, dtype=wl.torch_dtype,
                   alpha_lo=wl.alpha_lo, alpha_hi=wl.alpha_hi, qk_scale=2.0, s0_std=wl.s0_std, steps=steps,
                   device="cuda")
    S = d["S0"].clone()
    o = torch.empty(wl.B, wl.H, wl.d_v, dtype=wl.torch_dtype, device="cuda")
    it = {"s": 0}

    def step():
        s = it["s"] % steps
        it["s"] += 1
        g.decode_step_ex(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s], d["w"][s], S,
                         prep=True, gate=d["gate"][s], norm_weight=d["norm_weight"], o=o, stream=stream)

    for _ in range(8):
        step()
    torch.cuda.synchronize()
    S.copy_(d["S0"])
    it["s"] = 0
    ms = device_time_ms(step, steps, stream)
    if g.device_status() != 0:
        raise RuntimeError("fused decode kernel reported a device timeout")
    return ms / steps


def bench_chunk_e2e(g, wl, d, steps, stream, o_dev=None, st_dev=None):
    """The same step through the host-buffer C-ABI entry (gdn2_chunk_fwd_host):
    every step copies the pinned host inputs in and o, S_T out, the library
    overlapping the copies of one slice of sequences with the kernel of the
    next."""
    names = ("q", "k", "v", "log_alpha", "b", "w")
    host = {n: d[n].cpu().pin_memory() for n in names}
    s0_host = d["S0"].cpu().pin_memory() if d["S0"] is not None else None
    o_host = torch.empty(d["v"].shape, dtype=d["v"].dtype).pin_memory()
    st_host = torch.empty(wl.B, wl.H, wl.d_k, wl.d_v, dtype=torch.float32).pin_memory()
    ws = torch.empty(g.chunk_fwd_host_workspace_bytes(wl.B, wl.T, wl.H, wl.d_k, wl.d_v, d["q"].dtype),
                     dtype=torch.uint8, device="cuda")
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + \
        (s0_host.numel() * 4 if s0_host is not None else 0)
    d2h = o_host.numel() * o_host.element_size() + st_host.numel() * 4

    def step():
        g.chunk_fwd_host(*(host[n] for n in names), s0_host, o=o_host, S_T=st_host, workspace=ws,
                         stream=stream)

    step()
    torch.cuda.synchronize()
    ms = device_time_ms(step, steps, stream)
    torch.cuda.synchronize()
    # the host-buffer results must equal the device entry's on the same inputs
    same = None
    if o_dev is not None and st_dev is not None:
        same = bool(torch.equal(o_host, o_dev.cpu()) and torch.equal(st_host, st_dev.cpu()))
    return ms, h2d, d2h, same


def bench_decode(g, wl, steps, rank, stream, graph: bool = False):
    """The decode workload: `steps` consecutive steps, timed on the device.  With
    graph=True the same steps are also captured once as one CUDA graph and the
    graph replay is timed; returns (plain ms, graph ms or None)."""
    d = W.make_decode_inputs(wl, steps, seed=rank_seed(wl, rank), device="cuda")
    S = d["S0"].clone()
    o = torch.empty(wl.B, wl.H, wl.d_v, dtype=wl.torch_dtype, device="cuda")
    it = {"s": 0}

    def step(st=stream):
        s = it["s"] % steps
        it["s"] += 1
        g.decode_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["b"][s], d["w"][s], S,
                      o=o, stream=st)

    for _ in range(8):
        step()
    torch.cuda.synchronize()
    S.copy_(d["S0"])
    it["s"] = 0
    ms = device_time_ms(step, steps, stream)
    if g.device_status() != 0:
        raise RuntimeError("decode kernel reported a device timeout")
    ms_graph = None
    if graph:
        cg = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        it["s"] = 0
        with torch.cuda.graph(cg, stream=cap):
            for _ in range(steps):
                step(cap)
        torch.cuda.synchronize()
        for _ in range(2):   # warm the graph
            cg.replay()
        torch.cuda.synchronize()
        S.copy_(d["S0"])
        with torch.cuda.stream(stream):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            cg.replay()
            e1.record(stream)
        e1.synchronize()
        ms_graph = e0.elapsed_time(e1)
        del cg
        if g.device_status() != 0:
            raise RuntimeError("decode kernel reported a device timeout")
    return ms, ms_graph


# --------------------------------------------------------- oracle (CPU)
def oracle_sample(wl, d_cpu_fn, budget_s: float = 10.0):
    """Time the fp64 oracle, as it stands, on whole heads of the workload
    until about `budget_s` of wall time has passed.  Returns (tokens/s,
    cores, description); a token is one (b, t) through all H heads."""
    import oracle
    cores = oracle.max_threads()
    heads_done, t_used, rounds = 0, 0.0, 0
    while t_used < budget_s and rounds < 64:
        inp = d_cpu_fn(cores, rounds)
        t0 = time.perf_counter()
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                       S0=inp["S0"], n_threads=cores, want_state=True)
        t_used += time.perf_counter() - t0
        heads_done += inp["q"].shape[2]
        rounds += 1
    tok = heads_done * wl.T / wl.H
    return tok / t_used, cores, f"{heads_done} whole heads (T={wl.T}) of {wl.describe()}, {t_used:.1f} s"


def head_sample_fn(wl):
    """Sample n heads of the workload as a [1, T, n, d] CPU batch."""
    def fn(n, r):
        return W.draw(1, wl.T, n, wl.d_k, wl.d_v, seed=wl.seed + 7919 * (r + 1), dtype=wl.torch_dtype,
                      alpha_lo=wl.alpha_lo, alpha_hi=wl.alpha_hi, b_scale=wl.b_scale, s0_std=wl.s0_std)
    return fn


def profile_case(g, args, stream):
    """A reduced launch of one kernel for profiler captures."""
    import dataclasses
    if args.profile_case == "decode":
        wl = dataclasses.replace(W.BY_NAME["decode_bf16"], decode_steps=args.warmup + args.steps)
        ms, _ = bench_decode(g, wl, wl.decode_steps, 0, stream)
        print(json.dumps({"profile_case": "decode", "workload": wl.describe(),
                          "us_per_step": 1e3 * ms / wl.decode_steps}))
        return
    if args.profile_case == "chunk_fused":   # the headline shape at B = 2, fused prep + epilogue
        wl = dataclasses.replace(W.BY_NAME[HEADLINE], B=2)
        ms = bench_chunk_fused(g, wl, args.steps, args.warmup, 0, stream)
        print(json.dumps({"profile_case": "chunk_fused", "workload": wl.describe(), "ms_per_call": ms}))
        return
    base = W.BY_NAME[HEADLINE if args.profile_case == "chunk" else "chunk_bf16_negeig"]
    wl = dataclasses.replace(base, B=2 if base.d_v == 128 else 1)
    ms, d, _, _ = bench_chunk(g, wl, args.steps, args.warmup, 0, 1, stream)
    print(json.dumps({"profile_case": args.profile_case, "workload": wl.describe(),
                      "ms_per_call": ms / args.steps,
                      "bytes_per_call": chunk_bytes(wl, with_s0=d["S0"] is not None)}))


# ------------------------------------------------------------------ main
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world


def run_reference(args, world):
    """The reference arm: the fp64 oracle on the host cores (no GPU)."""
    wl = W.BY_NAME[HEADLINE]
    fn = head_sample_fn(wl)
    import oracle
    cores = oracle.max_threads()
    for r in range(args.warmup):
        inp = fn(cores, 1000 + r)
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                       S0=inp["S0"], n_threads=cores)
    t_total, heads = 0.0, 0
    for r in range(args.steps):
        inp = fn(cores, r)
        t0 = time.perf_counter()
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                       S0=inp["S0"], n_threads=cores)
        t_total += time.perf_counter() - t0
        heads += inp["q"].shape[2]
    tok_s = heads * wl.T / wl.H / t_total
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.describe(), "parallelism": "host cores (OpenMP over heads)"},
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {cores} whole heads (T={wl.T}) of {wl.describe()}"},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--steady-s", type=float, default=0.5,
                    help="after the timed steps, time rounds of 50 calls for at least this long (median reported)")
    ap.add_argument("--no-extras", action="store_true", help="skip decode/expanded-value/CPU legs")
    ap.add_argument("--profile-case", choices=["chunk", "chunk_v256", "chunk_fused", "decode"], default=None,
                    help="only launch one kernel on a reduced batch (inputs still larger than L2), "
                         "for ncu captures; prints a short line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, world)
        return

    rank, world = dist_setup()
    import gated_delta_rule_92_b200 as g
    g.lib()
    peaks = load_peaks()
    stream = torch.cuda.Stream()
    wl = W.BY_NAME[HEADLINE]
    if args.profile_case is not None:
        profile_case(g, args, stream)
        return

    sampler = ClockSampler(period_s=0.002)
    ms, d, o, S_T, steady = bench_chunk(g, wl, args.steps, args.warmup, rank, world, stream, sampler,
                                        steady_s=args.steady_s)
    value, ms_max = aggregate_throughput(ms, args.steps, wl.B * wl.T, world)
    launch_ms = ms / args.steps
    abytes = chunk_bytes(wl, with_s0=d["S0"] is not None)
    achieved = abytes / (launch_ms / 1e3) / 1e9
    flops = chunk_flops(wl)

    with nvtx("e2e host buffers"):
        e2e_ms, h2d, d2h, e2e_same = bench_chunk_e2e(g, wl, d, args.e2e_steps, stream, o, S_T)
    e2e_val, e2e_ms = aggregate_throughput(e2e_ms, args.e2e_steps, wl.B * wl.T, world)
    del d, o, S_T
    torch.cuda.empty_cache()

    extras = {}
    torch.cuda.nvtx.range_push("other workloads")
    if not args.no_extras:
        wl3 = W.BY_NAME["chunk_bf16_negeig"]
        ms3, d3, _, _ = bench_chunk(g, wl3, max(5, args.steps // 4), 3, rank, world, stream)
        l3 = ms3 / max(5, args.steps // 4)
        b3 = chunk_bytes(wl3, with_s0=True)
        extras["expanded_v"] = {
            "workload": wl3.describe(), "value": wl3.B * wl3.T / (l3 / 1e3), "unit": "tokens/s",
            "ms_per_call": l3,
            "roofline": {"bound": "hbm", "achieved": b3 / (l3 / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": b3 / (l3 / 1e3) / 1e9 / peaks["hbm_gbs"]}}
        del d3
        torch.cuda.empty_cache()
        wl4 = W.BY_NAME["decode_bf16"]
        with ClockSampler(period_s=0.002) as s4:
            ms4, ms4g = bench_decode(g, wl4, wl4.decode_steps, rank, stream, graph=True)
        ms4 = max_over_ranks(ms4, world)
        ms4g = max_over_ranks(ms4g, world)
        per = ms4 / wl4.decode_steps
        b4 = decode_bytes(wl4)
        extras["decode"] = {
            "workload": wl4.describe(), "value": wl4.B * world * wl4.decode_steps / (ms4 / 1e3),
            "unit": "tokens/s", "us_per_step": 1e3 * per, "steps": wl4.decode_steps,
            "roofline": {"bound": "hbm", "achieved": b4 / (per / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": b4 / (per / 1e3) / 1e9 / peaks["hbm_gbs"],
                         "bytes_per_step": b4, "traffic": measured_traffic("decode_step", wl4.B)},
            "graph": {"value": wl4.B * world * wl4.decode_steps / (ms4g / 1e3), "unit": "tokens/s",
                      "us_per_step": 1e3 * ms4g / wl4.decode_steps,
                      "frac": b4 / (ms4g / wl4.decode_steps / 1e3) / 1e9 / peaks["hbm_gbs"],
                      "how": f"the {wl4.decode_steps} steps captured once as one CUDA graph, one replay timed"},
            "clocks": s4.summary()}
        torch.cuda.empty_cache()
        # f1 + f2: the headline chunk workload and the decode workload from raw
        # projections, input prep and gated RMS-norm epilogue fused in
        io_b = 2 if wl.io == "bf16" else 4
        lf = bench_chunk_fused(g, wl, max(10, args.steps // 4), 3, rank, stream)
        bf = chunk_bytes(wl, with_s0=wl.s0_std is not None) + wl.B * wl.T * wl.H * wl.d_v * io_b + 4 * wl.d_v
        extras["chunk_fused_prep_epilogue"] = {
            "workload": wl.describe() + " + fused input prep + gated RMS-norm epilogue",
            "value": wl.B * wl.T / (lf / 1e3), "unit": "tokens/s", "ms_per_call": lf,
            "roofline": {"bound": "hbm", "achieved": bf / (lf / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": bf / (lf / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes_per_launch": bf}}
        torch.cuda.empty_cache()
        nfs = 256
        pf = bench_decode_fused(g, wl4, nfs, rank, stream)
        bdf = decode_bytes(wl4) + wl4.B * wl4.H * wl4.d_v * 2 + 4 * wl4.d_v
        extras["decode_fused_prep_epilogue"] = {
            "workload": wl4.describe().replace(f"steps{wl4.decode_steps}", f"steps{nfs}")
            + " + fused input prep + gated RMS-norm epilogue",
            "value": wl4.B / (pf / 1e3), "unit": "tokens/s", "us_per_step": 1e3 * pf, "steps": nfs,
            "roofline": {"bound": "hbm", "achieved": bdf / (pf / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": bdf / (pf / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes_per_step": bdf}}
        torch.cuda.empty_cache()

        # f3: the headline's 32768 tokens as packed sequences of mixed length, and
        # value heads (8 key heads shared by 16 value heads) at the headline shape
        lens = W.packed_lengths(64, wl.T // 8, seed=rank_seed(wl, rank) + 13, min_len=1)
        nst = max(10, args.steps // 4)
        for name, kw, desc in (
                ("packed_varlen", dict(lengths=lens),
                 f"chunk_fwd {len(lens)} packed sequences, {sum(lens)} tokens (lengths ~ exponential, "
                 f"mean {wl.T // 8}), H{wl.H} d_k{wl.d_k} d_v{wl.d_v} chunk64 bf16"),
                ("value_heads", dict(H=wl.H // 2, HV=wl.H),
                 f"chunk_fwd B{wl.B} T{wl.T} H{wl.H // 2} key heads, HV{wl.H} value heads, "
                 f"d_k{wl.d_k} d_v{wl.d_v} chunk64 bf16")):
            lg, bg, ntok = bench_chunk_general(g, wl, nst, rank, stream, **kw)
            extras[name] = {
                "workload": desc, "value": ntok / (lg / 1e3), "unit": "tokens/s", "ms_per_call": lg,
                "roofline": {"bound": "hbm", "achieved": bg / (lg / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": bg / (lg / 1e3) / 1e9 / peaks["hbm_gbs"],
                             "bytes_per_launch": bg}}
            torch.cuda.empty_cache()

        # strong decay: the tensor-core form near its range, and the token tail
        for kind, nsd in (("alpha_005_05", max(10, args.steps // 4)), ("mixed", 3)):
            ld = bench_chunk_decay(g, wl, nsd, rank, stream, kind)
            extras["strong_decay_" + kind] = {
                "workload": wl.describe() + (" with alpha ~ U[0.05, 0.5]" if kind == "alpha_005_05" else
                                             " with even key channels alpha ~ 1e-3 (token tail)"),
                "value": wl.B * wl.T / (ld / 1e3), "unit": "tokens/s", "ms_per_call": ld,
                "roofline": {"bound": "hbm", "achieved": abytes / (ld / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": abytes / (ld / 1e3) / 1e9 / peaks["hbm_gbs"]}}
            torch.cuda.empty_cache()

        # f4: the second, query-derived erase direction (CUDA cores)
        lq = bench_chunk_qed(g, wl, 3, rank, stream)
        bq = chunk_bytes(wl, with_s0=wl.s0_std is not None) + wl.B * wl.T * wl.H * wl.d_k * io_b
        extras["chunk_qed"] = {
            "workload": wl.describe() + " + second erase direction (query-derived)",
            "value": wl.B * wl.T / (lq / 1e3), "unit": "tokens/s", "ms_per_call": lq,
            "roofline": {"bound": "hbm", "achieved": bq / (lq / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": bq / (lq / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes_per_launch": bq}}
        torch.cuda.empty_cache()
        nq = 256
        pq = bench_decode_qed(g, wl4, nq, rank, stream)
        bdq = decode_bytes(wl4) + wl4.B * wl4.H * wl4.d_k * 2
        extras["decode_qed"] = {
            "workload": wl4.describe().replace(f"steps{wl4.decode_steps}", f"steps{nq}")
            + " + second erase direction (query-derived)",
            "value": wl4.B / (pq / 1e3), "unit": "tokens/s", "us_per_step": 1e3 * pq, "steps": nq,
            "roofline": {"bound": "hbm", "achieved": bdq / (pq / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": bdq / (pq / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes_per_step": bdq}}
        torch.cuda.empty_cache()

    torch.cuda.nvtx.range_pop()
    cpu = None
    if rank == 0 and world == 1 and not args.no_extras:
        with nvtx("oracle on the host cores"):
            tok_s, cores, desc = oracle_sample(wl, head_sample_fn(wl))
        cpu = {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.describe(), "global_batch": wl.B * world, "seq_len": wl.T,
                       "heads": wl.H, "d_k": wl.d_k, "d_v": wl.d_v, "chunk": wl.chunk,
                       "state": "fp32", "parallelism": f"dp{world} (independent batches)",
                       "l2": f"inputs larger than L2 ({abytes / 1e6:.0f} MB per step); no flush"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"],
                         "traffic": measured_traffic("chunk_fwd_tc", wl.B),
                         "peak_source": peaks["source"], "bytes_per_launch": abytes,
                         "tensor_tflops": flops / (launch_ms / 1e3) / 1e12,
                         "tensor_frac": flops / (launch_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                         # max(t_flop, t_byte) / t: the fraction of the tighter of the two bounds
                         "attainable_frac": max(abytes / (peaks["hbm_gbs"] * 1e9),
                                                flops / (peaks["bf16_tflops"] * 1e12)) / (launch_ms / 1e3)},
            "steady": steady,
            "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                    "equals_device_path": e2e_same},
            "gpu_launches": args.steps,
            "clocks": sampler.summary(),
            "cpu_baseline": cpu,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
