"""Seeded synthetic inputs for the Gated DeltaNet-2 mixer.

This module only draws random numbers and casts them; it holds none of the
recurrence's arithmetic, so both the CUDA path's tests and the fp64 oracle can
take their inputs from here without sharing method code.

Workloads (sizes follow the burn-gdn2 README "Configuration" table: 16 heads,
head_dim 128, hidden 2048 by default, chunk 64):

  chunk_f32_small   B1 T256  H4  d_k=d_v=64   fp32 I/O, S0 = 0
  chunk_bf16_small  B1 T1024 H4  d_k=d_v=64   bf16 I/O, S0 ~ N(0, 0.02)
  chunk_bf16_h2048  B8 T4096 H16 d_k=d_v=128  bf16 I/O, S0 = 0
  chunk_bf16_negeig B4 T8192 H16 d_k=128 d_v=256, bf16, b in (0,2),
                    alpha in [0.8, 0.9999], S0 ~ N(0, 0.02)
  decode_bf16       256 sequences x H16 x d128, one token per step,
                    1024 steps, S0 ~ N(0, 0.02)

Recipe (every workload): a CPU ``torch.Generator`` seeded with
``1000 + index``; draw order q, k, v, alpha, b, w, S0.  q and k are N(0,1)
then L2-normalised over d_k per (b, t, h) in fp32 before the cast (the README
puts an L2-norm in front of the mixer); v ~ N(0,1); alpha ~ U[lo, hi] i.i.d.
per (b, t, h, key channel) and log_alpha = ln(alpha); b = scale * sigmoid(N(0,1))
per key channel (scale 2 when negative eigenvalues are allowed, "b x 2" in the
README table); w = sigmoid(N(0,1)) per value channel; S0 ~ N(0, std) in fp32.
Token tensors are then cast to the I/O dtype; the oracle reads the cast values.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    T: int
    H: int
    d_k: int
    d_v: int
    io: str                    # "f32" or "bf16"
    chunk: int = 64
    alpha_lo: float = 0.9
    alpha_hi: float = 0.999
    b_scale: float = 1.0
    s0_std: Optional[float] = None
    decode_steps: int = 0      # > 0: decode workload (T is 1 per step)
    extra: dict = field(default_factory=dict)

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def torch_dtype(self):
        return torch.float32 if self.io == "f32" else torch.bfloat16

    def describe(self) -> str:
        if self.decode_steps:
            return (f"decode B{self.B} H{self.H} d_k{self.d_k} d_v{self.d_v} "
                    f"{self.io} steps{self.decode_steps}")
        return (f"chunk_fwd B{self.B} T{self.T} H{self.H} d_k{self.d_k} d_v{self.d_v} "
                f"chunk{self.chunk} {self.io}")


WORKLOADS = [
    Workload(0, "chunk_f32_small", B=1, T=256, H=4, d_k=64, d_v=64, io="f32"),
    Workload(1, "chunk_bf16_small", B=1, T=1024, H=4, d_k=64, d_v=64, io="bf16", s0_std=0.02),
    Workload(2, "chunk_bf16_h2048", B=8, T=4096, H=16, d_k=128, d_v=128, io="bf16"),
    Workload(3, "chunk_bf16_negeig", B=4, T=8192, H=16, d_k=128, d_v=256, io="bf16",
             alpha_lo=0.8, alpha_hi=0.9999, b_scale=2.0, s0_std=0.02),
    Workload(4, "decode_bf16", B=256, T=1, H=16, d_k=128, d_v=128, io="bf16",
             s0_std=0.02, decode_steps=1024),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def draw(B: int, T: int, H: int, d_k: int, d_v: int, *, seed: int,
         dtype=torch.bfloat16, alpha_lo: float = 0.9, alpha_hi: float = 0.999,
         b_scale: float = 1.0, s0_std: Optional[float] = None, HV: Optional[int] = None,
         generator: Optional[torch.Generator] = None, device="cpu") -> dict:
    """Draw one batch of token inputs [B, T, H, d].

    Returns a dict with q, k, log_alpha, b [B, T, H, d_k] and v, w
    [B, T, HV, d_v] in ``dtype`` (HV value heads, default H) and S0 (fp32
    [B, HV, d_k, d_v] or None).  With ``device="cuda"`` the draws are made by
    a CUDA generator with the same seed and recipe (a different stream of
    numbers than the CPU generator; used where only the distribution matters,
    e.g. timing).
    """
    g = generator if generator is not None else torch.Generator(device=device).manual_seed(seed)
    f32 = torch.float32
    kw = dict(generator=g, dtype=f32, device=device)
    HV = H if HV is None else HV
    q = _l2n(torch.randn(B, T, H, d_k, **kw))
    k = _l2n(torch.randn(B, T, H, d_k, **kw))
    v = torch.randn(B, T, HV, d_v, **kw)
    alpha = torch.empty(B, T, H, d_k, dtype=f32, device=device).uniform_(alpha_lo, alpha_hi, generator=g)
    b = b_scale * torch.sigmoid(torch.randn(B, T, H, d_k, **kw))
    w = torch.sigmoid(torch.randn(B, T, HV, d_v, **kw))
    S0 = None
    if s0_std is not None:
        S0 = s0_std * torch.randn(B, HV, d_k, d_v, **kw)
    out = dict(q=q, k=k, v=v, log_alpha=torch.log(alpha), b=b, w=w)
    out = {n: t.to(dtype).contiguous() for n, t in out.items()}
    out["S0"] = S0
    return out


def draw_raw(B: int, T: int, H: int, d_k: int, d_v: int, *, seed: int,
             dtype=torch.bfloat16, alpha_lo: float = 0.9, alpha_hi: float = 0.999,
             qk_scale: float = 1.0, s0_std: Optional[float] = None, steps: Optional[int] = None,
             HV: Optional[int] = None, generator: Optional[torch.Generator] = None, device="cpu") -> dict:
    """Inputs for the fused input prep and output epilogue: the raw
    projections the layer would hand the mixer.

    q, k ~ qk_scale N(0,1) (not normalised); b, w ~ N(0,1) (gate logits);
    v ~ N(0,1); alpha ~ U[alpha_lo, alpha_hi], log_alpha = ln alpha; the
    output gate g ~ N(0,1); the RMS-norm weight ~ U[0.5, 1.5] (synthetic, one
    [d_v] vector, fp32); S0 ~ N(0, s0_std) or None.  Token tensors are
    [B, T, H, d], or [steps, B, H, d] for decode when ``steps`` is given;
    v, w and g carry HV value heads (default H), S0 is [B, HV, d_k, d_v].
    """
    g = generator if generator is not None else torch.Generator(device=device).manual_seed(seed)
    f32 = torch.float32
    kw = dict(generator=g, dtype=f32, device=device)
    HV = H if HV is None else HV
    lead = (steps, B, H) if steps is not None else (B, T, H)
    vlead = lead[:-1] + (HV,)
    q = qk_scale * torch.randn(*lead, d_k, **kw)
    k = qk_scale * torch.randn(*lead, d_k, **kw)
    v = torch.randn(*vlead, d_v, **kw)
    alpha = torch.empty(*lead, d_k, dtype=f32, device=device).uniform_(alpha_lo, alpha_hi, generator=g)
    b = torch.randn(*lead, d_k, **kw)
    w = torch.randn(*vlead, d_v, **kw)
    gate = torch.randn(*vlead, d_v, **kw)
    weight = torch.empty(d_v, dtype=f32, device=device).uniform_(0.5, 1.5, generator=g)
    S0 = None
    if s0_std is not None:
        S0 = s0_std * torch.randn(B, HV, d_k, d_v, **kw)
    out = dict(q=q, k=k, v=v, log_alpha=torch.log(alpha), b=b, w=w, gate=gate)
    out = {n: t.to(dtype).contiguous() for n, t in out.items()}
    out["S0"] = S0
    out["norm_weight"] = weight
    return out


def draw_qed_gate(lead, d_k: int, *, seed: int, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """The second erase gate c of the query-derived erase direction: sigmoid(N(0,1))
    per key channel, shape lead + (d_k,), from its own generator (the other inputs'
    draws are unchanged)."""
    g = torch.Generator(device=device).manual_seed(seed)
    c = torch.sigmoid(torch.randn(*lead, d_k, generator=g, dtype=torch.float32, device=device))
    return c.to(dtype).contiguous()


def packed_lengths(n: int, mean: int, *, seed: int, min_len: int = 0) -> list:
    """Lengths of ``n`` packed sequences: a geometric-like mix around ``mean``
    tokens (exponential draw, rounded), at least ``min_len``.  Used for the
    packed variable-length cases."""
    g = torch.Generator().manual_seed(seed)
    e = torch.empty(n, dtype=torch.float64).exponential_(1.0, generator=g)
    return [max(min_len, int(round(float(x) * mean))) for x in e]


def cu_seqlens_of(lengths) -> torch.Tensor:
    """int32 [n + 1] offsets of sequences of the given lengths packed back to back."""
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def make_chunk_inputs(wl: Workload, *, B: Optional[int] = None, T: Optional[int] = None,
                      H: Optional[int] = None, seed: Optional[int] = None, device="cpu") -> dict:
    """Inputs of a chunk workload (optionally resized, same recipe)."""
    return draw(B or wl.B, T or wl.T, H or wl.H, wl.d_k, wl.d_v,
                seed=wl.seed if seed is None else seed, dtype=wl.torch_dtype,
                alpha_lo=wl.alpha_lo, alpha_hi=wl.alpha_hi, b_scale=wl.b_scale,
                s0_std=wl.s0_std, device=device)


def make_decode_inputs(wl: Workload, steps: int, *, B: Optional[int] = None,
                       seed: Optional[int] = None, device="cpu") -> dict:
    """Decode inputs: token tensors [steps, B, H, d] and S0 [B, H, d_k, d_v].

    Drawn as a [B, steps, H, d] batch with the same recipe, then laid out with
    the step axis first so that step s is one contiguous [B, H, d] slab.
    """
    Bn = B or wl.B
    d = draw(Bn, steps, wl.H, wl.d_k, wl.d_v, seed=wl.seed if seed is None else seed,
             dtype=wl.torch_dtype, alpha_lo=wl.alpha_lo, alpha_hi=wl.alpha_hi,
             b_scale=wl.b_scale, s0_std=wl.s0_std, device=device)
    for n in ("q", "k", "v", "log_alpha", "b", "w"):
        d[n] = d[n].transpose(0, 1).contiguous()
    return d


def kda_collapse(inp: dict, seed: int, b_scale: float = 1.0) -> dict:
    """Same inputs with b and w replaced by one scalar beta per (b, t, h).

    beta is drawn with the workload's b recipe (b_scale * sigmoid(N(0,1))) and
    broadcast over d_k (for b) and over d_v (for w).
    """
    g = torch.Generator().manual_seed(seed)
    q = inp["q"]
    B, T, H, dk = q.shape
    dv = inp["v"].shape[-1]
    beta = b_scale * torch.sigmoid(torch.randn(B, T, H, 1, generator=g, dtype=torch.float32))
    out = dict(inp)
    out["b"] = beta.expand(B, T, H, dk).to(q.dtype).contiguous()
    out["w"] = beta.expand(B, T, H, dv).to(q.dtype).contiguous()
    return out


def gdn_collapse(inp: dict, seed: int, b_scale: float = 1.0) -> dict:
    """KDA collapse plus a scalar decay per (b, t, h): channel 0 broadcast."""
    out = kda_collapse(inp, seed, b_scale)
    la = inp["log_alpha"]
    out["log_alpha"] = la[..., :1].expand_as(la).contiguous()
    return out


# ------------------------------------------------ strong-decay input variants
# These only replace log_alpha with other random draws; the recurrence itself
# accepts any log_alpha <= 0 and these cover the regimes where a chunked
# evaluation has to keep its exponents in range.

def with_mixed_decay(inp: dict, seed: int, fast=(5e-4, 2e-3), slow=(0.99, 0.9999)) -> dict:
    """Even key channels decay fast (alpha ~ U[fast]), odd ones barely (alpha ~ U[slow])."""
    g = torch.Generator().manual_seed(seed)
    la = inp["log_alpha"]
    shape = la.shape
    u = torch.rand(shape, generator=g, dtype=torch.float64)
    lo = torch.tensor([fast[0], slow[0]], dtype=torch.float64)[torch.arange(shape[-1]) % 2]
    hi = torch.tensor([fast[1], slow[1]], dtype=torch.float64)[torch.arange(shape[-1]) % 2]
    out = dict(inp)
    out["log_alpha"] = torch.log(lo + (hi - lo) * u).to(la.dtype).contiguous()
    return out


def with_decay_spikes(inp: dict, seed: int, prob: float = 0.03, value: float = -20.0) -> dict:
    """Each (b, t, h) token independently, with probability `prob`, gets
    log_alpha = `value` on every key channel (a near-reset of the state)."""
    g = torch.Generator().manual_seed(seed)
    la = inp["log_alpha"]
    hit = torch.rand(la.shape[:-1], generator=g) < prob
    out = dict(inp)
    out["log_alpha"] = torch.where(hit[..., None], torch.full_like(la, value), la).contiguous()
    return out


def with_decay_burst(inp: dict, t0: int, t1: int, value: float) -> dict:
    """Tokens t0 <= t < t1 of every sequence and head get log_alpha = `value` (token axis 1)."""
    la = inp["log_alpha"].clone()
    la[:, t0:t1] = value
    out = dict(inp)
    out["log_alpha"] = la.contiguous()
    return out
