"""Helpers for the GPU parity tests: inputs to device, oracle on the same
values, and the error measure the tolerances are stated in."""
import numpy as np
import torch

import oracle

# Tolerances (max-abs error relative to the reference's max-abs value):
# fp32 I/O 1e-4 and bf16 I/O 2e-2, for o and for the final state alike.
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def to_dev(inp, dev="cuda"):
    out = {n: (t.to(dev) if t is not None else None) for n, t in inp.items()}
    return out


def rel_inf(got: np.ndarray, ref: np.ndarray) -> float:
    scale = float(np.max(np.abs(ref)))
    if scale == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref))) / scale


def heads_of(o_btHd: torch.Tensor, heads, H):
    """[B,T,H,d] -> [n_heads, T, d] for flat head indices b*H+h."""
    return np.stack([o_btHd[h // H, :, h % H, :].float().cpu().numpy() for h in heads])


def state_heads(S: torch.Tensor, heads, H):
    return np.stack([S[h // H, h % H].double().cpu().numpy() for h in heads])


def oracle_chunk(inp, heads=None):
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"],
                          S0=None if inp["S0"] is None else inp["S0"], heads=heads)
