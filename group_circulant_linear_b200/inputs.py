"""Seeded synthetic inputs for the EQ-Linear layer.

This module is shared by the CUDA path's tests and benchmark and by the
oracle's tests.  It holds no arithmetic of the method: it only draws random
tensors in a fixed order from a seeded generator and casts them.

Recipe (one generator per call, seeded; draws in the order x, W, b, gy, all in
float32, then cast to the requested dtype):

* x  ~ N(0, 1), shape [N, C'*T]
* W  ~ U(-1/sqrt(C), 1/sqrt(C)) with C = C'*T the full input width, shape [D', C', T]
* b  ~ U(-0.1, 0.1), shape [D']
* gy ~ N(0, 1), shape [N, D'*T]

The integer recipe (for bit-exact checks) draws x, W, gy uniformly from the
integers in [-amp, amp] and b from {-1, 0, 1}.
"""
from __future__ import annotations

import math

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _dtype(dtype) -> torch.dtype:
    if isinstance(dtype, torch.dtype):
        return dtype
    return DTYPES[dtype]


def make_inputs(T: int, Cp: int, Dp: int, N: int, dtype="f32", seed: int = 0,
                with_gy: bool = True, device="cpu") -> dict:
    """Draw x, W, b (and gy) for one layer; returns a dict of tensors."""
    dt = _dtype(dtype)
    g = torch.Generator(device=device).manual_seed(seed)
    C = Cp * T
    bound = 1.0 / math.sqrt(C)
    x = torch.randn((N, C), generator=g, dtype=torch.float32, device=device)
    W = torch.rand((Dp, Cp, T), generator=g, dtype=torch.float32, device=device)
    W = W * (2 * bound) - bound
    b = torch.rand((Dp,), generator=g, dtype=torch.float32, device=device) * 0.2 - 0.1
    out = {"x": x.to(dt), "W": W.to(dt), "b": b.to(dt)}
    if with_gy:
        out["gy"] = torch.randn((N, Dp * T), generator=g, dtype=torch.float32,
                                device=device).to(dt)
    return out


def make_integer_inputs(T: int, Cp: int, Dp: int, N: int, dtype="f32", seed: int = 0,
                        amp: int = 4, device="cpu") -> dict:
    """Integer-valued x, W, gy in [-amp, amp] and b in {-1, 0, 1}."""
    dt = _dtype(dtype)
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randint(-amp, amp + 1, (N, Cp * T), generator=g, device=device)
    W = torch.randint(-amp, amp + 1, (Dp, Cp, T), generator=g, device=device)
    b = torch.randint(-1, 2, (Dp,), generator=g, device=device)
    gy = torch.randint(-amp, amp + 1, (N, Dp * T), generator=g, device=device)
    return {"x": x.to(dt), "W": W.to(dt), "b": b.to(dt), "gy": gy.to(dt)}
