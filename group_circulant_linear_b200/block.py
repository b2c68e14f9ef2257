"""EQ-Linear as a torch autograd layer, and a synthetic EQ-ViT block built on it.

The pages present Flash EQ-Linear as a drop-in replacement for the naive
equivariant linear layer, with no retraining, and time it inside EQ-ViT
blocks ("Flash EQ-Linear", technical summary, sections "Implementacao" and
"Resultados Experimentais").  This module is that drop-in:

* ``EQLinearFunction`` -- when gradients are needed and every pass runs on
  the tensor cores, forward runs ``eqlin_forward_stash`` and keeps the input's
  spectrum X = DFT(x) (instead of x) for the backward, which is one
  ``eqlin_backward`` call: dx with G = DFT(gy) stashed, then dW and db from
  the two spectra.  Otherwise forward runs ``eqlin_forward`` and backward
  ``eqlin_backward_dx`` and ``eqlin_backward_dw``.  All through the C ABI
  binding.
* ``EQLinear`` -- an ``nn.Module`` holding W [D', C', T] and b [D'] as
  parameters and one library handle; it re-runs the weight transform
  (``eqlin_set_weights``) only when the parameters have changed.
* ``GroupLayerNorm`` and ``EQViTBlock`` -- a pre-norm transformer block whose
  qkv, projection and MLP layers are EQ-Linear.  Features are [C', T]: the
  norm's statistics run over all C'T features and its affine parameters are
  shared along the group axis, attention heads split C', and GELU is
  pointwise, so the block commutes with a cyclic shift of the group axis.
  Weights are synthetic (random).
* ``expand_dense`` and ``DenseEQViTBlock`` -- the naive layer the pages
  compare against: the block-circulant dense matrix W_dense[d*T+s, c*T+t] =
  W[d, c, (s-t) mod T] applied with an ordinary (cuBLAS) linear.  It is
  timed beside the Flash block for context only.

``python -m group_circulant_linear_b200.block`` times one block, forward and
forward + backward, both ways, and prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math

import torch
import torch.nn as nn
import torch.nn.functional as F

from . import eqlin


class EQLinearFunction(torch.autograd.Function):
    """y = EQ-Linear(x; W, b) with the library's kernels in both directions."""

    @staticmethod
    def forward(ctx, x, W, b, layer):
        lead = x.shape[:-1]
        x2 = x.reshape(-1, layer.Cp * layer.T).to(layer.dtype).contiguous()
        layer.sync_weights(W, b)
        N = x2.shape[0]
        y = torch.empty((N, layer.Dp * layer.T), dtype=layer.dtype, device=x.device)
        fused = layer.fused and any(ctx.needs_input_grad[:3]) and N > 0
        if fused:
            xs = eqlin.empty_spectra(layer.h, "x", N, device=x.device)
            eqlin.forward_stash(layer.h, x2, y, xs)
            ctx.save_for_backward(xs)
        else:
            eqlin.forward(layer.h, x2, y)
            ctx.save_for_backward(x2)
        ctx.fused = fused
        ctx.N = N
        ctx.layer = layer
        ctx.lead = lead
        ctx.x_dtype = x.dtype
        ctx.w_dtype = W.dtype
        ctx.b_dtype = None if b is None else b.dtype
        return y.reshape(*lead, layer.Dp * layer.T)

    @staticmethod
    def backward(ctx, gy):
        (saved,) = ctx.saved_tensors
        L = ctx.layer
        gy2 = gy.reshape(-1, L.Dp * L.T).to(L.dtype).contiguous()
        dx = dW = db = None
        want_w = ctx.needs_input_grad[1] or ctx.needs_input_grad[2]
        dx2 = torch.empty((ctx.N, L.Cp * L.T), dtype=L.dtype, device=gy.device) \
            if (ctx.needs_input_grad[0] or (ctx.fused and want_w)) else None
        if want_w:
            dWf = torch.empty((L.Dp, L.Cp, L.T), dtype=torch.float32, device=gy.device)
            dbf = torch.empty((L.Dp,), dtype=torch.float32, device=gy.device)
        if ctx.fused and want_w:
            # one pass over gy: dx and G = DFT(gy), then dW, db from the spectra
            gs = eqlin.empty_spectra(L.h, "gy", ctx.N, device=gy.device)
            eqlin.backward(L.h, gy2, saved, dx2, gs, dWf, dbf)
        else:
            if dx2 is not None:
                eqlin.backward_dx(L.h, gy2, dx2)
            if want_w:
                eqlin.backward_dw(L.h, saved, gy2, dWf, dbf)
        if ctx.needs_input_grad[0]:
            dx = dx2.reshape(*ctx.lead, L.Cp * L.T).to(ctx.x_dtype)
        if ctx.needs_input_grad[1]:
            dW = dWf.to(ctx.w_dtype)
        if ctx.needs_input_grad[2]:
            db = dbf.to(ctx.b_dtype)
        return dx, dW, db, None


class EQLinear(nn.Module):
    """Group-circulant linear layer: [..., C'*T] -> [..., D'*T].

    ``dtype`` is the compute dtype of the library handle (bf16, f16 or f32);
    the parameters are created in it.  Init: W and b uniform in
    +-1/sqrt(C'*T), as for an ordinary linear layer with C'*T inputs.
    """

    def __init__(self, Cp: int, Dp: int, T: int = 4, bias: bool = True, dtype=torch.bfloat16,
                 device="cuda", generator: torch.Generator | None = None):
        super().__init__()
        self.Cp, self.Dp, self.T, self.dtype = int(Cp), int(Dp), int(T), dtype
        bound = 1.0 / math.sqrt(Cp * T)
        w = (torch.rand((Dp, Cp, T), generator=generator) * 2 - 1) * bound
        self.weight = nn.Parameter(w.to(device=device, dtype=dtype))
        if bias:
            bb = (torch.rand((Dp,), generator=generator) * 2 - 1) * bound
            self.bias = nn.Parameter(bb.to(device=device, dtype=dtype))
        else:
            self.register_parameter("bias", None)
        self.h = eqlin.create(T, Cp, Dp, dtype)
        # the stash forms (fused backward) serve f16/bf16 layers of order T | 8
        # whose passes all run on tensor cores
        self.fused = (self.h.backend() == "fwd=tcgen05 dx=tcgen05 dw=tcgen05" and self.h.T in (1, 2, 4, 8)
                      and self.dtype != torch.float32)
        self._seen = None

    def sync_weights(self, W: torch.Tensor, b: torch.Tensor | None):
        """Run the weight transform if W or b changed since it last ran."""
        # the handle's identity too: a deep copy of the module gets a new,
        # empty handle and must load its weights again
        key = (id(self.h), W.data_ptr(), W._version, None if b is None else (b.data_ptr(), b._version))
        if key != self._seen:
            eqlin.set_weights(self.h, W.detach().to(self.dtype).contiguous(),
                              None if b is None else b.detach().to(self.dtype).contiguous())
            self._seen = key

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        return EQLinearFunction.apply(x, self.weight, self.bias, self)

    def extra_repr(self) -> str:
        return f"C'={self.Cp}, D'={self.Dp}, T={self.T}, dtype={self.dtype}, backend={self.h.backend()}"


class GroupLayerNorm(nn.Module):
    """LayerNorm over all C'*T features, with one scale and shift per channel
    c shared by its T group positions (so it commutes with a cyclic shift)."""

    def __init__(self, Cp: int, T: int, eps: float = 1e-6, dtype=torch.bfloat16, device="cuda"):
        super().__init__()
        self.Cp, self.T, self.eps = Cp, T, eps
        self.weight = nn.Parameter(torch.ones(Cp, dtype=dtype, device=device))
        self.bias = nn.Parameter(torch.zeros(Cp, dtype=dtype, device=device))

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        y = F.layer_norm(x, (self.Cp * self.T,), None, None, self.eps)
        y = y.view(*x.shape[:-1], self.Cp, self.T) * self.weight[:, None] + self.bias[:, None]
        return y.view(x.shape)


def _attention(h: torch.Tensor, heads: int, Cp: int, T: int) -> torch.Tensor:
    """Multi-head self-attention on qkv features [B, L, 3*C'*T]; heads split C'."""
    B, L, _ = h.shape
    q, k, v = h.view(B, L, 3, heads, (Cp // heads) * T).permute(2, 0, 3, 1, 4)
    o = F.scaled_dot_product_attention(q, k, v)
    return o.transpose(1, 2).reshape(B, L, Cp * T)


class EQViTBlock(nn.Module):
    """Pre-norm ViT block on features [B, L, C'*T] with EQ-Linear layers."""

    def __init__(self, Cp: int, heads: int, T: int = 4, mlp_ratio: int = 4, dtype=torch.bfloat16,
                 device="cuda", seed: int = 0):
        super().__init__()
        if Cp % heads:
            raise ValueError("heads must divide C'")
        g = torch.Generator().manual_seed(seed)
        self.Cp, self.T, self.heads = Cp, T, heads
        self.norm1 = GroupLayerNorm(Cp, T, dtype=dtype, device=device)
        self.qkv = EQLinear(Cp, 3 * Cp, T, dtype=dtype, device=device, generator=g)
        self.proj = EQLinear(Cp, Cp, T, dtype=dtype, device=device, generator=g)
        self.norm2 = GroupLayerNorm(Cp, T, dtype=dtype, device=device)
        self.fc1 = EQLinear(Cp, mlp_ratio * Cp, T, dtype=dtype, device=device, generator=g)
        self.fc2 = EQLinear(mlp_ratio * Cp, Cp, T, dtype=dtype, device=device, generator=g)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        x = x + self.proj(_attention(self.qkv(self.norm1(x)), self.heads, self.Cp, self.T))
        return x + self.fc2(F.gelu(self.fc1(self.norm2(x))))


def expand_dense(W: torch.Tensor) -> torch.Tensor:
    """The naive layer's matrix: W_dense[d*T+s, c*T+t] = W[d, c, (s-t) mod T]."""
    Dp, Cp, T = W.shape
    s = torch.arange(T, device=W.device)
    idx = (s[:, None] - s[None, :]) % T               # [s, t]
    return W[:, :, idx].permute(0, 2, 1, 3).reshape(Dp * T, Cp * T)


class DenseEQViTBlock(nn.Module):
    """The same block with every EQ-Linear applied as the expanded dense
    matrix (``F.linear``), sharing the parameters of ``src``.  Context only:
    the naive layer the pages measure against."""

    def __init__(self, src: EQViTBlock, dtype=None):
        super().__init__()
        self.src, self.dtype = src, dtype

    def _lin(self, layer: EQLinear, x: torch.Tensor) -> torch.Tensor:
        W, b = layer.weight, layer.bias
        if self.dtype is not None:
            W, b = W.to(self.dtype), None if b is None else b.to(self.dtype)
        return F.linear(x, expand_dense(W), None if b is None else b.repeat_interleave(layer.T))

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        s = self.src

        def norm(n, v):
            w, b = n.weight, n.bias
            if self.dtype is not None:
                w, b = w.to(self.dtype), b.to(self.dtype)
            y = F.layer_norm(v, (n.Cp * n.T,), None, None, n.eps)
            return (y.view(*v.shape[:-1], n.Cp, n.T) * w[:, None] + b[:, None]).view(v.shape)

        x = x + self._lin(s.proj, _attention(self._lin(s.qkv, norm(s.norm1, x)), s.heads, s.Cp, s.T))
        return x + self._lin(s.fc2, F.gelu(self._lin(s.fc1, norm(s.norm2, x))))


MODELS = {  # name: (C' at T = 4, heads); tokens per image 197 (224 x 224, patch 16)
    "eq-vit-s": (96, 6),
    "eq-vit-b": (192, 12),
}


def _time(fn, iters: int, warmup: int) -> float:
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def main(argv=None):
    ap = argparse.ArgumentParser(description="Time one synthetic EQ-ViT block, Flash EQ-Linear vs the dense matrix.")
    ap.add_argument("--model", default="eq-vit-b", choices=sorted(MODELS))
    ap.add_argument("--batch", type=int, default=64)
    ap.add_argument("--tokens", type=int, default=197)
    ap.add_argument("--dtype", default="bf16", choices=("bf16", "f16"))
    ap.add_argument("--iters", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    args = ap.parse_args(argv)
    dt = {"bf16": torch.bfloat16, "f16": torch.float16}[args.dtype]
    Cp, heads = MODELS[args.model]
    T = 4
    blk = EQViTBlock(Cp, heads, T, dtype=dt)
    dense = DenseEQViTBlock(blk)
    g = torch.Generator(device="cuda").manual_seed(1)
    x = torch.randn((args.batch, args.tokens, Cp * T), generator=g, device="cuda", dtype=dt, requires_grad=True)
    gy = torch.randn((args.batch, args.tokens, Cp * T), generator=g, device="cuda", dtype=dt)

    def fwd(m):
        with torch.no_grad():
            m(x)

    def fwd_bwd(m):
        m(x).backward(gy)

    out = {"model": args.model, "batch": args.batch, "tokens": args.tokens, "dtype": args.dtype, "T": T,
           "C_prime": Cp, "heads": heads, "unit": "ms", "weights": "synthetic (random)"}
    for name, m in (("flash", blk), ("dense_matrix", dense)):
        out[f"{name}_fwd_ms"] = _time(lambda: fwd(m), args.iters, args.warmup)
        out[f"{name}_fwd_bwd_ms"] = _time(lambda: fwd_bwd(m), args.iters, args.warmup)
    out["speedup_fwd"] = out["dense_matrix_fwd_ms"] / out["flash_fwd_ms"]
    out["speedup_fwd_bwd"] = out["dense_matrix_fwd_bwd_ms"] / out["flash_fwd_bwd_ms"]
    for layer in (blk.qkv, blk.proj, blk.fc1, blk.fc2):
        if eqlin.get_error(layer.h) != 0:
            raise RuntimeError("device-side timeout in an EQ-Linear kernel")
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
