"""Synthetic workload shapes and the work/traffic accounting of one layer.

The shapes stand in for the layers the paper accelerates (EQ-ViT and EQ-Swin
on 224x224 inputs: 197 tokens per image for ViT/16, a 56x56 stage-1 grid for
Swin-T), with the p4 group (T=4) and a cyclic-group sweep.  No dataset or
trained weight is involved; values come from ``inputs.make_inputs``.

Counting conventions ("Flash EQ-Linear", technical summary, sections
"Abordagem Algoritmica" and "Especializacao para o Grupo de Rotacao p4"):

* R(T) real per-frequency GEMMs of N x C' x D': one for each real frequency
  (k=0, and k=T/2 when T is even) and four for each complex frequency of the
  half spectrum.  R(4) = 6, against the T*T = 16 of the unrolled dense matrix.
* dense-equivalent FLOP of one pass = 2*N*C*D (C = C'*T, D = D'*T), the work
  of the unrolled dense layer; "actual" FLOP = 2*R(T)*N*C'*D'.
"""
from __future__ import annotations

from dataclasses import dataclass, field


def real_gemms(T: int) -> int:
    """R(T): real GEMMs per layer on the non-redundant half spectrum."""
    if T < 1:
        raise ValueError("T must be >= 1")
    n_real = 1 if T % 2 else 2           # k = 0, plus k = T/2 for even T
    n_complex = (T - n_real) // 2        # frequencies 1 .. ceil(T/2)-1
    return n_real + 4 * n_complex


BYTES = {"f32": 4, "f16": 2, "bf16": 2}


@dataclass(frozen=True)
class Layer:
    name: str
    T: int
    Cp: int
    Dp: int
    N: int
    dtype: str
    passes: tuple = ("fwd",)            # subset of ("fwd", "dx", "dw")

    @property
    def C(self) -> int:
        return self.Cp * self.T

    @property
    def D(self) -> int:
        return self.Dp * self.T

    def dense_flop(self) -> int:
        """2*N*C*D per pass (what the unrolled dense layer computes)."""
        return 2 * self.N * self.C * self.D

    def actual_flop(self) -> int:
        """2*R(T)*N*C'*D' per pass (the per-frequency GEMMs only)."""
        return 2 * real_gemms(self.T) * self.N * self.Cp * self.Dp

    def bytes_fwd(self) -> int:
        """Algorithmic bytes of a forward (or dx) pass: read input, write
        output, read the R(T) Fourier weight planes and the bias once."""
        e = BYTES[self.dtype]
        return (self.N * self.C * e + self.N * self.D * e
                + real_gemms(self.T) * self.Cp * self.Dp * e + 4 * self.Dp)

    def bytes_dw(self) -> int:
        """Algorithmic bytes of the dW/db pass: read x and gy once, write
        the FP32 dW [D', C', T] and db [D']."""
        e = BYTES[self.dtype]
        return (self.N * self.C * e + self.N * self.D * e
                + 4 * self.Dp * self.Cp * self.T + 4 * self.Dp)


def _vit_s(N=64 * 197):
    return [Layer("EQ-ViT-S qkv", 4, 96, 288, N, "f16", ("fwd",)),
            Layer("EQ-ViT-S proj", 4, 96, 96, N, "f16", ("fwd",))]


def _vit_b(N=64 * 197, dtype="bf16"):
    p = ("fwd", "dx", "dw")
    return [Layer("EQ-ViT-B fc1", 4, 192, 768, N, dtype, p),
            Layer("EQ-ViT-B fc2", 4, 768, 192, N, dtype, p)]


def _swin_t(N=128 * 56 * 56):
    p = ("fwd", "dx", "dw")
    return [Layer("EQ-Swin-T s1 fc1", 4, 24, 96, N, "f16", p),
            Layer("EQ-Swin-T s1 fc2", 4, 96, 24, N, "f16", p)]


def _sweep(N=16384, C=1024):
    p = ("fwd", "dx", "dw")
    out = []
    for dtype in ("f32", "f16"):
        for T in (2, 4, 8):
            out.append(Layer(f"cyclic T={T} {dtype}", T, C // T, C // T, N, dtype, p))
    return out


# The five workloads, named by what they are.
WORKLOADS = {
    "p4-tiny-f32-fwd": [Layer("p4 tiny", 4, 16, 16, 256, "f32", ("fwd",))],
    "eq-vit-s-f16-fwd": _vit_s(),
    "eq-vit-b-mlp-bf16-fwdbwd": _vit_b(),
    "eq-swin-t-s1-f16-fwdbwd": _swin_t(),
    "cyclic-sweep-fwdbwd": _sweep(),
}

# The workload the benchmark times by default: p4 fwd+bwd at EQ-ViT-B MLP
# shapes (fc1 768->3072 and fc2 3072->768, 64 images x 197 tokens).
DEFAULT_BENCH = "eq-vit-b-mlp-bf16-fwdbwd"
