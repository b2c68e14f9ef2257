"""GPU parity of the dihedral-group layer against the oracle's group functions.

The layer over D_m (element r^a s^f at group index f*m + a) is the group
convolution y[d, g] = b[d] + sum_c sum_h W[d, c, h^-1 g] x[c, h]; the library
evaluates it by the Fourier transform over D_m's irreducible representations
in FP32 CUDA-core kernels.  Tolerances as for the cyclic layer (relative
Frobenius norm: FP32 1e-5, FP16/BF16 inputs 2e-2); for m in {1, 2, 4} every
irrep entry is 0 or +-1 and the inverse scales are powers of two, so integer
inputs give results that must match bit for bit.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from _parity import TOL, check, check_exact
from group_circulant_linear_b200 import eqlin, inputs

pytestmark = pytest.mark.gpu


def _roll_group(v, ch, tab, u):
    mul, inv = tab
    G = inv.shape[0]
    return v.reshape(v.shape[0], ch, G)[:, :, torch.as_tensor(mul[inv[u]], device=v.device)].reshape(v.shape[0], -1)


def _run(m, inp):
    g = {k: v.cuda() for k, v in inp.items()}
    layer = eqlin.EQLinear(g["W"], g["b"], group="dihedral")
    assert layer.h.backend() == "fwd=simt dx=simt dw=simt"
    y = layer.forward(g["x"])
    dx = layer.backward_dx(g["gy"])
    dW, db = layer.backward_dw(g["x"], g["gy"])
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == 0
    return layer, g, {"y": y, "dx": dx, "dW": dW, "db": db}


CASES = [  # (m, C', D', N, dtype)
    (4, 16, 24, 300, "f32"), (4, 32, 16, 129, "bf16"), (4, 24, 40, 200, "f16"),
    (2, 32, 32, 257, "f32"), (3, 16, 24, 130, "f32"), (3, 16, 8, 100, "bf16"),
    (6, 8, 16, 131, "f32"), (8, 8, 8, 70, "f32"), (8, 8, 16, 65, "f16"), (1, 16, 16, 100, "f32"),
    (5, 8, 8, 64, "f32"),
]


@pytest.mark.parametrize("m,Cp,Dp,N,dt", CASES, ids=lambda v: str(v))
def test_dihedral_parity(m, Cp, Dp, N, dt):
    G = 2 * m
    inp = inputs.make_inputs(G, Cp, Dp, N, dt, seed=31)
    tab = oracle.dihedral_table(m)
    _, _, out = _run(m, inp)
    tol = TOL[dt]
    tag = f"D_{m} C'={Cp} D'={Dp} N={N} {dt}"
    check(f"{tag} y", out["y"], oracle.forward_group(inp["x"], inp["W"], inp["b"], tab), tol)
    check(f"{tag} dx", out["dx"], oracle.backward_dx_group(inp["gy"], inp["W"], tab), tol)
    dW, db = oracle.backward_dw_group(inp["x"], inp["gy"], tab, Cp, Dp)
    check(f"{tag} dW", out["dW"], dW, tol)
    check(f"{tag} db", out["db"], db, tol)


@pytest.mark.parametrize("m,Cp,Dp,N,dt", [(4, 16, 16, 1000, "f32"), (4, 8, 8, 300, "bf16"), (2, 16, 24, 500, "f16"),
                                          (1, 16, 16, 200, "f32")], ids=lambda v: str(v))
def test_dihedral_integer_inputs_bit_exact(m, Cp, Dp, N, dt):
    inp = inputs.make_integer_inputs(2 * m, Cp, Dp, N, dt, seed=5, amp=2)
    tab = oracle.dihedral_table(m)
    _, _, out = _run(m, inp)
    tag = f"integer D_{m} C'={Cp} D'={Dp} N={N} {dt}"
    check_exact(f"{tag} y", out["y"], oracle.forward_group(inp["x"], inp["W"], inp["b"], tab))
    check_exact(f"{tag} dx", out["dx"], oracle.backward_dx_group(inp["gy"], inp["W"], tab))
    dW, db = oracle.backward_dw_group(inp["x"], inp["gy"], tab, Cp, Dp)
    check_exact(f"{tag} dW", out["dW"], dW)
    check_exact(f"{tag} db", out["db"], db)


@pytest.mark.parametrize("m", [3, 4])
def test_dihedral_equivariance_on_gpu(m):
    """Acting on x with any group element u acts on y the same way."""
    Cp, Dp, N = 8, 16, 200
    inp = inputs.make_inputs(2 * m, Cp, Dp, N, "f32", seed=33)
    tab = oracle.dihedral_table(m)
    layer, g, out = _run(m, inp)
    for u in range(2 * m):
        yu = layer.forward(_roll_group(g["x"], Cp, tab, u))
        check(f"D_{m} equivariance u={u}", yu, _roll_group(out["y"], Dp, tab, u), 1e-5)


def test_dihedral_rejects_stash_forms():
    h = eqlin.create_group("dihedral", 4, 8, 8, torch.bfloat16)
    eqlin.set_weights(h, torch.zeros((8, 8, 8), device="cuda", dtype=torch.bfloat16), None)
    x = torch.zeros((4, 64), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(eqlin.EqlinError):
        eqlin.forward_stash(h, x, torch.empty_like(x), eqlin.empty_spectra(h, "x", 4))
    h.close()
