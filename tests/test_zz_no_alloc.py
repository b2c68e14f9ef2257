"""eqlin_backward_dw_noalloc: dW/db without a handle and without allocation.

This entry point is for callers that cannot call cudaMalloc (another
allocator owns the device memory, or allocation is forbidden after start-up),
so they cannot create a handle either.  The test calls it through the C ABI
twice in a row, on different inputs, and compares each result with the CPU
oracle and with the handle-based eqlin_backward_dw, within the tolerance the
parity tests use.  It lives in a file of its own, collected last, and passes
both alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from _parity import check
from group_circulant_linear_b200 import eqlin, inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2   # relative Frobenius error for f16/bf16, as in the parity tests


def _noalloc(T, Cp, Dp, dt, x, gy, dW, db):
    L = eqlin.lib()
    s = torch.cuda.current_stream().cuda_stream
    vp = ctypes.c_void_p
    return L.eqlin_backward_dw_noalloc(T, Cp, Dp, eqlin._DT[dt], vp(x.data_ptr()), vp(gy.data_ptr()),
                                       vp(dW.data_ptr()), vp(db.data_ptr()) if db is not None else None,
                                       x.shape[0], vp(s))


@pytest.mark.parametrize("T,Cp,Dp,N,dt", [(4, 192, 768, 12608, torch.bfloat16),
                                          (2, 40, 72, 1000, torch.float16),
                                          (8, 64, 16, 333, torch.bfloat16)])
def test_noalloc_matches_oracle_and_handle_path_on_two_calls(T, Cp, Dp, N, dt):
    name = "bf16" if dt == torch.bfloat16 else "f16"
    dW = torch.full((Dp, Cp, T), float("nan"), device="cuda")
    db = torch.full((Dp,), float("nan"), device="cuda")
    for seed in (11, 12):                       # two calls in a row, different inputs
        inp = inputs.make_inputs(T, Cp, Dp, N, name, seed=seed)
        g = {k: v.cuda() for k, v in inp.items()}
        assert _noalloc(T, Cp, Dp, dt, g["x"], g["gy"], dW, db) == 0
        layer = eqlin.EQLinear(g["W"], g["b"])
        ref_dW, ref_db = layer.backward_dw(g["x"], g["gy"])
        torch.cuda.synchronize()
        assert eqlin.get_error(layer.h) == 0
        want_dW, want_db = oracle.backward_dw(inp["x"], inp["gy"], T, Cp, Dp)
        tag = f"noalloc T={T} C'={Cp} D'={Dp} N={N} {name} seed {seed}"
        check(f"{tag} dW vs oracle", dW, want_dW, TOL)
        check(f"{tag} db vs oracle", db, want_db, TOL)
        check(f"{tag} dW vs eqlin_backward_dw", dW, ref_dW, TOL)
        check(f"{tag} db vs eqlin_backward_dw", db, ref_db, TOL)


def test_noalloc_python_binding():
    """The binding derives C', D' and the dtype from the tensors and checks them."""
    T, Cp, Dp, N = 4, 64, 96, 700
    inp = inputs.make_inputs(T, Cp, Dp, N, "f16", seed=21)
    g = {k: v.cuda() for k, v in inp.items()}
    dW = torch.empty((Dp, Cp, T), device="cuda")
    db = torch.empty((Dp,), device="cuda")
    eqlin.backward_dw_noalloc(T, g["x"], g["gy"], dW, db)
    torch.cuda.synchronize()
    want_dW, want_db = oracle.backward_dw(inp["x"], inp["gy"], T, Cp, Dp)
    check("noalloc binding dW vs oracle", dW, want_dW, TOL)
    check("noalloc binding db vs oracle", db, want_db, TOL)
    with pytest.raises(TypeError):                       # gy of another dtype than x
        eqlin.backward_dw_noalloc(T, g["x"], g["gy"].bfloat16(), dW, db)
    with pytest.raises(ValueError):                      # gy with the wrong width
        eqlin.backward_dw_noalloc(T, g["x"], g["gy"][:, :-8].contiguous(), dW, db)
    with pytest.raises(ValueError):                      # db of the wrong length
        eqlin.backward_dw_noalloc(T, g["x"], g["gy"], dW, db[:-1])


def test_noalloc_rejects_what_it_cannot_serve():
    x = torch.zeros((4, 8 * 4), dtype=torch.bfloat16, device="cuda")
    dW = torch.zeros((8, 8, 4), device="cuda")
    assert _noalloc(4, 8, 8, torch.float32, x.float(), x.float(), dW, None) == -2   # f32
    assert _noalloc(3, 8, 8, torch.bfloat16, x, x, dW, None) == -2                 # T = 3
    # partial sums of a 2048 x 2048 p4 layer do not fit the fixed scratch
    big_x = torch.zeros((4, 2048 * 4), dtype=torch.bfloat16, device="cuda")
    big_dW = torch.zeros((2048, 2048, 4), device="cuda")
    assert _noalloc(4, 2048, 2048, torch.bfloat16, big_x, big_x, big_dW, None) == -2
    # N = 0 zeroes the outputs
    dW.fill_(5.0)
    db = torch.full((8,), 5.0, device="cuda")
    assert _noalloc(4, 8, 8, torch.bfloat16, x[:0], x[:0], dW, db) == 0
    torch.cuda.synchronize()
    assert not dW.any() and not db.any()
