"""GPU parity: the CUDA library against the CPU oracle on the same seeded inputs.

Tolerances (relative Frobenius norm of the difference, i.e. RMS(err)/RMS(ref)):
FP32 1e-5; FP16/BF16 with FP32 accumulation 2e-2.  Integer-valued inputs
whose every intermediate is exactly representable must match bit for bit
(T in {1, 2, 4}: the p4 and T=2 transforms use only +-1 and +-1/2, +-1/4).
Every comparison records the error it achieved (tests/_parity.py).

Coverage:
* small cases that span several 128-token tiles with a ragged tail;
* bit-exact integer cases, including ones whose persistent grid runs three
  or more output tiles per CTA (accumulator double-buffer phase flips, ring
  wrap-around) and dW splits of many token stages;
* every full-size workload in the benchmark's launch path: the EQ-ViT-S,
  EQ-ViT-B and EQ-Swin-T layers compared on every output element (y, dx, dW,
  db); the cyclic sweep on one token row of every 128-token tile and on
  sampled (d, c) pairs of every 128 x 128 weight block; plus the
  equivariance property on the whole output.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from _parity import TOL, Accum, check, check_exact, finish
from group_circulant_linear_b200 import eqlin, inputs, workloads

pytestmark = pytest.mark.gpu


def _dev(d):
    return {k: v.cuda() for k, v in d.items()}


def _fused_capable(T, Cp, Dp, dt) -> bool:
    """The stash forms serve f16/bf16 layers whose passes all run on tensor cores."""
    return dt != "f32" and T in (1, 2, 4, 8) and Cp % 8 == 0 and Dp % 8 == 0


def _run_fused(layer, g):
    """Forward with the input's spectrum stashed, then the one-call backward
    (dx with G stashed, dW/db from the two spectra)."""
    h = layer.h
    N = g["x"].shape[0]
    xs = eqlin.empty_spectra(h, "x", N)
    gs = eqlin.empty_spectra(h, "gy", N)
    y = torch.empty((N, h.Dp * h.T), dtype=h.dtype, device="cuda")
    dx = torch.empty((N, h.Cp * h.T), dtype=h.dtype, device="cuda")
    dW = torch.full((h.Dp, h.Cp, h.T), float("nan"), device="cuda")
    db = torch.full((h.Dp,), float("nan"), device="cuda")
    eqlin.forward_stash(h, g["x"], y, xs)
    eqlin.backward(h, g["gy"], xs, dx, gs, dW, db)
    torch.cuda.synchronize()
    assert eqlin.get_error(h) == 0
    return {"y": y, "dx": dx, "dW": dW, "db": db, "xs": xs, "gs": gs}


def _spectrum(v: np.ndarray, ch: int, T: int) -> np.ndarray:
    """[T planes, ch, N] real planes of the DFT along the group axis of v [N, ch*T],
    from numpy's real FFT: Re V_0, Re V_{T/2} (even T), then Re V_k, Im V_k."""
    F = np.fft.rfft(np.asarray(v, dtype=np.float64).reshape(-1, ch, T), axis=-1)
    planes = [F[..., 0].real] + ([F[..., T // 2].real] if T % 2 == 0 else [])
    for k in range(1, (T + 1) // 2):
        planes += [F[..., k].real, F[..., k].imag]
    return np.stack(planes).transpose(0, 2, 1)


def _run_all(T, Cp, Dp, dt, inp, passes=("fwd", "dx", "dw"), split=False):
    g = _dev(inp)
    layer = eqlin.EQLinear(g["W"], g["b"])
    if split:
        eqlin.set_tail_split(layer.h, True)
    out = {}
    if "fwd" in passes:
        out["y"] = layer.forward(g["x"])
    if "dx" in passes:
        out["dx"] = layer.backward_dx(g["gy"])
    if "dw" in passes:
        out["dW"], out["db"] = layer.backward_dw(g["x"], g["gy"])
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == 0
    return layer, {k: v.float().cpu().numpy() for k, v in out.items()}


SMALL = [  # (T, C', D', N, dtype)
    (4, 16, 16, 256, "f32"),        # p4 tiny forward
    (4, 96, 288, 333, "f16"),       # EQ-ViT-S qkv-like, ragged N
    (4, 96, 96, 300, "f16"),        # EQ-ViT-S proj-like
    (4, 192, 768, 300, "bf16"),     # EQ-ViT-B fc1-like
    (4, 768, 192, 260, "bf16"),     # EQ-ViT-B fc2-like
    (4, 24, 96, 1000, "f16"),       # EQ-Swin-T stage-1 fc1-like
    (4, 96, 24, 1000, "f16"),       # EQ-Swin-T stage-1 fc2-like
    (2, 64, 64, 257, "f32"), (4, 64, 64, 257, "f32"), (8, 32, 32, 257, "f32"),
    (2, 64, 64, 257, "f16"), (4, 64, 64, 257, "f16"), (8, 32, 32, 257, "f16"),
    (1, 64, 48, 200, "f32"), (1, 64, 48, 200, "bf16"),
    (8, 64, 16, 130, "bf16"), (2, 40, 72, 129, "bf16"),
    (4, 8, 8, 1, "f16"), (4, 200, 40, 131, "f16"),
    # T = 3 and 6: sqrt(3)/2 twiddles, one real frequency for odd T (tensor cores
    # for f16/bf16 with 8-aligned channels, SIMT otherwise), several tiles per CTA
    (3, 64, 48, 257, "f32"), (6, 32, 40, 130, "f32"), (3, 40, 64, 300, "bf16"), (6, 48, 24, 200, "f16"),
    (3, 192, 768, 3000, "bf16"), (3, 768, 192, 1000, "f16"), (6, 128, 256, 5000, "f16"), (6, 256, 64, 777, "bf16"),
    (3, 24, 96, 4000, "f16"), (6, 96, 24, 3000, "bf16"),
    (6, 20, 36, 300, "bf16"),       # K not a multiple of 8: forward and dx on the SIMT kernels
    # FP32 on the tensor cores (3xTF32) for T = 1, 2, 4: every tile width
    # (T = 4: 64 and 32), several output tiles per persistent CTA, ragged N,
    # and K not a multiple of the 8-channel stage (zero-filled tail)
    (4, 64, 128, 40000, "f32"), (4, 40, 96, 20000, "f32"), (2, 128, 256, 30000, "f32"),
    (1, 256, 512, 20000, "f32"), (4, 20, 36, 300, "f32"), (2, 6, 10, 130, "f32"), (1, 12, 20, 99, "f32"),
    # FP32 dW with c on the MMA's M side (C' a multiple of 128, D' not)
    (2, 128, 72, 5000, "f32"), (4, 128, 40, 9000, "f32"),
    # FP32 dW N sides wider than 128 channels (two per transform thread; with
    # d on the N side, db from rows past 128), and token ranges of two passes
    (2, 256, 128, 5000, "f32"), (2, 128, 200, 3000, "f32"),
    (2, 128, 128, 160000, "f32"), (1, 128, 128, 160000, "f32"),
    # FP32 dW over more than four waves of token chunks: two passes, the
    # second adding to the first's partial planes
    (2, 16, 24, 700000, "f32"),
    # FP32 T = 8 forward and dx on 3xTF32 (one operand slot, all transform
    # warps on every stage): several tiles per CTA, and K not a multiple of 8
    (8, 128, 96, 20000, "f32"), (8, 20, 12, 300, "f32"),
]


@pytest.mark.parametrize("T,Cp,Dp,N,dt", SMALL, ids=lambda v: str(v))
def test_small_parity(T, Cp, Dp, N, dt):
    inp = inputs.make_inputs(T, Cp, Dp, N, dt, seed=0)
    _, out = _run_all(T, Cp, Dp, dt, inp)
    y = oracle.forward(inp["x"], inp["W"], inp["b"])
    dx = oracle.backward_dx(inp["gy"], inp["W"])
    dW, db = oracle.backward_dw(inp["x"], inp["gy"], T, Cp, Dp)
    tol = TOL[dt]
    tag = f"small T={T} C'={Cp} D'={Dp} N={N} {dt}"
    check(f"{tag} y", out["y"], y, tol)
    check(f"{tag} dx", out["dx"], dx, tol)
    check(f"{tag} dW", out["dW"], dW, tol)
    check(f"{tag} db", out["db"], db, tol)


# (T, C', D', N, dtype, amp): integer inputs in [-amp, amp] whose every
# intermediate is exactly representable, so the result must equal the
# oracle's exactly.  Bounds: y and dx are at most K*T*amp^2 + 1 in magnitude
# (K = C' or D'), below 2^11 for f16 and 2^8 for bf16; the transformed
# operands at most T*amp; every dW partial sum at most N*(T*amp)^2 <= 2^24,
# exact in the FP32 accumulator.
EXACT = [
    (4, 64, 64, 1024, "f32", 4), (2, 64, 48, 515, "f32", 4), (1, 32, 64, 300, "f32", 4),
    # FP32 dW over three waves of token chunks, and over two passes (the
    # second adds to the first's partials)
    (4, 64, 64, 100000, "f32", 1), (4, 16, 16, 250000, "f32", 1),
    # FP32 dW with N sides past 128 channels (two rows per transform thread;
    # T = 1 with 16-token stages)
    (2, 200, 256, 2000, "f32", 2), (1, 160, 256, 1500, "f32", 2),
    # f16 dW chunks of 27 stages: the two transform groups, on alternate
    # stages, take 14 and 13
    (4, 16, 16, 63936, "f16", 2),
    (4, 16, 16, 700, "f16", 4), (2, 16, 16, 300, "f16", 4), (4, 16, 8, 129, "f16", 4),
    (4, 8, 8, 400, "bf16", 2), (2, 8, 8, 200, "bf16", 2),
    # 512 token tiles: 3-4 output tiles per persistent CTA of the forward and
    # dx kernels, the dW token split over 147 chunks of 28 stages each
    (4, 16, 16, 65536, "f16", 2),        # BO = 32 both ways (double-buffered accumulator)
    (4, 16, 128, 65536, "f16", 2),       # forward BO = 128 (single accumulator), dx BO = 32
    (4, 16, 96, 65536, "f16", 2),        # forward BO = 96
    (4, 128, 16, 65536, "f16", 1),       # dx BO = 128, dW with c on the MMA's M side
    (2, 16, 16, 65536, "f16", 2), (1, 16, 32, 65536, "f16", 2),
    (4, 8, 8, 65536, "bf16", 2),
]


@pytest.mark.parametrize("T,Cp,Dp,N,dt,amp", EXACT, ids=lambda v: str(v))
def test_integer_inputs_bit_exact(T, Cp, Dp, N, dt, amp):
    inp = inputs.make_integer_inputs(T, Cp, Dp, N, dt, seed=3, amp=amp)
    _, out = _run_all(T, Cp, Dp, dt, inp)
    y = oracle.forward(inp["x"], inp["W"], inp["b"])
    dx = oracle.backward_dx(inp["gy"], inp["W"])
    dW, db = oracle.backward_dw(inp["x"], inp["gy"], T, Cp, Dp)
    tag = f"integer T={T} C'={Cp} D'={Dp} N={N} {dt}"
    check_exact(f"{tag} y", out["y"], y)
    check_exact(f"{tag} dx", out["dx"], dx)
    check_exact(f"{tag} dW", out["dW"], dW)
    check_exact(f"{tag} db", out["db"], db)
    if _fused_capable(T, Cp, Dp, dt):
        layer = eqlin.EQLinear(*(t.cuda() for t in (inp["W"], inp["b"])))
        f = _run_fused(layer, _dev(inp))
        check_exact(f"{tag} fused y", f["y"], y)
        check_exact(f"{tag} fused dx", f["dx"], dx)
        check_exact(f"{tag} fused dW", f["dW"], dW)
        check_exact(f"{tag} fused db", f["db"], db)
        # integer inputs have integer spectra for T in {1, 2, 4} (twiddles 0, +-1):
        # exact in the operand type; the FFT's rounding noise is removed by rint
        check_exact(f"{tag} stashed X", f["xs"][..., :N], np.rint(_spectrum(inp["x"].double().numpy(), Cp, T)))
        check_exact(f"{tag} stashed G", f["gs"][..., :N], np.rint(_spectrum(inp["gy"].double().numpy(), Dp, T)))


# The p4 forward with the complex products as three real GEMMs (Gauss): against
# the oracle (random inputs within the FP16/BF16 tolerance, integer inputs bit
# for bit: Re X + Im X, Im W - Re W and Re W + Im W stay exact there), and
# several tiles per CTA at N = 65536.
GAUSS = [  # (C', D', N, dtype)
    (192, 768, 1000, "bf16"), (768, 192, 777, "bf16"), (96, 288, 333, "f16"), (64, 96, 700, "bf16"),
    (24, 96, 3000, "f16"), (16, 40, 129, "f16"),
]
GAUSS_EXACT = [  # (C', D', N, dtype, amp)
    (16, 16, 700, "f16", 4), (16, 96, 65536, "f16", 2), (16, 64, 65536, "f16", 2), (8, 32, 300, "bf16", 1),
]


def _gauss_forward(inp):
    g = _dev(inp)
    layer = eqlin.EQLinear(g["W"], g["b"])
    N = g["x"].shape[0]
    y = torch.empty((N, layer.h.Dp * 4), dtype=layer.h.dtype, device="cuda")
    eqlin.forward_gauss(layer.h, g["x"], y)
    y4 = layer.forward(g["x"])
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == 0
    return y.float().cpu().numpy(), y4.float().cpu().numpy()


@pytest.mark.parametrize("Cp,Dp,N,dt", GAUSS, ids=lambda v: str(v))
def test_gauss_forward(Cp, Dp, N, dt):
    inp = inputs.make_inputs(4, Cp, Dp, N, dt, seed=11, with_gy=False)
    y3, y4 = _gauss_forward(inp)
    ref = oracle.forward(inp["x"], inp["W"], inp["b"])
    tag = f"gauss T=4 C'={Cp} D'={Dp} N={N} {dt}"
    check(f"{tag} y", y3, ref, TOL[dt])
    check(f"{tag} y (four-product form)", y4, ref, TOL[dt])


@pytest.mark.parametrize("Cp,Dp,N,dt,amp", GAUSS_EXACT, ids=lambda v: str(v))
def test_gauss_forward_integer_exact(Cp, Dp, N, dt, amp):
    inp = inputs.make_integer_inputs(4, Cp, Dp, N, dt, seed=13, amp=amp)
    y3, _ = _gauss_forward(inp)
    check_exact(f"gauss integer T=4 C'={Cp} D'={Dp} N={N} {dt} y", y3, oracle.forward(inp["x"], inp["W"], inp["b"]))


@pytest.mark.parametrize("Cp,Dp,N", [(256, 96, 3000), (272, 64, 20000)], ids=lambda v: str(v))
def test_gauss_forward_tail_split(Cp, Dp, N):
    # the three-product forward with the tail split on (five accumulator planes,
    # 480 or 320 columns handed over): integer inputs, bit for bit
    inp = inputs.make_integer_inputs(4, Cp, Dp, N, "f16", seed=17, amp=1)
    g = _dev(inp)
    layer = eqlin.EQLinear(g["W"], g["b"])
    eqlin.set_tail_split(layer.h, True)
    y = torch.empty((N, Dp * 4), dtype=torch.float16, device="cuda")
    eqlin.forward_gauss(layer.h, g["x"], y)
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == 0
    check_exact(f"gauss split C'={Cp} D'={Dp} N={N} y", y, oracle.forward(inp["x"], inp["W"], inp["b"]))


def test_gauss_forward_rejects_what_it_cannot_serve():
    for T, dt in ((2, torch.bfloat16), (8, torch.float16), (4, torch.float32)):
        h = eqlin.create(T, 16, 16, dt)
        W = torch.zeros((16, 16, T), dtype=dt, device="cuda")
        eqlin.set_weights(h, W, None)
        x = torch.zeros((4, 16 * T), dtype=dt, device="cuda")
        y = torch.empty((4, 16 * T), dtype=dt, device="cuda")
        with pytest.raises(eqlin.EqlinError):
            eqlin.forward_gauss(h, x, y)
        h.close()


FUSED = [  # (T, C', D', N, dtype): the stash forms and the one-call backward
    (4, 192, 768, 1000, "bf16"), (4, 768, 192, 777, "bf16"), (4, 24, 96, 3000, "f16"),
    (4, 96, 24, 3000, "f16"), (4, 96, 288, 333, "f16"), (2, 64, 48, 515, "bf16"),
    (8, 64, 16, 257, "f16"), (1, 64, 48, 200, "bf16"), (4, 8, 8, 1, "f16"), (4, 200, 40, 131, "f16"),
]


@pytest.mark.parametrize("T,Cp,Dp,N,dt", FUSED, ids=lambda v: str(v))
def test_fused_backward(T, Cp, Dp, N, dt):
    inp = inputs.make_inputs(T, Cp, Dp, N, dt, seed=9)
    g = _dev(inp)
    layer = eqlin.EQLinear(g["W"], g["b"])
    f = _run_fused(layer, g)
    plain_y, plain_dx = layer.forward(g["x"]), layer.backward_dx(g["gy"])
    torch.cuda.synchronize()
    tag = f"fused T={T} C'={Cp} D'={Dp} N={N} {dt}"
    # the stash forms run the same kernels: identical outputs
    check_exact(f"{tag} y vs eqlin_forward", f["y"], plain_y)
    check_exact(f"{tag} dx vs eqlin_backward_dx", f["dx"], plain_dx)
    tol = TOL[dt]
    check(f"{tag} y", f["y"], oracle.forward(inp["x"], inp["W"], inp["b"]), tol)
    check(f"{tag} dx", f["dx"], oracle.backward_dx(inp["gy"], inp["W"]), tol)
    dW, db = oracle.backward_dw(inp["x"], inp["gy"], T, Cp, Dp)
    check(f"{tag} dW", f["dW"], dW, tol)
    check(f"{tag} db", f["db"], db, tol)
    # the spectra themselves, against numpy's FFT of the same inputs
    check(f"{tag} stashed X", f["xs"][..., :N], _spectrum(inp["x"].double().numpy(), Cp, T), tol)
    check(f"{tag} stashed G", f["gs"][..., :N], _spectrum(inp["gy"].double().numpy(), Dp, T), tol)
    # dW from the spectra alone equals the one-call backward's
    dW2 = torch.empty_like(f["dW"])
    db2 = torch.empty_like(f["db"])
    eqlin.backward_dw_spectra(layer.h, f["xs"], f["gs"], N, dW2, db2)
    torch.cuda.synchronize()
    check_exact(f"{tag} dW_spectra vs eqlin_backward", dW2, f["dW"])
    check_exact(f"{tag} db_spectra vs eqlin_backward", db2, f["db"])
    assert eqlin.get_error(layer.h) == 0


# Tail split (eqlin_set_tail_split; reductions of 16+ stages): the last
# wave's tiles run as two parts of the reduction, stages [0, 3K/8) and the
# rest, and the part that finishes second adds the other's FP32 accumulator.
# (T, C', D', N, dtype, amp): amp > 0 integer inputs, compared bit for bit
# (bounds as for EXACT); amp = 0 random inputs within the dtype's tolerance.
# 160 tiles = one wave + 12 split tiles; 40-71 tiles all split; odd stage
# counts (K = 264: 17 stages, parts of 6 and 11); T = 3, 6 (no stash form).
SPLIT = [
    (4, 256, 96, 20480, "f16", 1), (4, 256, 16, 5120, "f16", 1), (4, 16, 256, 5120, "f16", 1),
    (4, 264, 16, 3000, "f16", 1), (2, 512, 16, 9000, "f16", 1), (1, 512, 32, 4000, "f16", 1),
    (4, 256, 96, 20480, "bf16", 0), (4, 96, 264, 6000, "bf16", 0), (2, 320, 128, 9000, "f16", 0),
    (8, 256, 32, 3000, "bf16", 0), (3, 768, 192, 3000, "f16", 0), (6, 256, 64, 3000, "bf16", 0),
]


@pytest.mark.parametrize("T,Cp,Dp,N,dt,amp", SPLIT, ids=lambda v: str(v))
def test_tail_split(T, Cp, Dp, N, dt, amp):
    inp = (inputs.make_integer_inputs(T, Cp, Dp, N, dt, seed=3, amp=amp) if amp
           else inputs.make_inputs(T, Cp, Dp, N, dt, seed=0))
    layer, out = _run_all(T, Cp, Dp, dt, inp, passes=("fwd", "dx"), split=True)
    y = oracle.forward(inp["x"], inp["W"], inp["b"])
    dx = oracle.backward_dx(inp["gy"], inp["W"])
    tag = f"split T={T} C'={Cp} D'={Dp} N={N} {dt}"
    if amp:
        check_exact(f"{tag} y", out["y"], y)
        check_exact(f"{tag} dx", out["dx"], dx)
    else:
        check(f"{tag} y", out["y"], y, TOL[dt])
        check(f"{tag} dx", out["dx"], dx, TOL[dt])
    if _fused_capable(T, Cp, Dp, dt):
        # the stash forms split the same tiles: identical outputs
        g = _dev(inp)
        f = _run_fused(layer, g)
        check_exact(f"{tag} stash y vs split forward", f["y"], out["y"])
        check_exact(f"{tag} stash dx vs split dx", f["dx"], out["dx"])
    # switched off again, the same handle computes whole tiles
    eqlin.set_tail_split(layer.h, False)
    g = _dev(inp)
    y0 = layer.forward(g["x"])
    torch.cuda.synchronize()
    if amp:
        check_exact(f"{tag} y unsplit", y0, y)
    else:
        check(f"{tag} y unsplit", y0, y, TOL[dt])


@pytest.mark.parametrize("T,Cp,Dp,N,dt", [(4, 768, 192, 12608, "bf16"), (4, 264, 96, 3000, "f16"),
                                          (3, 768, 192, 3000, "f16")], ids=lambda v: str(v))
def test_split_tiles_repeatable(T, Cp, Dp, N, dt):
    # the split tiles' hand-over state is reset by each launch: back-to-back
    # forwards and dx give identical results, whichever part of a pair
    # finished first
    inp = inputs.make_inputs(T, Cp, Dp, N, dt, seed=21)
    g = _dev(inp)
    layer = eqlin.EQLinear(g["W"], g["b"])
    eqlin.set_tail_split(layer.h, True)
    ys = [layer.forward(g["x"]) for _ in range(6)]
    dxs = [layer.backward_dx(g["gy"]) for _ in range(4)]
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == 0
    for i in range(1, len(ys)):
        check_exact(f"split forward run {i}", ys[i], ys[0])
    for i in range(1, len(dxs)):
        check_exact(f"split dx run {i}", dxs[i], dxs[0])
    # the split tiles are the last ones (the last token blocks): the oracle on
    # the last 300 rows
    tail = slice(N - 300, N)
    check("split forward", ys[0][tail], oracle.forward(inp["x"][tail], inp["W"], inp["b"]), TOL[dt])
    if T in (1, 2, 4, 8):
        f = _run_fused(layer, g)
        check_exact("split forward, stash form", f["y"], ys[0])


def test_tail_split_switch():
    # FP32 and dihedral handles accept the switch and compute as before; an
    # f16 handle switches on and off repeatedly
    for T, dt, grp in ((4, "f32", "cyclic"), (2, "bf16", "dihedral"), (4, "f16", "cyclic")):
        inp = inputs.make_inputs(T, 256, 32, 700, dt, seed=2)
        g = _dev(inp)
        layer = eqlin.EQLinear(g["W"], g["b"], group=grp) if grp == "dihedral" else eqlin.EQLinear(g["W"], g["b"])
        for on in (True, False, True, True, False):
            eqlin.set_tail_split(layer.h, on)
        eqlin.set_tail_split(layer.h, True)
        y = layer.forward(g["x"])
        torch.cuda.synchronize()
        assert eqlin.get_error(layer.h) == 0
        if grp == "cyclic":
            check(f"switch T={T} {dt} y", y, oracle.forward(inp["x"], inp["W"], inp["b"]), TOL[dt])
        layer.h.close()


def test_stash_forms_reject_what_they_cannot_serve():
    h32 = eqlin.create(4, 16, 16, "f32")
    W = torch.zeros((16, 16, 4), device="cuda")
    eqlin.set_weights(h32, W, None)
    x = torch.zeros((10, 64), device="cuda")
    with pytest.raises(eqlin.EqlinError):
        eqlin.forward_stash(h32, x, torch.empty_like(x), eqlin.empty_spectra(h32, "x", 10))
    h3 = eqlin.create(3, 16, 16, "bf16")
    eqlin.set_weights(h3, torch.zeros((16, 16, 3), device="cuda", dtype=torch.bfloat16), None)
    xb = torch.zeros((10, 48), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(eqlin.EqlinError):
        eqlin.forward_stash(h3, xb, torch.empty_like(xb), eqlin.empty_spectra(h3, "x", 10))
    assert eqlin.spectra_ld(0) == 0 and eqlin.spectra_ld(1) == 64 and eqlin.spectra_ld(129) == 192
    h32.close()
    h3.close()


def test_back_to_back_dependencies():
    """Kernels launched back to back may start their prologue under the
    previous kernel's tail; each must still read its predecessor's output
    (read after write) and must not overwrite a buffer an earlier kernel
    reads (write after read).  Chain: x -L1-> y1 -L2-> y2 -L2dx-> g1
    -L1dx-> x (overwriting the x that the first kernel read)."""
    T, C1, C2, N = 4, 64, 96, 1000
    a = inputs.make_inputs(T, C1, C2, N, "bf16", seed=7)
    b = inputs.make_inputs(T, C2, C1, N, "bf16", seed=8)
    ga, gb = _dev(a), _dev(b)
    L1 = eqlin.EQLinear(ga["W"], ga["b"])
    L2 = eqlin.EQLinear(gb["W"], gb["b"])
    x = ga["x"].clone()
    y1 = torch.empty((N, C2 * T), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((N, C1 * T), dtype=torch.bfloat16, device="cuda")
    g1 = torch.empty((N, C2 * T), dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        x_in = x.float().cpu().numpy()
        eqlin.forward(L1.h, x, y1)
        eqlin.forward(L2.h, y1, y2)
        eqlin.backward_dx(L2.h, y2, g1)
        eqlin.backward_dx(L1.h, g1, x)
        torch.cuda.synchronize()
        assert eqlin.get_error(L1.h) == 0 and eqlin.get_error(L2.h) == 0
        k = {n: t.float().cpu().numpy() for n, t in (("y1", y1), ("y2", y2), ("g1", g1), ("x", x))}
        tol = TOL["bf16"]
        check("chain y1", k["y1"], oracle.forward(x_in, a["W"], a["b"]), tol)
        check("chain y2", k["y2"], oracle.forward(k["y1"], b["W"], b["b"]), tol)
        check("chain g1", k["g1"], oracle.backward_dx(k["y2"], b["W"]), tol)
        check("chain x", k["x"], oracle.backward_dx(k["g1"], a["W"]), tol)


@pytest.mark.parametrize("T,dt", [(3, "f32"), (6, "f32"), (3, "bf16"), (6, "f16")], ids=str)
def test_odd_and_sixfold_groups_are_equivariant(T, dt):
    """T = 3 and 6 run the tensor-core kernels in f16/bf16 (the SIMT ones in
    FP32); a cyclic shift of the input's group axis shifts the output's, and
    the backend says which kernels ran."""
    Cp, Dp, N = 16, 24, 150
    inp = _dev(inputs.make_inputs(T, Cp, Dp, N, dt, seed=15))
    layer = eqlin.EQLinear(inp["W"], inp["b"])
    want = "fwd=simt dx=simt dw=simt" if dt == "f32" else "fwd=tcgen05 dx=tcgen05 dw=tcgen05"
    assert layer.h.backend() == want
    y = layer.forward(inp["x"])
    tol = 1e-5 if dt == "f32" else TOL[dt]
    for r in range(1, T):
        yr = layer.forward(_roll(inp["x"], Cp, T, r))
        check(f"T={T} {dt} equivariance shift {r}", yr, _roll(y, Dp, T, r), tol)
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == 0


def test_calls_from_another_host_thread():
    """A host thread other than the one that created the handle (an autograd
    worker, for one) can call every entry point."""
    import threading
    T, Cp, Dp, N = 4, 64, 96, 300
    inp = inputs.make_inputs(T, Cp, Dp, N, "bf16", seed=14)
    g = _dev(inp)
    layer = eqlin.EQLinear(g["W"], g["b"])
    torch.cuda.synchronize()
    out, errs = {}, []

    def worker():
        try:
            out["y"] = layer.forward(g["x"])
            out["dx"] = layer.backward_dx(g["gy"])
            out["dW"], out["db"] = layer.backward_dw(g["x"], g["gy"])
            eqlin.set_weights(layer.h, g["W"], g["b"])
            torch.cuda.synchronize()
        except Exception as e:  # reported below, in the test's own thread
            errs.append(repr(e))

    th = threading.Thread(target=worker)
    th.start()
    th.join()
    assert not errs, errs
    assert eqlin.get_error(layer.h) == 0
    tol = TOL["bf16"]
    check("other thread y", out["y"], oracle.forward(inp["x"], inp["W"], inp["b"]), tol)
    check("other thread dx", out["dx"], oracle.backward_dx(inp["gy"], inp["W"]), tol)
    dW, db = oracle.backward_dw(inp["x"], inp["gy"], T, Cp, Dp)
    check("other thread dW", out["dW"], dW, tol)
    check("other thread db", out["db"], db, tol)


def _roll(a: torch.Tensor, ch: int, T: int, r: int) -> torch.Tensor:
    N = a.shape[0]
    return torch.roll(a.reshape(N, ch, T), r, dims=2).reshape(N, ch * T).contiguous()


FULL = [(name, i) for name, layers in workloads.WORKLOADS.items() for i in range(len(layers))]
# workloads compared on every output element; the others on stratified samples
WHOLE = {"p4-tiny-f32-fwd", "eq-vit-s-f16-fwd", "eq-vit-b-mlp-bf16-fwdbwd", "eq-swin-t-s1-f16-fwdbwd"}
ROW_BLOCK = 16384          # tokens per oracle call when the whole output is compared


def _rows_one_per_tile(N: int, rng) -> np.ndarray:
    """One random token of every 128-token tile, plus the first and the last."""
    starts = np.arange(0, N, 128)
    ends = np.minimum(starts + 128, N)
    pick = starts + (rng.random(len(starts)) * (ends - starts)).astype(np.int64)
    return np.unique(np.concatenate([[0, N - 1], pick]))


def _pairs_every_block(Dp: int, Cp: int, rng, per_block: int = 8) -> np.ndarray:
    """`per_block` random (d, c) pairs in every 128 x 128 block of the weight."""
    out = []
    for d0 in range(0, Dp, 128):
        for c0 in range(0, Cp, 128):
            d1, c1 = min(Dp, d0 + 128), min(Cp, c0 + 128)
            out.append(np.stack([rng.integers(d0, d1, per_block), rng.integers(c0, c1, per_block)], 1))
    return np.concatenate(out)


def _compare_rows(label, got, ref_fn, N, tol, rows=None):
    """Compare a [N, width] device output with the oracle, in row blocks."""
    acc = Accum()
    if rows is None:
        for a in range(0, N, ROW_BLOCK):
            r = np.arange(a, min(N, a + ROW_BLOCK))
            acc.add(got[a:a + len(r)], ref_fn(r))
    else:
        acc.add(got[torch.as_tensor(rows, device=got.device)], ref_fn(rows))
    finish(label, acc, tol)


@pytest.mark.parametrize("name,idx", FULL, ids=lambda v: str(v))
def test_full_size(name, idx):
    """Every workload at full size, through the same entry points bench.py times."""
    L = workloads.WORKLOADS[name][idx]
    T, Cp, Dp, N, dt = L.T, L.Cp, L.Dp, L.N, L.dtype
    whole = name in WHOLE
    inp = inputs.make_inputs(T, Cp, Dp, N, dt, seed=0, with_gy=("dx" in L.passes or "dw" in L.passes))
    g = _dev(inp)
    f64 = {k: v.double().numpy() for k, v in inp.items()}
    layer = eqlin.EQLinear(g["W"], g["b"])
    rng = np.random.default_rng(1)
    rows = None if whole else _rows_one_per_tile(N, rng)
    tol = TOL[dt]
    tag = f"full {L.name} N={N} {dt}" + ("" if whole else " (sampled)")
    y = layer.forward(g["x"])
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == 0
    _compare_rows(f"{tag} y", y, lambda r: oracle.forward(f64["x"], f64["W"], f64["b"], rows=r), N, tol, rows)
    # equivariance on the whole output: rotate the group axis of x by one step
    yr = layer.forward(_roll(g["x"], Cp, T, 1))
    check(f"{tag} y equivariance", yr, _roll(y, Dp, T, 1), tol)
    del yr
    fused = None
    if "dx" in L.passes and "dw" in L.passes and _fused_capable(T, Cp, Dp, dt):
        fused = _run_fused(layer, g)
        check_exact(f"{tag} fused y vs eqlin_forward", fused["y"], y)
        del fused["xs"], fused["gs"]
    del y
    if "dx" in L.passes:
        dx = layer.backward_dx(g["gy"])
        torch.cuda.synchronize()
        _compare_rows(f"{tag} dx", dx, lambda r: oracle.backward_dx(f64["gy"], f64["W"], rows=r), N, tol, rows)
        if fused is not None:
            check_exact(f"{tag} fused dx vs eqlin_backward_dx", fused["dx"], dx)
        del dx
    if "dw" in L.passes:
        dW, db = layer.backward_dw(g["x"], g["gy"])
        torch.cuda.synchronize()
        if whole:
            want, want_db = oracle.backward_dw(f64["x"], f64["gy"], T, Cp, Dp)
            check(f"{tag} dW", dW, want, tol)
            if fused is not None:
                check(f"{tag} fused dW", fused["dW"], want, tol)
        else:
            pairs = _pairs_every_block(Dp, Cp, rng)
            want, want_db = oracle.backward_dw(f64["x"], f64["gy"], T, Cp, Dp, pairs=pairs)
            check(f"{tag} dW", dW.cpu().numpy()[pairs[:, 0], pairs[:, 1]], want, tol)
            if fused is not None:
                check(f"{tag} fused dW", fused["dW"].cpu().numpy()[pairs[:, 0], pairs[:, 1]], want, tol)
        check(f"{tag} db", db, want_db, tol)
        if fused is not None:
            check(f"{tag} fused db", fused["db"], want_db, tol)
    assert eqlin.get_error(layer.h) == 0


# ------------------------------------------------------------- error paths

def test_error_paths():
    T, Cp, Dp = 4, 16, 16
    h = eqlin.create(T, Cp, Dp, "f16")
    x = torch.zeros((10, Cp * T), dtype=torch.float16, device="cuda")
    y = torch.zeros((10, Dp * T), dtype=torch.float16, device="cuda")
    L = eqlin.lib()
    s = torch.cuda.current_stream().cuda_stream
    import ctypes
    vp = ctypes.c_void_p
    # before set_weights
    assert L.eqlin_forward(h.ptr, vp(x.data_ptr()), vp(y.data_ptr()), 10, vp(s)) == -5
    W = torch.randn((Dp, Cp, T), device="cuda").half()
    eqlin.set_weights(h, W, None)
    # misaligned pointers
    assert L.eqlin_forward(h.ptr, vp(x.data_ptr() + 2), vp(y.data_ptr()), 9, vp(s)) == -3
    assert L.eqlin_forward(h.ptr, vp(x.data_ptr()), vp(y.data_ptr() + 8), 9, vp(s)) == -3
    # negative N, null pointers
    assert L.eqlin_forward(h.ptr, vp(x.data_ptr()), vp(y.data_ptr()), -1, vp(s)) == -1
    assert L.eqlin_forward(h.ptr, None, vp(y.data_ptr()), 10, vp(s)) == -1
    # N = 0 is a no-op; dW/db are zeroed
    assert L.eqlin_forward(h.ptr, None, None, 0, vp(s)) == 0
    dW = torch.full((Dp, Cp, T), 7.0, device="cuda")
    db = torch.full((Dp,), 7.0, device="cuda")
    assert L.eqlin_backward_dw(h.ptr, None, None, vp(dW.data_ptr()), vp(db.data_ptr()), 0, vp(s)) == 0
    torch.cuda.synchronize()
    assert not dW.any() and not db.any()
    # wrong dtype / shape are rejected by the binding
    with pytest.raises(TypeError):
        eqlin.forward(h, x.float(), y)
    with pytest.raises(ValueError):
        eqlin.forward(h, x[:, :8].contiguous(), y)
    assert eqlin.get_error(h) == 0
    h.close()


def test_outputs_have_no_stray_writes():
    """Canary rows around the output stay untouched (ragged N, odd D')."""
    T, Cp, Dp, N = 4, 96, 40, 133
    inp = _dev(inputs.make_inputs(T, Cp, Dp, N, "bf16", seed=2))
    layer = eqlin.EQLinear(inp["W"], inp["b"])
    buf = torch.full((N + 64, Dp * T), 123.0, dtype=torch.bfloat16, device="cuda")
    eqlin.forward(layer.h, inp["x"], buf[32:32 + N])
    dxb = torch.full((N + 64, Cp * T), 123.0, dtype=torch.bfloat16, device="cuda")
    eqlin.backward_dx(layer.h, inp["gy"], dxb[32:32 + N])
    torch.cuda.synchronize()
    assert (buf[:32] == 123).all() and (buf[32 + N:] == 123).all()
    assert (dxb[:32] == 123).all() and (dxb[32 + N:] == 123).all()
    assert not (buf[32:32 + N] == 123).all()


def test_backend_is_reported_per_pass():
    """f16/bf16 handles with 8-aligned channel counts run the tcgen05 kernels in
    every pass; a pass whose K is not a multiple of 8 runs the SIMT kernels, and
    the handle says which pass."""
    for dt in ("f16", "bf16"):
        for T in (1, 2, 3, 4, 6, 8):
            h = eqlin.create(T, 64, 64, dt)
            assert h.backend() == "fwd=tcgen05 dx=tcgen05 dw=tcgen05", (T, dt, h.backend())
            h.close()
    for T in (1, 2, 4):      # FP32: 3xTF32 tensor cores
        assert eqlin.create(T, 16, 16, "f32").backend() == "fwd=tcgen05 dx=tcgen05 dw=tcgen05", T
    assert eqlin.create(8, 16, 16, "f32").backend() == "fwd=tcgen05 dx=tcgen05 dw=simt"
    for T in (3, 6):
        assert eqlin.create(T, 16, 16, "f32").backend() == "fwd=simt dx=simt dw=simt", T
    # FP32 passes whose reduction is too long for the 3xTF32 error bound
    # (more than 256 MMAs into one accumulator) run on the SIMT kernels
    assert eqlin.create(4, 344, 16, "f32").backend() == "fwd=simt dx=tcgen05 dw=tcgen05"
    assert eqlin.create(2, 16, 688, "f32").backend() == "fwd=tcgen05 dx=simt dw=tcgen05"
    assert eqlin.create(1, 680, 680, "f32").backend() == "fwd=tcgen05 dx=tcgen05 dw=tcgen05"
    assert eqlin.create(4, 6, 16, "f16").backend() == "fwd=simt dx=tcgen05 dw=tcgen05"
    assert eqlin.create(4, 16, 6, "bf16").backend() == "fwd=tcgen05 dx=simt dw=tcgen05"


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait cap of one poll makes the kernel give up, record EQLIN_ERR_TIMEOUT
    and return; with the default cap the same handle then computes correctly."""
    T, Cp, Dp, N = 4, 768, 192, 4096
    inp = inputs.make_inputs(T, Cp, Dp, N, "bf16", seed=4)
    g = _dev(inp)
    layer = eqlin.EQLinear(g["W"], g["b"])
    assert layer.h.backend().startswith("fwd=tcgen05")
    eqlin.set_wait_limit(layer.h, 1)
    layer.forward(g["x"])
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == -6
    assert eqlin.get_error(layer.h) == 0          # reading clears it
    eqlin.set_wait_limit(layer.h, 0)
    y = layer.forward(g["x"])
    torch.cuda.synchronize()
    assert eqlin.get_error(layer.h) == 0
    rows = np.arange(0, N, 97)
    check("after timeout y (sampled rows)", y[torch.as_tensor(rows, device="cuda")],
          oracle.forward(inp["x"], inp["W"], inp["b"], rows=rows), TOL["bf16"])
