"""Pins for the CPU oracle: facts the oracle must match that do not come from it.

Each pin below is a check function ``pin_*(impl)`` that takes an object with
``forward``, ``backward_dx`` and ``backward_dw`` (the oracle's signatures) and
raises AssertionError on a mismatch.  The real oracle must pass all of them;
each planted mistake in ``test_pins_catch_planted_mistakes`` (a deliberately
wrong copy of one oracle function, on the CPU, at tiny sizes) must fail at
least one, so a dropped term, a flipped shift or a transposed index cannot
slip through.

Facts used (none of them re-types the oracle's loops):

* the dense group-circulant matrix built block by block with
  ``scipy.linalg.circulant`` ("replicating and cyclically shifting one set of
  parameters": Flash EQ-Linear technical summary, section "Insight Central");
* T = 1 reduces to an ordinary linear layer (numpy matmul);
* rotation equivariance (summary, "Garantias Teoricas": the method preserves
  the equivariance of the operator): shifting x cyclically along t shifts y
  along s, and likewise for gy -> dx; dW is invariant under a joint shift;
* special cases: W supported at tau = 0 only gives T independent linears;
  W constant in tau gives an output that does not depend on s; linearity;
* the convolution theorem ("Abordagem Algoritmica", step 1) restated with
  numpy's real FFT for forward, dx and dW;
* exact integer arithmetic through the dense matrix (int64 matmul);
* float64 autograd of the dense layer for dx, dW, db, and central finite
  differences of the oracle's own forward.
"""
from __future__ import annotations

import types

import numpy as np
import pytest
import scipy.linalg
import torch

SHAPES = [(1, 3, 2, 5), (2, 2, 3, 4), (3, 2, 2, 3), (4, 3, 2, 5), (4, 1, 1, 2),
          (8, 2, 3, 3), (6, 2, 2, 2), (5, 1, 2, 3)]   # (T, C', D', N)


def _rand(T, Cp, Dp, N, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, Cp * T)), rng.standard_normal((Dp, Cp, T)),
            rng.standard_normal(Dp), rng.standard_normal((N, Dp * T)))


def dense_matrix(W):
    """[D'T, C'T] matrix whose (d, c) block is scipy's circulant of W[d, c, :]."""
    Dp, Cp, T = W.shape
    M = np.zeros((Dp * T, Cp * T), dtype=np.result_type(W, np.float64))
    for d in range(Dp):
        for c in range(Cp):
            M[d * T:(d + 1) * T, c * T:(c + 1) * T] = scipy.linalg.circulant(W[d, c, :])
    return M


def _close(a, b, tol=1e-11):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    scale = max(1.0, float(np.abs(b).max()) if b.size else 1.0)
    err = float(np.abs(a - b).max()) if a.size else 0.0
    assert err <= tol * scale, f"max abs err {err} > {tol} * {scale}"


# --------------------------------------------------------------------------- pins

def pin_dense(impl):
    for i, (T, Cp, Dp, N) in enumerate(SHAPES):
        x, W, b, gy = _rand(T, Cp, Dp, N, 100 + i)
        M = dense_matrix(W)
        _close(impl.forward(x, W, b), x @ M.T + np.repeat(b, T))
        _close(impl.forward(x, W, None), x @ M.T)
        _close(impl.backward_dx(gy, W), gy @ M)


def pin_t1_is_linear(impl):
    x, W, b, gy = _rand(1, 5, 4, 7, 7)
    _close(impl.forward(x, W, b), x @ W[:, :, 0].T + b)
    _close(impl.backward_dx(gy, W), gy @ W[:, :, 0])
    dW, db = impl.backward_dw(x, gy, 1, 5, 4)
    _close(dW[:, :, 0], gy.T @ x)
    _close(db, gy.sum(0))


def _roll(a, ch, T, r):
    N = a.shape[0]
    return np.roll(a.reshape(N, ch, T), r, axis=2).reshape(N, ch * T)


def pin_equivariance(impl):
    for i, (T, Cp, Dp, N) in enumerate(SHAPES):
        x, W, b, gy = _rand(T, Cp, Dp, N, 200 + i)
        y = impl.forward(x, W, b)
        dx = impl.backward_dx(gy, W)
        dW, db = impl.backward_dw(x, gy, T, Cp, Dp)
        for r in range(T):
            _close(impl.forward(_roll(x, Cp, T, r), W, b), _roll(y, Dp, T, r))
            _close(impl.backward_dx(_roll(gy, Dp, T, r), W), _roll(dx, Cp, T, r))
            dWr, dbr = impl.backward_dw(_roll(x, Cp, T, r), _roll(gy, Dp, T, r), T, Cp, Dp)
            _close(dWr, dW)
            _close(dbr, db)


def pin_special_cases(impl):
    T, Cp, Dp, N = 4, 3, 2, 5
    x, W, b, gy = _rand(T, Cp, Dp, N, 11)
    # Support at tau = 0 only: T independent ordinary linears, one per s.
    W0 = np.zeros_like(W)
    W0[:, :, 0] = W[:, :, 0]
    want = np.einsum("dc,ncs->nds", W[:, :, 0], x.reshape(N, Cp, T)) + b[None, :, None]
    _close(impl.forward(x, W0, b), want.reshape(N, Dp * T))
    # W constant along tau: every output position s sees the same sum.
    Wc = np.repeat(W[:, :, :1], T, axis=2)
    yc = impl.forward(x, Wc, b).reshape(N, Dp, T)
    want_c = np.einsum("dc,nc->nd", W[:, :, 0], x.reshape(N, Cp, T).sum(2)) + b
    for s in range(T):
        _close(yc[:, :, s], want_c)
    # Linearity in x (bias enters once) and in W.
    x2 = _rand(T, Cp, Dp, N, 12)[0]
    _close(impl.forward(2.5 * x + x2, W, b) - b.repeat(T),
           2.5 * (impl.forward(x, W, b) - b.repeat(T)) + (impl.forward(x2, W, b) - b.repeat(T)))
    W2 = _rand(T, Cp, Dp, N, 13)[1]
    _close(impl.forward(x, W + W2, None), impl.forward(x, W, None) + impl.forward(x, W2, None))


def pin_fft(impl):
    for i, (T, Cp, Dp, N) in enumerate(SHAPES):
        x, W, b, gy = _rand(T, Cp, Dp, N, 300 + i)
        X = np.fft.rfft(x.reshape(N, Cp, T), axis=2)
        G = np.fft.rfft(gy.reshape(N, Dp, T), axis=2)
        Wf = np.fft.rfft(W, axis=2)
        Y = np.einsum("dck,nck->ndk", Wf, X)
        y = np.fft.irfft(Y, n=T, axis=2) + b[None, :, None]
        _close(impl.forward(x, W, b), y.reshape(N, Dp * T))
        DX = np.einsum("dck,ndk->nck", np.conj(Wf), G)
        _close(impl.backward_dx(gy, W), np.fft.irfft(DX, n=T, axis=2).reshape(N, Cp * T))
        dWf = np.einsum("ndk,nck->dck", G, np.conj(X))
        dW, db = impl.backward_dw(x, gy, T, Cp, Dp)
        _close(dW, np.fft.irfft(dWf, n=T, axis=2))
        _close(db, G[:, :, 0].real.sum(0))


def pin_integer_exact(impl):
    rng = np.random.default_rng(5)
    for T, Cp, Dp, N in [(4, 3, 2, 4), (2, 4, 3, 5), (8, 2, 2, 3), (3, 2, 3, 2), (6, 2, 2, 3)]:
        x = rng.integers(-4, 5, (N, Cp * T))
        W = rng.integers(-4, 5, (Dp, Cp, T))
        b = rng.integers(-1, 2, Dp)
        gy = rng.integers(-4, 5, (N, Dp * T))
        M = dense_matrix(W).astype(np.int64)
        assert np.array_equal(impl.forward(x, W, b), x @ M.T + np.repeat(b, T))
        assert np.array_equal(impl.backward_dx(gy, W), gy @ M)
        dW, db = impl.backward_dw(x, gy, T, Cp, Dp)
        dM = gy.T @ x     # gradient of the dense matrix, then gather per tied parameter
        want = np.zeros((Dp, Cp, T), dtype=np.int64)
        for tau in range(T):
            P = scipy.linalg.circulant(np.eye(T, dtype=np.int64)[tau])
            want[:, :, tau] = np.einsum("dsct,st->dc", dM.reshape(Dp, T, Cp, T), P)
        assert np.array_equal(dW, want)
        assert np.array_equal(db, gy.reshape(N, Dp, T).sum((0, 2)))


def pin_autograd(impl):
    for i, (T, Cp, Dp, N) in enumerate(SHAPES):
        x, W, b, gy = _rand(T, Cp, Dp, N, 400 + i)
        P = torch.tensor(np.stack([scipy.linalg.circulant(np.eye(T)[u]) for u in range(T)]))
        xt = torch.tensor(x, requires_grad=True)
        Wt = torch.tensor(W, requires_grad=True)
        bt = torch.tensor(b, requires_grad=True)
        dense = torch.einsum("dcu,ust->dsct", Wt, P).reshape(Dp * T, Cp * T)
        y = torch.nn.functional.linear(xt, dense, bt.repeat_interleave(T))
        (y * torch.tensor(gy)).sum().backward()
        _close(impl.backward_dx(gy, W), xt.grad.numpy())
        dW, db = impl.backward_dw(x, gy, T, Cp, Dp)
        _close(dW, Wt.grad.numpy())
        _close(db, bt.grad.numpy())


def pin_finite_difference(impl):
    T, Cp, Dp, N = 4, 2, 3, 3
    x, W, b, gy = _rand(T, Cp, Dp, N, 21)
    loss = lambda x_, W_, b_: float((impl.forward(x_, W_, b_) * gy).sum())
    h = 1e-5
    dx = impl.backward_dx(gy, W)
    dW, db = impl.backward_dw(x, gy, T, Cp, Dp)
    rng = np.random.default_rng(0)
    for _ in range(6):
        i, j = rng.integers(N), rng.integers(Cp * T)
        xp, xm = x.copy(), x.copy()
        xp[i, j] += h
        xm[i, j] -= h
        assert abs((loss(xp, W, b) - loss(xm, W, b)) / (2 * h) - dx[i, j]) < 1e-6
        d, c, u = rng.integers(Dp), rng.integers(Cp), rng.integers(T)
        Wp, Wm = W.copy(), W.copy()
        Wp[d, c, u] += h
        Wm[d, c, u] -= h
        assert abs((loss(x, Wp, b) - loss(x, Wm, b)) / (2 * h) - dW[d, c, u]) < 1e-6
        bp, bm = b.copy(), b.copy()
        bp[d] += h
        bm[d] -= h
        assert abs((loss(x, W, bp) - loss(x, W, bm)) / (2 * h) - db[d]) < 1e-6


ALL_PINS = [pin_dense, pin_t1_is_linear, pin_equivariance, pin_special_cases, pin_fft,
            pin_integer_exact, pin_autograd, pin_finite_difference]


# --------------------------------------------------------------------------- tests

@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_passes_pin(pin, oracle_mod):
    pin(oracle_mod)


def test_dense_matrix_is_block_circulant():
    """The pins' dense matrix itself: T distinct cyclic shifts per block."""
    rng = np.random.default_rng(1)
    W = rng.standard_normal((2, 3, 5))
    M = dense_matrix(W)
    for d in range(2):
        for c in range(3):
            blk = M[d * 5:(d + 1) * 5, c * 5:(c + 1) * 5]
            for s in range(5):
                assert np.array_equal(blk[s], np.roll(blk[0], s))
            assert len({tuple(r) for r in blk}) == 5


def test_rows_and_pairs_subsets(oracle_mod):
    x, W, b, gy = _rand(4, 3, 2, 9, 3)
    rows = np.array([8, 0, 3])
    _close(oracle_mod.forward(x, W, b, rows=rows), oracle_mod.forward(x, W, b)[rows])
    _close(oracle_mod.backward_dx(gy, W, rows=rows), oracle_mod.backward_dx(gy, W)[rows])
    pairs = np.array([[1, 2], [0, 0], [1, 0]])
    dWs, _ = oracle_mod.backward_dw(x, gy, 4, 3, 2, pairs=pairs, want_db=False)
    dW, _ = oracle_mod.backward_dw(x, gy, 4, 3, 2)
    _close(dWs, dW[pairs[:, 0], pairs[:, 1]])


def test_empty_batch(oracle_mod):
    x, W, b, gy = _rand(4, 2, 2, 0, 3)
    assert oracle_mod.forward(x, W, b).shape == (0, 8)
    dW, db = oracle_mod.backward_dw(x, gy, 4, 2, 2)
    assert not dW.any() and not db.any()


# ------------------------------------------------------------ planted mistakes

def _loop_impl(fwd_idx=None, use_bias=True, dx_idx=None, dw_idx=None, db_s=None):
    """A plain-loop copy of the oracle with one index or term replaced."""
    fwd_idx = fwd_idx or (lambda s, t, T: (s - t) % T)
    dx_idx = dx_idx or (lambda s, t, T: (s - t) % T)
    dw_idx = dw_idx or (lambda s, tau, T: (s - tau) % T)
    db_s = db_s or (lambda T: range(T))

    def forward(x, W, b=None, rows=None):
        x, W = np.asarray(x, float), np.asarray(W, float)
        Dp, Cp, T = W.shape
        y = np.zeros((x.shape[0], Dp * T))
        for n in range(x.shape[0]):
            for d in range(Dp):
                for s in range(T):
                    acc = sum(W[d, c, fwd_idx(s, t, T)] * x[n, c * T + t]
                              for c in range(Cp) for t in range(T))
                    y[n, d * T + s] = acc + (b[d] if (b is not None and use_bias) else 0.0)
        return y

    def backward_dx(gy, W, rows=None):
        gy, W = np.asarray(gy, float), np.asarray(W, float)
        Dp, Cp, T = W.shape
        dx = np.zeros((gy.shape[0], Cp * T))
        for n in range(gy.shape[0]):
            for c in range(Cp):
                for t in range(T):
                    dx[n, c * T + t] = sum(W[d, c, dx_idx(s, t, T)] * gy[n, d * T + s]
                                           for d in range(Dp) for s in range(T))
        return dx

    def backward_dw(x, gy, T, Cp, Dp, pairs=None, want_db=True):
        x, gy = np.asarray(x, float), np.asarray(gy, float)
        dW = np.zeros((Dp, Cp, T))
        for d in range(Dp):
            for c in range(Cp):
                for tau in range(T):
                    dW[d, c, tau] = sum(gy[n, d * T + s] * x[n, c * T + dw_idx(s, tau, T)]
                                        for n in range(x.shape[0]) for s in range(T))
        db = np.array([sum(gy[n, d * T + s] for n in range(x.shape[0]) for s in db_s(T))
                       for d in range(Dp)])
        return dW, db

    return types.SimpleNamespace(forward=forward, backward_dx=backward_dx, backward_dw=backward_dw)


MUTANTS = {
    "faithful-copy": None,
    "fwd-shift-t-minus-s": dict(fwd_idx=lambda s, t, T: (t - s) % T),
    "fwd-shift-s-plus-t": dict(fwd_idx=lambda s, t, T: (s + t) % T),
    "fwd-bias-dropped": dict(use_bias=False),
    "dx-shift-flipped": dict(dx_idx=lambda s, t, T: (t - s) % T),
    "dw-shift-flipped": dict(dw_idx=lambda s, tau, T: (s + tau) % T),
    "db-only-s0": dict(db_s=lambda T: range(1)),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_catch_planted_mistakes(name):
    kw = MUTANTS[name]
    impl = _loop_impl(**(kw or {}))
    failures = []
    for pin in ALL_PINS:
        try:
            pin(impl)
        except AssertionError:
            failures.append(pin.__name__)
    if kw is None:
        assert failures == [], f"faithful copy failed {failures}"
    else:
        assert failures, f"planted mistake {name} passed every pin"
