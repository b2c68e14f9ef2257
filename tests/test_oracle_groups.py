"""Pins for the oracle's group-table functions (the layer over the dihedral groups).

The pages name reflection groups as future work and give no formula
("Flash EQ-Linear", technical summary, section "Limitacoes e Trabalho
Futuro").  The reading taken is the group convolution
    y[d, g] = b[d] + sum_c sum_h W[d, c, h^-1 g] x[c, h],
which for Z_T is the paper's (s - t) mod T.  Each pin below checks it against
a fact that does not come from the oracle:

* the tables satisfy the group axioms and the defining relations of D_m
  (r^m = e, s^2 = e, s r s^-1 = r^-1), and D_m is non-abelian for m >= 3;
* on the cyclic table the group functions equal the cyclic oracle (pinned in
  test_oracle_pins.py), and D_1 is Z_2;
* the layer commutes with the left action (L_u x)[h] = x[u^-1 h] of every
  group element (so does dx with gy; dW is invariant under the joint action);
* W supported on the rotations reduces, on the rotation coset, to the cyclic
  layer of order m;
* the convolution theorem over D_m's irreducible representations (1- and
  2-dimensional, built here from their definition and checked to be
  homomorphisms): x^(rho) W^(rho) is the transform of y;
* central finite differences of the forward for dx, dW and db.
Two planted mistakes (the right convolution W[g h^-1] and W[h g^-1]) must
fail the equivariance pin.
"""
from __future__ import annotations

import types

import numpy as np
import pytest

import oracle

MS = [1, 2, 3, 4, 5, 6, 8]


def _rand(G, Cp, Dp, N, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, Cp * G)), rng.standard_normal((Dp, Cp, G)),
            rng.standard_normal(Dp), rng.standard_normal((N, Dp * G)))


def _close(a, b, tol=1e-11):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    scale = max(1.0, float(np.abs(b).max()) if b.size else 1.0)
    err = float(np.abs(a - b).max()) if a.size else 0.0
    assert err <= tol * scale, f"max abs err {err} > {tol} * {scale}"


def _act(v, ch, table, u):
    """(L_u v)[c, h] = v[c, u^-1 h] on features [N, ch*|G|]."""
    mul, inv = table
    G = inv.shape[0]
    src = mul[inv[u]]                     # h -> u^-1 h
    return v.reshape(-1, ch, G)[:, :, src].reshape(-1, ch * G)


# ------------------------------------------------------------------ tables

@pytest.mark.parametrize("m", MS)
def test_dihedral_table_is_the_dihedral_group(m):
    mul, inv = oracle.dihedral_table(m)
    n = 2 * m
    e, r, s = 0, (1 % m), m
    assert mul.shape == (n, n)
    for g in range(n):
        assert mul[e, g] == g and mul[g, e] == g
        assert mul[g, inv[g]] == e and mul[inv[g], g] == e
        assert sorted(mul[g]) == list(range(n))          # Latin square
    for a in range(n):
        for b in range(n):
            for c in range(n):
                assert mul[mul[a, b], c] == mul[a, mul[b, c]]
    def power(g, k):
        out = e
        for _ in range(k):
            out = mul[out, g]
        return out
    assert power(r, m) == e and mul[s, s] == e
    assert mul[mul[s, r], inv[s]] == inv[r]                # s r s^-1 = r^-1
    assert (mul == mul.T).all() == (m <= 2)                # abelian only for m <= 2


@pytest.mark.parametrize("T", [1, 2, 3, 4, 8])
def test_cyclic_table_is_z_t(T):
    mul, inv = oracle.cyclic_table(T)
    for a in range(T):
        for b in range(T):
            assert mul[a, b] == (a + b) % T
        assert (a + inv[a]) % T == 0


# ------------------------------------------------------------------- pins

def pin_cyclic_agrees(impl):
    for T, Cp, Dp, N in [(1, 3, 2, 4), (2, 2, 3, 5), (4, 3, 2, 5), (6, 2, 2, 3), (8, 1, 2, 2)]:
        x, W, b, gy = _rand(T, Cp, Dp, N, 40 + T)
        tab = oracle.cyclic_table(T)
        _close(impl.forward_group(x, W, b, tab), oracle.forward(x, W, b))
        _close(impl.backward_dx_group(gy, W, tab), oracle.backward_dx(gy, W))
        dW, db = impl.backward_dw_group(x, gy, tab, Cp, Dp)
        wdW, wdb = oracle.backward_dw(x, gy, T, Cp, Dp)
        _close(dW, wdW)
        _close(db, wdb)
    # D_1 = {e, s} is Z_2, with the same element order
    x, W, b, gy = _rand(2, 3, 2, 4, 49)
    _close(impl.forward_group(x, W, b, oracle.dihedral_table(1)), oracle.forward(x, W, b))


def pin_equivariance(impl):
    for m in MS:
        tab = oracle.dihedral_table(m)
        G, Cp, Dp, N = 2 * m, 2, 3, 3
        x, W, b, gy = _rand(G, Cp, Dp, N, 50 + m)
        y = impl.forward_group(x, W, b, tab)
        dx = impl.backward_dx_group(gy, W, tab)
        dW, db = impl.backward_dw_group(x, gy, tab, Cp, Dp)
        for u in range(G):
            _close(impl.forward_group(_act(x, Cp, tab, u), W, b, tab), _act(y, Dp, tab, u))
            _close(impl.backward_dx_group(_act(gy, Dp, tab, u), W, tab), _act(dx, Cp, tab, u))
            dWu, dbu = impl.backward_dw_group(_act(x, Cp, tab, u), _act(gy, Dp, tab, u), tab, Cp, Dp)
            _close(dWu, dW)
            _close(dbu, db)


def pin_rotation_coset(impl):
    """W on the rotations r^a only: the rotation coset of y is the cyclic layer
    of order m on the rotation coset of x."""
    for m in [2, 3, 4, 6]:
        tab = oracle.dihedral_table(m)
        G, Cp, Dp, N = 2 * m, 3, 2, 4
        x, W, b, gy = _rand(G, Cp, Dp, N, 60 + m)
        Wr = W.copy()
        Wr[:, :, m:] = 0.0
        y = impl.forward_group(x, Wr, b, tab).reshape(N, Dp, G)[:, :, :m]
        want = oracle.forward(x.reshape(N, Cp, G)[:, :, :m].reshape(N, Cp * m), W[:, :, :m], b)
        _close(y.reshape(N, Dp * m), want)


def dihedral_irreps(m):
    """Real irreducible representations of D_m as [n, d, d] arrays over the
    element index f*m + a: the trivial one, the reflection sign (-1)^f, for
    even m also (-1)^a and (-1)^(a+f), and for k = 1 .. ceil(m/2)-1 the planar
    ones: rotation by 2 pi k a / m, then the mirror diag(1, -1) if f = 1."""
    n = 2 * m
    f = np.arange(n) // m
    a = np.arange(n) % m
    reps = [np.ones((n, 1, 1)), ((-1.0) ** f)[:, None, None]]
    if m % 2 == 0:
        reps += [((-1.0) ** a)[:, None, None], ((-1.0) ** (a + f))[:, None, None]]
    for k in range(1, (m + 1) // 2):
        th = 2 * np.pi * k * a / m
        R = np.stack([np.stack([np.cos(th), -np.sin(th)], -1), np.stack([np.sin(th), np.cos(th)], -1)], -2)
        M = np.where(f[:, None, None] == 1, R @ np.diag([1.0, -1.0]), R)
        reps.append(M)
    return reps


@pytest.mark.parametrize("m", [1, 2, 3, 4, 6, 8])
def test_irreps_are_the_irreducible_representations(m):
    mul, _ = oracle.dihedral_table(m)
    reps = dihedral_irreps(m)
    assert sum(r.shape[1] ** 2 for r in reps) == 2 * m            # sum of d^2 = |G|
    for r in reps:
        for g in range(2 * m):
            for h in range(2 * m):
                _close(r[mul[g, h]], r[g] @ r[h])                  # homomorphism
    # Schur orthogonality of the matrix entries: the transform is invertible
    F = np.concatenate([r.reshape(2 * m, -1) * np.sqrt(r.shape[1]) for r in reps], 1)
    _close(F.T @ F, 2 * m * np.eye(2 * m))


def pin_group_fourier(impl):
    """Convolution theorem over D_m: with f^(rho) = sum_g f(g) rho(g), the
    transform of y - b is x^(rho) W^(rho) (summed over input channels)."""
    for m in [1, 2, 3, 4, 6, 8]:
        tab = oracle.dihedral_table(m)
        G, Cp, Dp, N = 2 * m, 2, 3, 2
        x, W, b, gy = _rand(G, Cp, Dp, N, 70 + m)
        y = impl.forward_group(x, W, None, tab).reshape(N, Dp, G)
        xs = x.reshape(N, Cp, G)
        for rep in dihedral_irreps(m):
            X = np.einsum("ncg,gij->ncij", xs, rep)
            Wh = np.einsum("dcg,gij->dcij", W, rep)
            Y = np.einsum("ng,gij->nij", y.reshape(N * Dp, G), rep).reshape(N, Dp, *rep.shape[1:])
            _close(Y, np.einsum("ncik,dckj->ndij", X, Wh))


def pin_finite_differences(impl):
    m, Cp, Dp, N = 3, 2, 2, 2
    tab = oracle.dihedral_table(m)
    G = 2 * m
    x, W, b, gy = _rand(G, Cp, Dp, N, 80)
    h = 1e-6

    def loss(x_, W_, b_):
        return float((impl.forward_group(x_, W_, b_, tab) * gy).sum())

    dx = impl.backward_dx_group(gy, W, tab)
    dW, db = impl.backward_dw_group(x, gy, tab, Cp, Dp)
    for idx in [(0, 0), (1, 5), (0, Cp * G - 1)]:
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        _close((loss(xp, W, b) - loss(xm, W, b)) / (2 * h), dx[idx], tol=1e-6)
    for idx in [(0, 0, 0), (1, 1, 4), (0, 1, G - 1)]:
        Wp, Wm = W.copy(), W.copy()
        Wp[idx] += h
        Wm[idx] -= h
        _close((loss(x, Wp, b) - loss(x, Wm, b)) / (2 * h), dW[idx], tol=1e-6)
    for d in range(Dp):
        bp, bm = b.copy(), b.copy()
        bp[d] += h
        bm[d] -= h
        _close((loss(x, W, bp) - loss(x, W, bm)) / (2 * h), db[d], tol=1e-6)


PINS = [pin_cyclic_agrees, pin_equivariance, pin_rotation_coset, pin_group_fourier, pin_finite_differences]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_passes_pin(pin):
    pin(oracle)


def _mutant(index_fn):
    """A deliberately wrong group forward: kernel index index_fn(mul, inv, g, h)."""
    def forward_group(x, W, b, table, rows=None):
        mul, inv = table
        W = np.asarray(W, dtype=np.float64)
        Dp, Cp, G = W.shape
        xs = np.asarray(x, dtype=np.float64).reshape(-1, Cp, G)
        K = np.empty((G, G), dtype=np.int64)
        for g in range(G):
            for h in range(G):
                K[g, h] = index_fn(mul, inv, g, h)
        y = np.einsum("dcgh,nch->ndg", W[:, :, K], xs)
        if b is not None:
            y = y + np.asarray(b)[None, :, None]
        return y.reshape(xs.shape[0], Dp * G)
    return types.SimpleNamespace(forward_group=forward_group, backward_dx_group=oracle.backward_dx_group,
                                 backward_dw_group=oracle.backward_dw_group)


@pytest.mark.parametrize("name,fn", [
    ("right convolution g h^-1", lambda mul, inv, g, h: mul[g, inv[h]]),
    ("h g^-1", lambda mul, inv, g, h: mul[h, inv[g]]),
], ids=lambda v: v if isinstance(v, str) else "")
def test_equivariance_pin_catches_planted_mistakes(name, fn):
    with pytest.raises(AssertionError):
        pin_equivariance(_mutant(fn))


def test_mutant_harness_reproduces_the_oracle():
    """The harness with the right index equals the oracle (so the mutants differ by their index only)."""
    good = _mutant(lambda mul, inv, g, h: mul[inv[h], g])
    for m in [3, 4]:
        tab = oracle.dihedral_table(m)
        x, W, b, _ = _rand(2 * m, 2, 2, 3, 90 + m)
        _close(good.forward_group(x, W, b, tab), oracle.forward_group(x, W, b, tab))
