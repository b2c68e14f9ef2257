"""CPU oracle for the EQ-Linear layer (test infrastructure only).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product path (the CUDA library and its Python
binding) never imports, links or executes anything here, and nothing here
imports the product package.

The arithmetic lives in ``eqlin_oracle.c``: the plain index definition of the
layer from "Flash EQ-Linear: Accelerating Equivariant Linear Layers via
Group-wise Discrete Fourier Transform" (abstract; technical summary, section
"Insight Central") and its exact gradients, looped in double precision.  This
module only compiles that file with gcc, loads it with ctypes and converts
numpy arrays to float64.

Every function here is pinned by ``tests/test_oracle_pins.py`` against facts
that do not come from the oracle itself (explicit dense-matrix construction,
T=1 matmul, equivariance, special cases, a numpy FFT restatement, exact
integer brute force, float64 autograd and finite differences).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eqlin_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libeqlin_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math) if needed."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, dp, ip = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p
        lib.eqlin_oracle_threads.restype = ctypes.c_int
        lib.eqlin_oracle_forward.argtypes = [i64, i64, i64, dp, dp, dp, ip, i64, dp]
        lib.eqlin_oracle_forward.restype = None
        lib.eqlin_oracle_backward_dx.argtypes = [i64, i64, i64, dp, dp, ip, i64, dp]
        lib.eqlin_oracle_backward_dx.restype = None
        lib.eqlin_oracle_backward_dw.argtypes = [i64, i64, i64, i64, dp, dp, ip, i64, dp, dp]
        lib.eqlin_oracle_backward_dw.restype = None
        lib.eqlin_oracle_forward_group.argtypes = [i64, ip, ip, i64, i64, dp, dp, dp, ip, i64, dp]
        lib.eqlin_oracle_forward_group.restype = None
        lib.eqlin_oracle_backward_dx_group.argtypes = [i64, ip, ip, i64, i64, dp, dp, ip, i64, dp]
        lib.eqlin_oracle_backward_dx_group.restype = None
        lib.eqlin_oracle_backward_dw_group.argtypes = [i64, ip, i64, i64, i64, dp, dp, dp, dp]
        lib.eqlin_oracle_backward_dw_group.restype = None
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor: take its (CPU) values
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    """OpenMP threads the oracle runs with."""
    return int(_load().eqlin_oracle_threads())


def forward(x, W, b=None, rows=None) -> np.ndarray:
    """y = EQ-Linear(x); x [N, C'*T], W [D', C', T], b [D'] or None.

    ``rows`` (optional int array) restricts the output to those tokens; the
    result then has len(rows) rows.
    """
    W = _f64(W)
    Dp, Cp, T = W.shape
    x = _f64(x)
    if x.ndim != 2 or x.shape[1] != Cp * T:
        raise ValueError(f"x must be [N, {Cp * T}], got {x.shape}")
    bb = None if b is None else _f64(b)
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n_out = x.shape[0] if r is None else r.shape[0]
    if r is not None and n_out and (r.min() < 0 or r.max() >= x.shape[0]):
        raise IndexError("row index out of range")
    y = np.empty((n_out, Dp * T), dtype=np.float64)
    _load().eqlin_oracle_forward(T, Cp, Dp, _ptr(x), _ptr(W), _ptr(bb), _ptr(r), n_out, _ptr(y))
    return y


def backward_dx(gy, W, rows=None) -> np.ndarray:
    """dx = dL/dx given gy = dL/dy; gy [N, D'*T], W [D', C', T]."""
    W = _f64(W)
    Dp, Cp, T = W.shape
    gy = _f64(gy)
    if gy.ndim != 2 or gy.shape[1] != Dp * T:
        raise ValueError(f"gy must be [N, {Dp * T}], got {gy.shape}")
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n_out = gy.shape[0] if r is None else r.shape[0]
    if r is not None and n_out and (r.min() < 0 or r.max() >= gy.shape[0]):
        raise IndexError("row index out of range")
    dx = np.empty((n_out, Cp * T), dtype=np.float64)
    _load().eqlin_oracle_backward_dx(T, Cp, Dp, _ptr(gy), _ptr(W), _ptr(r), n_out, _ptr(dx))
    return dx


def backward_dw(x, gy, T: int, Cp: int, Dp: int, pairs=None, want_db: bool = True):
    """(dW, db) = dL/dW, dL/db over all tokens.

    dW is [D', C', T] when ``pairs`` is None, else [len(pairs), T] for the
    given (d, c) index pairs.  db is [D'] (or None when ``want_db`` is False).
    """
    x, gy = _f64(x), _f64(gy)
    N = x.shape[0]
    if x.shape != (N, Cp * T) or gy.shape != (N, Dp * T):
        raise ValueError("shape mismatch between x, gy and (T, C', D')")
    p = None
    if pairs is not None:
        p = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
        if p.shape[0] and (p[:, 0].min() < 0 or p[:, 0].max() >= Dp
                           or p[:, 1].min() < 0 or p[:, 1].max() >= Cp):
            raise IndexError("(d, c) pair out of range")
        dW = np.empty((p.shape[0], T), dtype=np.float64)
    else:
        dW = np.empty((Dp, Cp, T), dtype=np.float64)
    db = np.empty((Dp,), dtype=np.float64) if want_db else None
    _load().eqlin_oracle_backward_dw(T, Cp, Dp, N, _ptr(x), _ptr(gy), _ptr(p),
                                     0 if p is None else p.shape[0], _ptr(dW), _ptr(db))
    return dW, db


# ------------------------------------------------------------ other groups
#
# The layer over a finite group G given by its multiplication table (the
# group convolution y[d, g] = b[d] + sum_c sum_h W[d, c, h^-1 g] x[c, h]; for
# the cyclic group Z_T it is the formula above).  A table is a pair
# (mul, inv) of int64 arrays: mul[g, h] = index of g h, inv[g] = index of g^-1.

def cyclic_table(T: int):
    """Z_T with element t (rotation by t steps): t * u = (t + u) mod T."""
    g = np.arange(T)
    mul = (g[:, None] + g[None, :]) % T
    return np.ascontiguousarray(mul, dtype=np.int64), np.ascontiguousarray((-g) % T, dtype=np.int64)


def dihedral_table(m: int):
    """The dihedral group D_m of order 2m (symmetries of a regular m-gon):
    element r^a s^f (rotation by a steps, then f reflections) has index
    f*m + a.  Products follow from s r = r^-1 s:
    (r^a s^f)(r^b s^e) = r^(a + (-1)^f b) s^(f + e)."""
    n = 2 * m
    mul = np.empty((n, n), dtype=np.int64)
    for g in range(n):
        f, a = divmod(g, m)
        for h in range(n):
            e, b = divmod(h, m)
            mul[g, h] = ((f + e) % 2) * m + (a + (b if f == 0 else -b)) % m
    inv = np.array([(g // m) * m + ((-(g % m)) % m if g < m else g % m) for g in range(n)], dtype=np.int64)
    return np.ascontiguousarray(mul), inv


def _table(table):
    mul, inv = (np.ascontiguousarray(np.asarray(a, dtype=np.int64)) for a in table)
    G = inv.shape[0]
    if mul.shape != (G, G):
        raise ValueError("mul must be [G, G]")
    return G, mul, inv


def forward_group(x, W, b, table, rows=None) -> np.ndarray:
    """y = group-convolution layer over the group given by `table`; W [D', C', |G|]."""
    G, mul, inv = _table(table)
    W = _f64(W)
    Dp, Cp, n = W.shape
    if n != G:
        raise ValueError("W's last axis must be the group order")
    x = _f64(x)
    if x.ndim != 2 or x.shape[1] != Cp * G:
        raise ValueError(f"x must be [N, {Cp * G}], got {x.shape}")
    bb = None if b is None else _f64(b)
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n_out = x.shape[0] if r is None else r.shape[0]
    y = np.empty((n_out, Dp * G), dtype=np.float64)
    _load().eqlin_oracle_forward_group(G, _ptr(mul), _ptr(inv), Cp, Dp, _ptr(x), _ptr(W), _ptr(bb),
                                       _ptr(r), n_out, _ptr(y))
    return y


def backward_dx_group(gy, W, table, rows=None) -> np.ndarray:
    G, mul, inv = _table(table)
    W = _f64(W)
    Dp, Cp, _ = W.shape
    gy = _f64(gy)
    if gy.ndim != 2 or gy.shape[1] != Dp * G:
        raise ValueError(f"gy must be [N, {Dp * G}], got {gy.shape}")
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n_out = gy.shape[0] if r is None else r.shape[0]
    dx = np.empty((n_out, Cp * G), dtype=np.float64)
    _load().eqlin_oracle_backward_dx_group(G, _ptr(mul), _ptr(inv), Cp, Dp, _ptr(gy), _ptr(W), _ptr(r), n_out,
                                           _ptr(dx))
    return dx


def backward_dw_group(x, gy, table, Cp: int, Dp: int, want_db: bool = True):
    G, mul, _ = _table(table)
    x, gy = _f64(x), _f64(gy)
    N = x.shape[0]
    if x.shape != (N, Cp * G) or gy.shape != (N, Dp * G):
        raise ValueError("shape mismatch between x, gy and (G, C', D')")
    dW = np.empty((Dp, Cp, G), dtype=np.float64)
    db = np.empty((Dp,), dtype=np.float64) if want_db else None
    _load().eqlin_oracle_backward_dw_group(G, _ptr(mul), Cp, Dp, N, _ptr(x), _ptr(gy), _ptr(dW), _ptr(db))
    return dW, db
