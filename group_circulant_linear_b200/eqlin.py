"""Thin Python binding of the C ABI in ``include/eqlin.h`` (ctypes).

The functions carry the ABI's names (``eqlin_create`` -> ``create`` and so on)
and do argument marshalling only: they check that tensors are contiguous CUDA
tensors of the handle's dtype and shape, then pass raw device pointers and the
current CUDA stream.  Every step of the layer runs in ``libeqlin.so``.  There
is no fallback: if the library is missing or the call fails, this module
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libeqlin.so")

F32, F16, BF16 = 0, 1, 2
CYCLIC, DIHEDRAL = 0, 1
_GROUPS = {"cyclic": CYCLIC, "dihedral": DIHEDRAL}
_DT = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}
_TORCH_DT = {v: k for k, v in _DT.items()}
_NAMES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}

STATUS = {0: "EQLIN_OK", -1: "EQLIN_ERR_INVALID_ARG", -2: "EQLIN_ERR_UNSUPPORTED",
          -3: "EQLIN_ERR_MISALIGNED", -4: "EQLIN_ERR_CUDA", -5: "EQLIN_ERR_NO_WEIGHTS",
          -6: "EQLIN_ERR_TIMEOUT", -7: "EQLIN_ERR_OOM"}

# Every entry point include/eqlin.h declares, with its ctypes signature.
_vp, _i64, _int, _u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32
SIGNATURES = {
    "eqlin_create": ([_int, _i64, _i64, _int, ctypes.POINTER(_vp)], _int),
    "eqlin_create_group": ([_int, _int, _i64, _i64, _int, ctypes.POINTER(_vp)], _int),
    "eqlin_set_weights": ([_vp, _vp, _vp, _vp], _int),
    "eqlin_forward": ([_vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_forward_gauss": ([_vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_backward_dx": ([_vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_backward_dw": ([_vp, _vp, _vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_get_error": ([_vp], _int),
    "eqlin_error_detail": ([_vp, ctypes.POINTER(ctypes.c_uint32)], _int),
    "eqlin_set_wait_limit": ([_vp, _u32], _int),
    "eqlin_set_tail_split": ([_vp, _int], _int),
    "eqlin_backend_name": ([_vp], ctypes.c_char_p),
    "eqlin_status_string": ([_int], ctypes.c_char_p),
    "eqlin_launch_count": ([], ctypes.c_uint64),
    "eqlin_backward_dw_noalloc": ([_int, _i64, _i64, _int, _vp, _vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_spectra_ld": ([_i64], _i64),
    "eqlin_forward_stash": ([_vp, _vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_backward_dx_stash": ([_vp, _vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_backward_dw_spectra": ([_vp, _vp, _vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_backward": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp], _int),
    "eqlin_destroy": ([_vp], None),
}

_lib = None


class EqlinError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().eqlin_status_string(status).decode() if _lib else str(status)
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


def lib():
    """Load libeqlin.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m group_circulant_linear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise EqlinError(status, where)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev_ptr(t: torch.Tensor, dtype, shape, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


class Handle:
    """An eqlin_t plus the layer shape it was created for.

    ``T`` is the group order (the length of the group axis).  For
    ``group="dihedral"`` pass ``m`` (D_m, order 2m) and T = 2m, or T = None."""

    def __init__(self, T, Cp: int, Dp: int, dtype, group="cyclic", m: int | None = None):
        if isinstance(dtype, str):
            dtype = _NAMES[dtype]
        self.group = _GROUPS[group] if isinstance(group, str) else int(group)
        if self.group == DIHEDRAL:
            if m is None:
                m = int(T) // 2
            self.m = int(m)
            T = 2 * self.m
        else:
            self.m = int(T)
        self.T, self.Cp, self.Dp, self.dtype = int(T), int(Cp), int(Dp), dtype
        out = ctypes.c_void_p()
        _check(lib().eqlin_create_group(self.group, self.m, self.Cp, self.Dp, _DT[dtype], ctypes.byref(out)),
               "eqlin_create_group")
        self._h = out

    @property
    def ptr(self):
        return self._h

    def close(self):
        if self._h:
            lib().eqlin_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def backend(self) -> str:
        return lib().eqlin_backend_name(self._h).decode()

    def __copy__(self):
        raise TypeError("a Handle owns device buffers; use copy.deepcopy for a new handle of the same shape")

    def __deepcopy__(self, memo):
        # a new handle of the same shape; it holds no weights until set_weights
        return Handle(self.T, self.Cp, self.Dp, self.dtype, group=self.group, m=self.m)


# ------------------------------------------------------------------ the ABI

def create(T: int, Cp: int, Dp: int, dtype) -> Handle:
    return Handle(T, Cp, Dp, dtype)


def create_group(group, m: int, Cp: int, Dp: int, dtype) -> Handle:
    """A layer over the cyclic group Z_m or the dihedral group D_m (order 2m)."""
    g = _GROUPS[group] if isinstance(group, str) else int(group)
    return Handle(m if g == CYCLIC else 2 * m, Cp, Dp, dtype, group=g, m=m)


def set_weights(h: Handle, W: torch.Tensor, b: torch.Tensor | None = None, stream=None):
    pw = _dev_ptr(W, h.dtype, (h.Dp, h.Cp, h.T), "W")
    pb = None if b is None else _dev_ptr(b, h.dtype, (h.Dp,), "b")
    _check(lib().eqlin_set_weights(h.ptr, pw, pb, _stream(stream)), "eqlin_set_weights")


def forward(h: Handle, x: torch.Tensor, y: torch.Tensor, stream=None):
    N = x.shape[0]
    px = _dev_ptr(x, h.dtype, (N, h.Cp * h.T), "x")
    py = _dev_ptr(y, h.dtype, (N, h.Dp * h.T), "y")
    _check(lib().eqlin_forward(h.ptr, px, py, N, _stream(stream)), "eqlin_forward")


def forward_gauss(h: Handle, x: torch.Tensor, y: torch.Tensor, stream=None):
    """eqlin_forward with the complex products as three real GEMMs (p4 only)."""
    N = x.shape[0]
    px = _dev_ptr(x, h.dtype, (N, h.Cp * h.T), "x")
    py = _dev_ptr(y, h.dtype, (N, h.Dp * h.T), "y")
    _check(lib().eqlin_forward_gauss(h.ptr, px, py, N, _stream(stream)), "eqlin_forward_gauss")


def backward_dx(h: Handle, gy: torch.Tensor, dx: torch.Tensor, stream=None):
    N = gy.shape[0]
    pg = _dev_ptr(gy, h.dtype, (N, h.Dp * h.T), "gy")
    pd = _dev_ptr(dx, h.dtype, (N, h.Cp * h.T), "dx")
    _check(lib().eqlin_backward_dx(h.ptr, pg, pd, N, _stream(stream)), "eqlin_backward_dx")


def backward_dw(h: Handle, x: torch.Tensor, gy: torch.Tensor, dW: torch.Tensor,
                db: torch.Tensor | None = None, stream=None):
    N = x.shape[0]
    px = _dev_ptr(x, h.dtype, (N, h.Cp * h.T), "x")
    pg = _dev_ptr(gy, h.dtype, (N, h.Dp * h.T), "gy")
    pw = _dev_ptr(dW, torch.float32, (h.Dp, h.Cp, h.T), "dW")
    pb = None if db is None else _dev_ptr(db, torch.float32, (h.Dp,), "db")
    _check(lib().eqlin_backward_dw(h.ptr, px, pg, pw, pb, N, _stream(stream)), "eqlin_backward_dw")


def spectra_ld(N: int) -> int:
    """Row pitch (tokens) of a spectra buffer for N tokens."""
    return int(lib().eqlin_spectra_ld(int(N)))


def spectra_shape(h: Handle, which: str, N: int) -> tuple:
    """Shape of the spectra buffer of the input ("x": [T, C', ld]) or of the
    output gradient ("gy": [T, D', ld]) for N tokens."""
    ch = {"x": h.Cp, "gy": h.Dp}[which]
    return (h.T, ch, spectra_ld(N))


def empty_spectra(h: Handle, which: str, N: int, device=None) -> torch.Tensor:
    return torch.empty(spectra_shape(h, which, N), dtype=h.dtype, device=device or "cuda")


def forward_stash(h: Handle, x: torch.Tensor, y: torch.Tensor, xs: torch.Tensor, stream=None):
    """Forward that also writes X = DFT(x) into xs [T, C', ld]."""
    N = x.shape[0]
    px = _dev_ptr(x, h.dtype, (N, h.Cp * h.T), "x")
    py = _dev_ptr(y, h.dtype, (N, h.Dp * h.T), "y")
    ps = _dev_ptr(xs, h.dtype, spectra_shape(h, "x", N), "xs")
    _check(lib().eqlin_forward_stash(h.ptr, px, py, ps, N, _stream(stream)), "eqlin_forward_stash")


def backward_dx_stash(h: Handle, gy: torch.Tensor, dx: torch.Tensor, gs: torch.Tensor, stream=None):
    """Input gradient that also writes G = DFT(gy) into gs [T, D', ld]."""
    N = gy.shape[0]
    pg = _dev_ptr(gy, h.dtype, (N, h.Dp * h.T), "gy")
    pd = _dev_ptr(dx, h.dtype, (N, h.Cp * h.T), "dx")
    ps = _dev_ptr(gs, h.dtype, spectra_shape(h, "gy", N), "gs")
    _check(lib().eqlin_backward_dx_stash(h.ptr, pg, pd, ps, N, _stream(stream)), "eqlin_backward_dx_stash")


def backward_dw_spectra(h: Handle, xs: torch.Tensor, gs: torch.Tensor, N: int, dW: torch.Tensor,
                        db: torch.Tensor | None = None, stream=None):
    """dW, db from the spectra of the same N tokens."""
    pxs = _dev_ptr(xs, h.dtype, spectra_shape(h, "x", N), "xs")
    pgs = _dev_ptr(gs, h.dtype, spectra_shape(h, "gy", N), "gs")
    pw = _dev_ptr(dW, torch.float32, (h.Dp, h.Cp, h.T), "dW")
    pb = None if db is None else _dev_ptr(db, torch.float32, (h.Dp,), "db")
    _check(lib().eqlin_backward_dw_spectra(h.ptr, pxs, pgs, pw, pb, int(N), _stream(stream)),
           "eqlin_backward_dw_spectra")


def backward(h: Handle, gy: torch.Tensor, xs: torch.Tensor, dx: torch.Tensor, gs: torch.Tensor,
             dW: torch.Tensor, db: torch.Tensor | None = None, stream=None):
    """The whole backward (dx, dW, db) given the forward's stash xs; writes gs."""
    N = gy.shape[0]
    pg = _dev_ptr(gy, h.dtype, (N, h.Dp * h.T), "gy")
    pxs = _dev_ptr(xs, h.dtype, spectra_shape(h, "x", N), "xs")
    pd = _dev_ptr(dx, h.dtype, (N, h.Cp * h.T), "dx")
    pgs = _dev_ptr(gs, h.dtype, spectra_shape(h, "gy", N), "gs")
    pw = _dev_ptr(dW, torch.float32, (h.Dp, h.Cp, h.T), "dW")
    pb = None if db is None else _dev_ptr(db, torch.float32, (h.Dp,), "db")
    _check(lib().eqlin_backward(h.ptr, pg, pxs, pd, pgs, pw, pb, N, _stream(stream)), "eqlin_backward")


def backward_dw_noalloc(T: int, x: torch.Tensor, gy: torch.Tensor, dW: torch.Tensor,
                        db: torch.Tensor | None = None, stream=None):
    """dW/db with no handle and no device allocation (see eqlin_backward_dw_noalloc)."""
    Dp, Cp = dW.shape[0], dW.shape[1]
    N = x.shape[0]
    px = _dev_ptr(x, x.dtype, (N, Cp * T), "x")
    pg = _dev_ptr(gy, x.dtype, (N, Dp * T), "gy")
    pw = _dev_ptr(dW, torch.float32, (Dp, Cp, T), "dW")
    pb = None if db is None else _dev_ptr(db, torch.float32, (Dp,), "db")
    _check(lib().eqlin_backward_dw_noalloc(T, Cp, Dp, _DT[x.dtype], px, pg, pw, pb, N, _stream(stream)),
           "eqlin_backward_dw_noalloc")


def get_error(h: Handle) -> int:
    """Device-side status (0, or -6 for a wait that timed out); clears it."""
    return int(lib().eqlin_get_error(h.ptr))


def error_detail(h: Handle) -> dict:
    """Where the last non-OK eqlin_get_error came from (see eqlin_error_detail)."""
    d = (ctypes.c_uint32 * 4)()
    _check(lib().eqlin_error_detail(h.ptr, d), "eqlin_error_detail")
    return {"status": d[0], "kernel": d[1] >> 8, "role": (d[1] >> 4) & 15, "barrier": d[1] & 15,
            "cta": d[2] & 0xFFF, "iteration": d[2] >> 12, "polls": d[3] & 0xFFFFF, "ms": d[3] >> 20}


def set_tail_split(h: Handle, enable: bool):
    """Split the last wave's tiles of the f16/bf16 forward and dx over two SMs
    each (off by default): shorter lone calls, at the price of extra work."""
    _check(lib().eqlin_set_tail_split(h.ptr, 1 if enable else 0), "eqlin_set_tail_split")


def set_wait_limit(h: Handle, iterations: int):
    _check(lib().eqlin_set_wait_limit(h.ptr, int(iterations)), "eqlin_set_wait_limit")


def launch_count() -> int:
    """Kernels the library has enqueued in this process (all handles)."""
    return int(lib().eqlin_launch_count())


def status_string(status: int) -> str:
    return lib().eqlin_status_string(int(status)).decode()


def destroy(h: Handle):
    h.close()


# ------------------------------------------------------- allocating helpers

class EQLinear:
    """Convenience wrapper: owns a handle and allocates outputs with torch."""

    def __init__(self, W: torch.Tensor, b: torch.Tensor | None = None, group="cyclic"):
        Dp, Cp, T = W.shape
        if group == "dihedral":
            self.h = create_group("dihedral", T // 2, Cp, Dp, W.dtype)
        else:
            self.h = create(T, Cp, Dp, W.dtype)
        self.set_weights(W, b)

    def set_weights(self, W, b=None, stream=None):
        set_weights(self.h, W.contiguous(), None if b is None else b.contiguous(), stream)

    def forward(self, x, stream=None):
        y = torch.empty((x.shape[0], self.h.Dp * self.h.T), dtype=self.h.dtype, device=x.device)
        forward(self.h, x, y, stream)
        return y

    def backward_dx(self, gy, stream=None):
        dx = torch.empty((gy.shape[0], self.h.Cp * self.h.T), dtype=self.h.dtype, device=gy.device)
        backward_dx(self.h, gy, dx, stream)
        return dx

    def backward_dw(self, x, gy, stream=None):
        dW = torch.empty((self.h.Dp, self.h.Cp, self.h.T), dtype=torch.float32, device=x.device)
        db = torch.empty((self.h.Dp,), dtype=torch.float32, device=x.device)
        backward_dw(self.h, x, gy, dW, db, stream)
        return dW, db
