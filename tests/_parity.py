"""Comparison helpers shared by the GPU parity tests.

Every comparison is recorded with the error it achieved, so that a run shows
how far each output sits from its tolerance, not only whether it passed; the
table is printed at the end of the pytest run (tests/conftest.py) and, when
the environment variable EQLIN_PARITY_LOG names a file, written there as JSON.

Tolerances (relative Frobenius norm of the difference, i.e. RMS(err)/RMS(ref)):
FP32 1e-5; FP16/BF16 with FP32 accumulation 2e-2.  max|err|/RMS(ref) is
recorded beside it for information.
"""
from __future__ import annotations

import math

import numpy as np

TOL = {"f32": 1e-5, "f16": 2e-2, "bf16": 2e-2}
RECORDS: list[dict] = []


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().float().cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def rel_err(out, ref) -> float:
    out, ref = _f64(out), _f64(ref)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(out - ref) / (den if den > 0 else 1.0))


class Accum:
    """Running sums for a comparison done in pieces (row blocks of a large output)."""

    def __init__(self):
        self.se = 0.0      # sum of squared errors
        self.sr = 0.0      # sum of squared reference values
        self.mx = 0.0      # max |err|
        self.n = 0
        self.mismatches = 0

    def add(self, out, ref):
        out, ref = _f64(out), _f64(ref)
        assert out.shape == ref.shape, (out.shape, ref.shape)
        d = out - ref
        self.se += float((d * d).sum())
        self.sr += float((ref * ref).sum())
        self.mx = max(self.mx, float(np.abs(d).max()) if d.size else 0.0)
        self.n += d.size
        self.mismatches += int(np.count_nonzero(d))

    @property
    def rel(self) -> float:
        return math.sqrt(self.se / self.sr) if self.sr > 0 else math.sqrt(self.se)

    @property
    def max_over_rms(self) -> float:
        rms = math.sqrt(self.sr / self.n) if self.n and self.sr > 0 else 1.0
        return self.mx / rms


def finish(label: str, acc: Accum, tol: float, kind: str = "tolerance"):
    """Record an accumulated comparison and assert it (exact: no mismatching element)."""
    RECORDS.append({"case": label, "kind": kind, "rel_err": acc.rel, "max_over_rms": acc.max_over_rms,
                    "tol": tol, "elements": acc.n, "mismatches": acc.mismatches})
    if kind == "exact":
        assert acc.mismatches == 0, f"{label}: {acc.mismatches} of {acc.n} elements differ (max |err| {acc.mx})"
    else:
        assert acc.rel <= tol, f"{label}: relative error {acc.rel:.3e} > {tol:.1e}"


def check(label: str, out, ref, tol: float):
    a = Accum()
    a.add(out, ref)
    finish(label, a, tol)


def check_exact(label: str, out, ref):
    a = Accum()
    a.add(out, ref)
    finish(label, a, 0.0, kind="exact")
