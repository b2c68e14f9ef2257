"""Flash EQ-Linear for NVIDIA B200 (sm_100a).

The layer computes y[n, d*T+s] = b[d] + sum_c sum_t W[d, c, (s-t) mod T] x[n, c*T+t]
through a real DFT along the group axis, per-frequency channel GEMMs on the
half spectrum and an inverse DFT, all inside hand-written CUDA kernels behind
the C ABI declared in ``include/eqlin.h``.

``group_circulant_linear_b200.eqlin`` is the thin Python binding (argument
marshalling only).  Importing this package does not load the CUDA library;
the binding loads it on first use and raises if it is missing.
"""
from . import inputs, workloads  # noqa: F401  (no CUDA needed)

__all__ = ["inputs", "workloads", "eqlin"]


def __getattr__(name):
    if name == "eqlin":
        import importlib
        return importlib.import_module(".eqlin", __name__)
    raise AttributeError(name)
