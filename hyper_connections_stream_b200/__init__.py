"""B200-native Hyper-Connections residual step.

The step (write mix, read mix + pre-norm RMSNorm, mHC Sinkhorn projection) runs
in hand-written sm_100a CUDA kernels behind the C-ABI library libhc_b200.so
(declared in include/hc_api.h). This package is the thin Python binding: it
marshals torch tensors into pointers and a stream handle and calls the library.
There is no CPU fallback: if the library is missing the calls raise.

Import of the binding is lazy so that host-only helpers (traffic) load without
CUDA.
"""
from __future__ import annotations

__all__ = ["sinkhorn", "read_rmsnorm", "write_mix", "write_then_read", "HCError",
           "MIX_MATRIX", "MIX_SINKHORN_LOGITS", "READ_WEIGHTS", "READ_SOFTMAX_LOGITS"]


def __getattr__(name):
    if name in __all__ or name in ("lib", "status_string"):
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
