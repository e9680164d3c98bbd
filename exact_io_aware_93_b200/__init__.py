"""exact_io_aware_93_b200 -- exact attention, FlashAttention-style, for B200 (sm_100a).

softmax(scale * Q K^T) V and its recompute backward, computed by hand-written
sm_100a kernels behind a C ABI (``include/fa.h``).  Python only marshals
arguments: ``fwd`` / ``bwd`` call ``fa_fwd`` / ``fa_bwd`` in the compiled
library and fail loudly when it is missing.
"""
__all__ = ["fwd", "bwd", "attention"]


def __getattr__(name):
    if name in ("fwd", "bwd", "attention", "FAError"):
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
