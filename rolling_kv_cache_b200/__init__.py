"""Bounded rolling KV cache for block-autoregressive video diffusion on B200.

The hot path lives in librc.so (C ABI in include/rc.h, CUDA kernels for
sm_100a); this package is its ctypes binding plus a small torch-facing
wrapper. Importing it does not load the library; the first call does, and
fails loudly if the library is missing.
"""
from .binding import (RC_INFINITY_ROPE, RC_NONE, RC_REINDEX_CUT, RC_REINDEX_FLUSH,
                      RC_REINDEX_SINK, RC_ROLLING_SINK, RC_SLIDING, RcError)

__all__ = ["RC_NONE", "RC_SLIDING", "RC_ROLLING_SINK", "RC_INFINITY_ROPE", "RC_REINDEX_FLUSH",
           "RC_REINDEX_CUT", "RC_REINDEX_SINK", "RcError", "RollingKVCache", "make_config"]


def __getattr__(name):
    if name in ("RollingKVCache", "make_config"):
        from . import cache
        return getattr(cache, name)
    raise AttributeError(name)
