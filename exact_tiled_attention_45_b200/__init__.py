"""B200-native (sm_100a) exact attention forward (FlashAttention-2 style).

``fwd(q, k, v, causal, scale) -> (O, LSE)`` runs the tiled, online-softmax
forward in the hand-written CUDA kernels of ``libfa2.so`` (C ABI declared in
``include/fa2.h``).  The library is loaded on first use; nothing here falls
back to another implementation.
"""
from .binding import (EXPORTS, FA2Error, fwd, fwd_host, fwd_inject_timeout, load,  # noqa: F401
                      sync_status, workspace_bytes)

__all__ = ["fwd", "fwd_host", "fwd_inject_timeout", "load", "sync_status", "workspace_bytes", "FA2Error",
           "EXPORTS"]
