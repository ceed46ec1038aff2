"""B200-native (sm_100a) exact attention forward (FlashAttention-2 style).

``fwd(q, k, v, causal, scale) -> (O, LSE)`` runs the tiled, online-softmax
forward, and ``fwd_splitkv`` the same operation for few queries against many
keys (decoding) with the keys split over CTAs, and ``bwd`` the gradients, in the hand-written CUDA kernels of ``libfa2.so`` (C ABI declared in
``include/fa2.h``).  The library is loaded on first use; nothing here falls
back to another implementation.
"""
from .binding import (EXPORTS, FA2Error, bwd, bwd_inject_timeout, bwd_workspace_bytes, fwd, fwd_host,  # noqa: F401
                      fwd_inject_timeout, fwd_splitkv, fwd_splitkv_inject_timeout, fwd_splitkv_static, load,
                      splitkv_splits, splitkv_workspace_bytes, sync_status, workspace_bytes)

__all__ = ["fwd", "bwd", "bwd_inject_timeout", "bwd_workspace_bytes", "fwd_host", "fwd_inject_timeout",
           "fwd_splitkv", "fwd_splitkv_inject_timeout", "fwd_splitkv_static", "load", "splitkv_splits",
           "splitkv_workspace_bytes", "sync_status", "workspace_bytes", "FA2Error", "EXPORTS"]
