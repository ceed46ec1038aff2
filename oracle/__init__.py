"""fp64 CPU oracle for exact attention -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs import this package.  The CUDA path never does.
"""
from .attention import (attention_bwd_ref, attention_bwd_ref_rows, attention_probs, attention_ref,  # noqa: F401
                        attention_ref_rect, attention_ref_rows)
