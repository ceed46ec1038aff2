"""Failure path on the GPU without a fault: the kernel's bounded waits.

The test hook withholds the query-tile load, so the MMA warp's wait on it can
never complete.  Every wait in the kernel is bounded: after the time limit the
kernel records a status word, drains its own in-flight copies, frees tensor
memory and returns.  The host reads FA2_ERR_TIMEOUT, and the context stays
usable: a normal call right after matches the oracle.
"""
import numpy as np
import pytest

from exact_tiled_attention_45_b200 import binding, fwd, fwd_inject_timeout, sync_status
from exact_tiled_attention_45_b200.inputs import make_qkv
from oracle import attention_ref

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_withheld_load_times_out_and_context_survives(d, causal):
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 256, d, seed=0))
    status = fwd_inject_timeout(q, k, v, causal=causal, timeout_ns=50_000_000)
    assert status == binding.FA2_ERR_TIMEOUT
    # status word is cleared by the read
    sync_status()
    o, lse = fwd(q, k, v, causal=causal)
    sync_status()
    o_ref, lse_ref = attention_ref(q.double().cpu().numpy(), k.double().cpu().numpy(), v.double().cpu().numpy(),
                                   causal=causal, scale=d ** -0.5)
    assert np.abs(o.double().cpu().numpy() - o_ref).max() <= 2e-2
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() <= 1e-3
