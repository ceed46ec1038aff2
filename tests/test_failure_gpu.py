"""Failure path on the GPU without a fault: every kernel's bounded waits.

Each test hook withholds one tile load of one kernel, so the waits on it can
never complete.  Every wait is bounded: after the time limit (50 ms here) the
kernel records the device status word, drains its own in-flight copies and
MMAs, frees tensor memory and returns.  The host reads FA2_ERR_TIMEOUT, and
the context stays usable: a normal call right after (which would block on the
tensor-memory allocation if any CTA had kept its columns) matches the fp64
oracle at the parity tests' tolerance.

Kernels covered: the forward kernel (64- and 128-column tiles), the d = 256
forward (the one-tile kernel of the split-K/V path), the split-K/V range
kernel in full-tile and quarter mode with two or more key ranges (so the
merge kernel also runs, on the unspecified partials, after the time-out),
and each of the two backward kernels.  Grids stay below one wave, so every
CTA times out at the same time.
"""
import numpy as np
import pytest
import torch

from exact_tiled_attention_45_b200 import (binding, bwd, bwd_inject_timeout, fwd, fwd_inject_timeout, fwd_splitkv,
                                           fwd_splitkv_inject_timeout, splitkv_splits, sync_status)
from exact_tiled_attention_45_b200.inputs import make_q_kv, make_qkv
from oracle import attention_bwd_ref, attention_ref, attention_ref_rect

from test_parity_gpu import assert_close

pytestmark = pytest.mark.gpu

TIMEOUT_NS = 50_000_000


@pytest.mark.parametrize("d,causal", [(64, False), (128, True), (32, True), (96, False), (256, True),
                                      (256, False)])
def test_forward_withheld_load_times_out_and_context_survives(d, causal):
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 256, d, seed=0))
    status = fwd_inject_timeout(q, k, v, causal=causal, timeout_ns=TIMEOUT_NS)
    assert status == binding.FA2_ERR_TIMEOUT
    sync_status()  # the read cleared the status word
    o, lse = fwd(q, k, v, causal=causal)
    sync_status()
    o_ref, lse_ref = attention_ref(q.double().cpu().numpy(), k.double().cpu().numpy(), v.double().cpu().numpy(),
                                   causal=causal, scale=d ** -0.5)
    assert_close(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref, f"after time-out d={d}")


SPLITKV = [
    # (B, H, Nq, Nk, d, causal, n_splits): >= 2 ranges so the merge runs
    (1, 2, 1, 2000, 128, True, 4),     # quarter mode (Nq <= 32)
    (2, 1, 20, 1500, 64, False, 3),    # quarter mode, several rows
    (1, 2, 130, 1500, 128, True, 3),   # full-tile mode, two query tiles
    (1, 2, 40, 1000, 64, False, 2),    # full-tile mode (Nq > 32)
    (1, 2, 3, 1000, 256, True, 2),     # 64-key tiles
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,n_splits", SPLITKV,
                         ids=[f"q{nq}k{nk}d{d}s{s}" for _, _, nq, nk, d, _, s in SPLITKV])
def test_splitkv_withheld_load_times_out_and_context_survives(B, H, Nq, Nk, d, causal, n_splits):
    assert splitkv_splits(B, H, Nq, Nk, d, n_splits) >= 2
    q, k, v = (t.cuda() for t in make_q_kv(B, H, Nq, Nk, d, seed=3))
    status = fwd_splitkv_inject_timeout(q, k, v, causal=causal, n_splits=n_splits, timeout_ns=TIMEOUT_NS)
    assert status == binding.FA2_ERR_TIMEOUT
    sync_status()
    o, lse = fwd_splitkv(q, k, v, causal=causal, n_splits=n_splits)
    sync_status()
    o_ref, lse_ref = attention_ref_rect(q.double().cpu().numpy(), k.double().cpu().numpy(),
                                        v.double().cpu().numpy(), causal=causal, scale=d ** -0.5)
    assert_close(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref,
                 f"after time-out Nq={Nq} Nk={Nk} d={d}")


@pytest.mark.parametrize("kernel", [0, 1], ids=["dq_kernel", "dkdv_kernel"])
@pytest.mark.parametrize("d,causal", [(64, True), (128, False), (256, True)])
def test_backward_withheld_load_times_out_and_context_survives(kernel, d, causal):
    B, H, N = 1, 2, 300
    q, k, v = make_qkv(B, H, N, d, seed=5)
    g = torch.Generator(device="cpu")
    g.manual_seed(6)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fwd(qd, kd, vd, causal=causal)
    sync_status()
    status = bwd_inject_timeout(qd, kd, vd, o, lse, dod, kernel, causal=causal, timeout_ns=TIMEOUT_NS)
    assert status == binding.FA2_ERR_TIMEOUT
    sync_status()
    grads = bwd(qd, kd, vd, o, lse, dod, causal=causal)
    sync_status()
    refs = attention_bwd_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                             causal=causal, scale=d ** -0.5)
    for name, got, ref in zip(("dQ", "dK", "dV"), grads, refs):
        err = np.abs(got.double().cpu().numpy() - ref)
        assert np.isfinite(err).all() and err.max() <= 2.0 ** -6 * np.abs(ref).max(), f"{name} after time-out"

