"""The allocation-free split-K/V entry point (``fa2_fwd_splitkv_static``),
through the C ABI, against the workspace entry point (``fa2_fwd_splitkv``) and
against the fp64 oracle.

Collected last on purpose: it must pass both in a fresh process (the first
call on the device looks up the scratch array's address) and after every
other test.  Calls in a row with different shapes, head dimensions and range
counts: each finds the previous call's partials still in the shared scratch
array.  Tolerances are the parity tests' own (|dO| <= 1e-2 plus half a bf16
spacing of the exact value, |dLSE| <= 1e-3).  The device's free memory is the
same before and after the static calls: the entry point allocates nothing.
"""
import ctypes

import numpy as np
import pytest
import torch

from exact_tiled_attention_45_b200 import binding, fwd_splitkv, splitkv_splits, splitkv_workspace_bytes, sync_status
from exact_tiled_attention_45_b200.inputs import make_q_kv
from oracle import attention_ref_rect

from test_parity_gpu import assert_close

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
LSE_TOL = 1e-3


def _static_call(lib, q, k, v, causal, n_splits, o, lse):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    st = lib.fa2_fwd_splitkv_static(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                    ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                    ctypes.c_void_p(lse.data_ptr()), B, H, Nq, Nk, d, int(causal),
                                    ctypes.c_float(d ** -0.5), n_splits,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == binding.FA2_OK, lib.fa2_last_error_detail()


@pytest.mark.parametrize("order", ["a_then_b", "b_then_a"])
def test_static_scratch_matches_workspace_entry_on_two_calls(order):
    lib = binding.load()
    cases = {
        # (B, H, Nq, Nk, d, causal, n_splits): both use the scratch (>= 2 ranges)
        "a": (2, 4, 1, 5000, 128, True, 6),
        "b": (1, 3, 40, 3000, 64, False, 5),
    }
    seq = ["a", "b"] if order == "a_then_b" else ["b", "a"]
    for i, name in enumerate(seq):
        B, H, Nq, Nk, d, causal, s = cases[name]
        assert splitkv_splits(B, H, Nq, Nk, d, s) >= 2
        assert 0 < splitkv_workspace_bytes(B, H, Nq, Nk, d, s) <= binding.SPLITKV_STATIC_SCRATCH_BYTES
        q, k, v = (t.cuda() for t in make_q_kv(B, H, Nq, Nk, d, seed=30 + i))
        o_ref, l_ref = fwd_splitkv(q, k, v, causal=causal, n_splits=s)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
        _static_call(lib, q, k, v, causal, s, o, lse)
        sync_status()
        do = (o.double() - o_ref.double()).abs().max().item()
        dl = (lse.double() - l_ref.double()).abs().max().item()
        assert np.isfinite(do) and do <= O_TOL, f"call {i} ({name}): |dO| {do}"
        assert np.isfinite(dl) and dl <= LSE_TOL, f"call {i} ({name}): |dLSE| {dl}"


# Every head dimension the entry point accepts, with two or more key ranges
# (so the partials go through the scratch array), in quarter and full-tile
# modes; run back to back so each call meets the previous one's partials.
ORACLE_CASES = [
    # (B, H, Nq, Nk, d, causal, n_splits)
    (1, 2, 1, 3000, 32, True, 4),
    (2, 1, 37, 2100, 96, False, 3),
    (1, 2, 130, 1500, 128, True, 3),
    (1, 2, 5, 1000, 256, True, 4),
    (2, 2, 1, 4097, 64, False, 5),
]


def test_static_scratch_every_head_dim_against_oracle_without_allocating():
    lib = binding.load()
    prepared = []
    for i, (B, H, Nq, Nk, d, causal, s) in enumerate(ORACLE_CASES):
        assert splitkv_splits(B, H, Nq, Nk, d, s) >= 2
        assert 0 < splitkv_workspace_bytes(B, H, Nq, Nk, d, s) <= binding.SPLITKV_STATIC_SCRATCH_BYTES
        q, k, v = make_q_kv(B, H, Nq, Nk, d, seed=50 + i, qk_mult=2.0 if i % 2 else 1.0)
        dev = [t.cuda() for t in (q, k, v)]
        o = torch.empty_like(dev[0])
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=o.device)
        prepared.append(((q, k, v), dev, o, lse, causal, s))
    # Warm-up pass: the first call on the device looks up the scratch address,
    # and the first launch of each kernel may load its code onto the device.
    for _, dev, o, lse, causal, s in prepared:
        _static_call(lib, *dev, causal, s, o, lse)
    sync_status()
    free_before = torch.cuda.mem_get_info()[0]
    for host, dev, o, lse, causal, s in prepared + prepared[:1]:
        _static_call(lib, *dev, causal, s, o, lse)
    sync_status()
    free_after = torch.cuda.mem_get_info()[0]
    assert free_after == free_before, f"device free memory changed by {free_before - free_after} bytes"
    for (q, k, v), dev, o, lse, causal, s in prepared:
        d = q.shape[-1]
        o_ref, l_ref = attention_ref_rect(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                                          scale=d ** -0.5)
        assert_close(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, l_ref,
                     f"static d={d} Nq={q.shape[2]} Nk={k.shape[2]} splits={s}")


def test_static_scratch_rejects_requests_beyond_its_size():
    lib = binding.load()
    q, k, v = (t.cuda() for t in make_q_kv(1, 16, 4096, 4096, 128, seed=40))
    o = torch.empty_like(q)
    lse = torch.empty((1, 16, 4096), dtype=torch.float32, device=q.device)
    # 32 ranges x 16 heads x 4096 rows x 129 floats = 270 MB > 16 MiB
    assert splitkv_workspace_bytes(1, 16, 4096, 4096, 128, 32) > binding.SPLITKV_STATIC_SCRATCH_BYTES
    st = lib.fa2_fwd_splitkv_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                    1, 16, 4096, 4096, 128, 1, 128 ** -0.5, 32,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == binding.FA2_ERR_INVALID_ARG
    assert b"static scratch" in lib.fa2_last_error_detail()
