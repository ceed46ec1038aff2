"""GPU parity on seeded random shapes: forward, split-K/V and backward against
the fp64 oracle, at the tolerances of the dedicated parity tests.

The shapes are drawn once from a fixed seed (listed in the test ids): batch
and head counts 1-3, sequence lengths 1-700 (so most are ragged against the
64- and 128-row tiles), every supported head dimension, causal or not, the
default scale or another one drawn from [0.05, 0.3], and for split-K/V a query
count up to the key count and a range count from 0 (library choice) to 7.
These combinations are not covered one by one by the hand-written cases.
"""
import numpy as np
import pytest
import torch

from exact_tiled_attention_45_b200 import bwd, fwd, fwd_splitkv, sync_status
from exact_tiled_attention_45_b200.inputs import make_q_kv, make_qkv
from oracle import attention_bwd_ref, attention_ref, attention_ref_rect

from test_bwd_gpu import check as check_grads
from test_bwd_gpu import make_dout
from test_parity_gpu import assert_close

pytestmark = pytest.mark.gpu

D_CHOICES = (32, 64, 96, 128, 256)


def draw(n, seed, rect=False):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        B, H = int(rng.integers(1, 4)), int(rng.integers(1, 4))
        N = int(rng.choice([int(rng.integers(1, 130)), int(rng.integers(130, 701))]))
        d = int(rng.choice(D_CHOICES))
        causal = bool(rng.integers(0, 2))
        scale = None if rng.random() < 0.5 else float(np.round(rng.uniform(0.05, 0.3), 4))
        if rect:
            Nq = int(rng.integers(1, N + 1)) if rng.random() < 0.5 else int(rng.integers(1, min(N, 33) + 1))
            splits = int(rng.integers(0, 8))
            out.append((B, H, Nq, N, d, causal, scale, splits))
        else:
            out.append((B, H, N, d, causal, scale))
    return out


FWD = draw(14, 4001)
SKV = draw(12, 4002, rect=True)
BWD = draw(10, 4003)


def fid(c):
    return "-".join(str(x) for x in c)


@pytest.mark.parametrize("B,H,N,d,causal,scale", FWD, ids=[fid(c) for c in FWD])
def test_fwd_random_shape(B, H, N, d, causal, scale):
    q, k, v = make_qkv(B, H, N, d, seed=N + d)
    o, lse = fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    sync_status()
    o_ref, lse_ref = attention_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                                   scale=d ** -0.5 if scale is None else scale)
    assert_close(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref, f"fwd {B,H,N,d,causal,scale}")


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,scale,splits", SKV, ids=[fid(c) for c in SKV])
def test_splitkv_random_shape(B, H, Nq, Nk, d, causal, scale, splits):
    q, k, v = make_q_kv(B, H, Nq, Nk, d, seed=Nq + Nk + d)
    o, lse = fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale, n_splits=splits)
    sync_status()
    o_ref, lse_ref = attention_ref_rect(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                                        scale=d ** -0.5 if scale is None else scale)
    assert_close(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref,
                 f"split-K/V {B,H,Nq,Nk,d,causal,scale,splits}")


@pytest.mark.parametrize("B,H,N,d,causal,scale", BWD, ids=[fid(c) for c in BWD])
def test_bwd_random_shape(B, H, N, d, causal, scale):
    q, k, v = make_qkv(B, H, N, d, seed=2 * N + d)
    do = make_dout(B, H, N, d, seed=N + 7)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = fwd(qd, kd, vd, causal=causal, scale=scale)
    grads = bwd(qd, kd, vd, o, lse, do.cuda(), causal=causal, scale=scale)
    sync_status()
    ref = attention_bwd_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                            causal=causal, scale=d ** -0.5 if scale is None else scale)
    check_grads([g.double().cpu().numpy() for g in grads], ref, f"bwd {B,H,N,d,causal,scale}")
