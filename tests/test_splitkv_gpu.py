"""GPU parity of the split-K/V entry point (few queries, many keys) against the
fp64 oracle, through the C ABI.

Query row i of Nq sits at sequence position Nk - Nq + i; the oracle is
``attention_ref_rect``.  Same tolerances as the square kernel: |dO| <= 1e-2
plus half a bf16 spacing, |dLSE| <= 1e-3.  Cases cover one query (decoding),
a chunk of queries after a prefix (causal and not), Nq == Nk (must agree with
the oracle exactly like ``fwd``), ragged key counts, forced range counts
including more ranges than tiles, ranges that a causal tile never reaches
(empty partials), large logits, and a full-size decode batch on sampled heads.
"""
import numpy as np
import pytest
import torch

from exact_tiled_attention_45_b200 import fwd, fwd_splitkv, splitkv_splits, sync_status
from exact_tiled_attention_45_b200.inputs import make_q_kv, make_qkv
from oracle import attention_ref_rect

from test_parity_gpu import assert_close

pytestmark = pytest.mark.gpu


def make_rect(B, H, Nq, Nk, d, seed=0, mult=1.0):
    return make_q_kv(B, H, Nq, Nk, d, seed=seed, qk_mult=mult)


def run_splitkv(q, k, v, causal, n_splits=0, scale=None):
    o, lse = fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale, n_splits=n_splits)
    sync_status()
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


def oracle(q, k, v, causal, scale=None):
    d = q.shape[-1]
    return attention_ref_rect(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                              scale=d ** -0.5 if scale is None else scale)


CASES = [
    # (B, H, Nq, Nk, d, causal, n_splits, mult)
    (2, 3, 1, 1, 64, False, 0, 1.0),
    (2, 3, 1, 1, 128, True, 0, 1.0),
    (2, 3, 1, 127, 128, False, 0, 1.0),
    (2, 3, 1, 129, 128, True, 0, 1.0),
    (2, 3, 1, 1000, 64, False, 0, 1.0),
    (2, 3, 1, 1000, 128, True, 3, 1.0),
    (1, 4, 1, 4133, 128, False, 0, 1.0),
    (1, 4, 1, 4133, 64, True, 7, 1.0),
    (1, 2, 1, 2048, 128, False, 1, 1.0),
    (1, 2, 1, 2048, 128, False, 16, 1.0),
    (1, 2, 1, 2048, 128, False, 500, 1.0),   # capped at the tile count
    (1, 2, 5, 1500, 128, True, 0, 1.0),
    (1, 2, 5, 1500, 64, False, 4, 1.0),
    (1, 2, 130, 1500, 128, True, 5, 1.0),    # two query tiles, second ragged
    (1, 2, 130, 1500, 64, True, 0, 1.0),
    (1, 2, 300, 300, 128, True, 2, 1.0),     # Nq == Nk
    (2, 2, 1024, 1024, 64, True, 8, 1.0),    # early query tiles meet empty ranges
    (1, 2, 1024, 1024, 128, False, 0, 1.0),
    (1, 2, 1000, 1000, 128, True, 1, 1.0),   # one range: O and LSE written by the range kernel
    (2, 3, 77, 1111, 64, True, 1, 1.0),
    (3, 2, 1, 777, 64, False, 1, 4.0),
    (2, 2, 1, 3000, 128, False, 0, 4.0),     # large logits
    (2, 2, 64, 3000, 128, True, 6, 4.0),
    (2, 2, 64, 3000, 64, True, 0, 4.0),
    # zero-padded head dims
    (1, 2, 1, 3000, 96, True, 0, 1.0),
    (1, 2, 7, 2000, 32, False, 3, 1.0),
    (1, 2, 130, 1500, 96, True, 5, 1.0),
    (2, 1, 1, 900, 32, True, 1, 1.0),
    # two to four queries, long and short key ranges
    (1, 3, 2, 777, 128, True, 0, 1.0),
    (2, 2, 4, 3001, 64, False, 3, 1.0),
    (1, 2, 4, 4, 256, True, 0, 1.0),
    (2, 1, 3, 33, 128, True, 2, 4.0),
    (1, 2, 1, 20000, 64, True, 0, 4.0),
    # quarter mode (at most 32 query rows, d <= 128) at its edges
    (1, 2, 32, 2000, 128, True, 0, 1.0),
    (2, 1, 32, 33, 64, True, 3, 4.0),
    (1, 2, 33, 2000, 128, True, 0, 1.0),     # one row too many: the full-tile mode
    (1, 1, 31, 4096, 96, False, 2, 1.0),
    (3, 2, 1, 95, 32, True, 0, 1.0),         # fewer keys than one warp's quarter of a tile
    # d = 256: 64-key tiles
    (2, 2, 1, 4000, 256, True, 0, 1.0),
    (1, 2, 3, 1500, 256, False, 7, 1.0),
    (1, 2, 130, 1000, 256, True, 3, 4.0),
    (1, 1, 1, 65, 256, False, 2, 1.0),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,n_splits,mult", CASES,
                         ids=[f"B{b}H{h}q{nq}k{nk}d{d}{'c' if c else 'f'}s{s}x{int(m)}"
                              for b, h, nq, nk, d, c, s, m in CASES])
def test_splitkv_elementwise(B, H, Nq, Nk, d, causal, n_splits, mult):
    q, k, v = make_rect(B, H, Nq, Nk, d, seed=11, mult=mult)
    o, lse = run_splitkv(q, k, v, causal, n_splits)
    o_ref, lse_ref = oracle(q, k, v, causal)
    assert_close(o, lse, o_ref, lse_ref, f"Nq={Nq} Nk={Nk} d={d} causal={causal} splits={n_splits}")


def test_splitkv_square_matches_fwd_within_tolerance():
    q, k, v = make_qkv(1, 3, 777, 128, seed=12)
    for causal in (False, True):
        o_s, l_s = run_splitkv(q, k, v, causal, n_splits=3)
        o_f, l_f = fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
        sync_status()
        assert np.abs(o_s - o_f.double().cpu().numpy()).max() <= 2e-2
        assert np.abs(l_s - l_f.double().cpu().numpy()).max() <= 1e-3


def test_single_query_causal_equals_non_causal():
    # the last position sees every key
    q, k, v = make_rect(2, 2, 1, 2500, 128, seed=13)
    oc, lc = run_splitkv(q, k, v, True, 4)
    of, lf = run_splitkv(q, k, v, False, 4)
    assert np.array_equal(oc, of) and np.array_equal(lc, lf)


def test_split_count_changes_only_rounding():
    q, k, v = make_rect(1, 4, 3, 5000, 64, seed=14)
    o_ref, lse_ref = oracle(q, k, v, False)
    for s in (1, 2, 9, 40):
        o, lse = run_splitkv(q, k, v, False, s)
        assert_close(o, lse, o_ref, lse_ref, f"splits={s}")


def test_splitkv_repeatable_bitwise():
    q, k, v = (t.cuda() for t in make_rect(2, 4, 8, 3000, 128, seed=15))
    o1, l1 = fwd_splitkv(q, k, v, causal=True, n_splits=5)
    o2, l2 = fwd_splitkv(q, k, v, causal=True, n_splits=5)
    sync_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_non_default_scale():
    q, k, v = make_rect(1, 2, 17, 900, 128, seed=16)
    o, lse = run_splitkv(q, k, v, True, 0, scale=0.05)
    o_ref, lse_ref = oracle(q, k, v, True, scale=0.05)
    assert_close(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("mult", [1.0, 4.0], ids=["x1", "x4"])
def test_decode_full_size_sampled_heads(mult):
    # The decode workload: B=8, H=16, one query against 16384 keys, d=128.
    B, H, Nk, d = 8, 16, 16384, 128
    q, k, v = make_rect(B, H, 1, Nk, d, seed=0, mult=mult)
    assert splitkv_splits(B, H, 1, Nk, d) >= 1
    o_d, lse_d = fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=True)
    sync_status()
    o_all, lse_all = o_d.cpu(), lse_d.cpu()
    assert torch.isfinite(o_all.float()).all() and torch.isfinite(lse_all).all()
    rng = np.random.default_rng(2)
    heads = {(0, 0), (B - 1, H - 1)} | {(int(rng.integers(B)), int(rng.integers(H))) for _ in range(4)}
    for b, h in sorted(heads):
        o_ref, lse_ref = oracle(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], True)
        assert_close(o_all[b:b + 1, h:h + 1].double().numpy(), lse_all[b:b + 1, h:h + 1].double().numpy(),
                     o_ref, lse_ref, f"decode head ({b},{h}) x{mult}")
