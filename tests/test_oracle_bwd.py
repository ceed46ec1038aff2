"""Pins for the oracle's backward (dQ, dK, dV of exact attention).  No GPU.

Each pin checks the gradients against something other than their own
formulas: central finite differences of the (separately pinned) forward
oracle, torch autograd of torch's own attention in float64, and closed forms
of special cases (constant V, a single key, zero upstream gradient) and
invariants (the key gradients of a head sum to zero; dQ does not change when
every key is shifted by one vector).  Planted mistakes in the backward
formulas must each fail at least one pin.
"""
import numpy as np
import pytest
import torch

import oracle.attention as oa
from oracle import attention_bwd_ref, attention_bwd_ref_rows, attention_ref


def _rand(shape, seed, mult=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * mult


def _case(B=1, H=2, N=9, d=4, seed=0, mult=1.0):
    return (_rand((B, H, N, d), seed, mult), _rand((B, H, N, d), seed + 1, mult), _rand((B, H, N, d), seed + 2),
            _rand((B, H, N, d), seed + 3))


def pin_finite_differences(f):
    # d/dx of F = sum(O * dO) by central differences of the forward oracle.
    for causal in (False, True):
        q, k, v, do = _case(1, 1, 5, 3, seed=10)
        scale = 0.7
        dq, dk, dv = f(q, k, v, do, causal=causal, scale=scale)
        h = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = {"q": q, "k": k, "v": v, name: xp}
                args_m = {"q": q, "k": k, "v": v, name: xm}
                fp = np.sum(attention_ref(args_p["q"], args_p["k"], args_p["v"], causal=causal, scale=scale)[0] * do)
                fm = np.sum(attention_ref(args_m["q"], args_m["k"], args_m["v"], causal=causal, scale=scale)[0] * do)
                num[idx] = (fp - fm) / (2 * h)
            assert np.abs(num - g).max() < 1e-7, (name, causal, np.abs(num - g).max())


def pin_torch_autograd(f):
    for causal in (False, True):
        q, k, v, do = _case(2, 3, 33, 8, seed=20, mult=1.5)
        scale = 0.4
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        o.backward(torch.tensor(do))
        dq, dk, dv = f(q, k, v, do, causal=causal, scale=scale)
        for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            assert np.abs(a - b.numpy()).max() < 1e-10


def pin_constant_v(f):
    # V constant over keys: O does not depend on Q or K, so dQ = dK = 0, and
    # dV_j = sum_i P_ij dO_i.
    q, k, _, do = _case(1, 2, 12, 4, seed=30)
    v = np.broadcast_to(_rand((1, 2, 1, 4), 34), q.shape).copy()
    for causal in (False, True):
        dq, dk, dv = f(q, k, v, do, causal=causal, scale=0.5)
        assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12
        p = oa.attention_probs(q, k, causal=causal, scale=0.5)
        assert np.allclose(dv, np.einsum("bhij,bhid->bhjd", p, do), atol=1e-12)


def pin_single_key(f):
    # One key: P = 1, so dQ = dK = 0 and dV = sum_i dO_i.
    q, k, v, do = _case(1, 2, 1, 6, seed=40)
    dq, dk, dv = f(q, k, v, do, causal=False, scale=0.9)
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0
    assert np.allclose(dv, do, atol=1e-15)
    # causal row 0 sees only key 0: its dQ row is zero
    q, k, v, do = _case(1, 2, 7, 6, seed=41)
    dq, _, _ = f(q, k, v, do, causal=True, scale=0.9)
    assert np.abs(dq[:, :, 0]).max() < 1e-15


def pin_zero_upstream(f):
    q, k, v, _ = _case(1, 2, 8, 4, seed=50)
    dq, dk, dv = f(q, k, v, np.zeros_like(q), causal=True, scale=0.3)
    assert not dq.any() and not dk.any() and not dv.any()


def pin_key_gradients_sum_to_zero(f):
    # Each row of dS sums to zero, so sum_j dK_j = scale * sum_i (sum_j dS_ij) q_i = 0.
    q, k, v, do = _case(2, 2, 17, 5, seed=60, mult=2.0)
    for causal in (False, True):
        _, dk, _ = f(q, k, v, do, causal=causal, scale=0.6)
        assert np.abs(dk.sum(axis=2)).max() < 1e-11


def pin_key_translation(f):
    # Shifting every key by one vector c adds q_i.c to row i of the scores,
    # which softmax ignores; dQ_i = scale * sum_j dS_ij (k_j + c) is unchanged.
    q, k, v, do = _case(1, 2, 11, 4, seed=70)
    c = _rand((1, 2, 1, 4), 75, 3.0)
    for causal in (False, True):
        dq0, dk0, dv0 = f(q, k, v, do, causal=causal, scale=0.5)
        dq1, dk1, dv1 = f(q, k + c, v, do, causal=causal, scale=0.5)
        assert np.abs(dq0 - dq1).max() < 1e-11
        assert np.abs(dk0 - dk1).max() < 1e-11 and np.abs(dv0 - dv1).max() < 1e-11


PINS = [pin_finite_differences, pin_torch_autograd, pin_constant_v, pin_single_key, pin_zero_upstream,
        pin_key_gradients_sum_to_zero, pin_key_translation]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_backward_oracle_pin(pin):
    pin(attention_bwd_ref)


def test_rows_variant_matches_full():
    q, k, v, do = _case(1, 2, 70, 8, seed=80)
    rows = [0, 1, 31, 32, 63, 69]
    for causal in (False, True):
        dq, dk, dv = attention_bwd_ref(q, k, v, do, causal=causal, scale=0.35)
        for b, h in ((0, 0), (0, 1)):
            rq, rk, rv = attention_bwd_ref_rows(q, k, v, do, b, h, rows, causal=causal, scale=0.35, row_block=16)
            assert np.abs(rq - dq[b, h, rows]).max() < 1e-12
            assert np.abs(rk - dk[b, h, rows]).max() < 1e-12
            assert np.abs(rv - dv[b, h, rows]).max() < 1e-12


# ------------------------------------------------------------ planted mistakes

def _bwd_with(bug):
    def bwd(q, k, v, do, causal, scale):
        p = oa._probs_one_head(q, k, causal, scale)
        dv = p.T @ do
        dp = do @ v.T
        delta = np.sum(p * dp, axis=1, keepdims=True)
        if bug == "delta_sign":
            ds = p * (dp + delta)
        elif bug == "no_delta":
            ds = p * dp
        elif bug == "delta_axis":
            ds = p * (dp - np.sum(p * dp, axis=0, keepdims=True))
        else:
            ds = p * (dp - delta)
        dq = scale * (ds @ k)
        dk = scale * (ds.T @ q)
        if bug == "dq_no_scale":
            dq = ds @ k
        if bug == "dk_untransposed":
            dk = scale * (ds @ q)
        if bug == "dv_untransposed":
            dv = p @ do
        if bug == "dp_uses_k":
            dp2 = do @ k.T
            ds = p * (dp2 - np.sum(p * dp2, axis=1, keepdims=True))
            dq, dk = scale * (ds @ k), scale * (ds.T @ q)
        return dq, dk, dv
    return bwd


BUGS = ["delta_sign", "no_delta", "delta_axis", "dq_no_scale", "dk_untransposed", "dv_untransposed", "dp_uses_k"]


@pytest.mark.parametrize("bug", BUGS)
def test_planted_backward_mistake_is_caught(bug, monkeypatch):
    monkeypatch.setattr(oa, "_bwd_one_head", _bwd_with(bug))
    failed = []
    for pin in PINS:
        try:
            pin(oa.attention_bwd_ref)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin catches {bug}"
