"""Pins for the oracle's rectangular form (Nq query rows against Nk >= Nq
keys; query row i is sequence position Nk - Nq + i), used by the split-K/V
decode path.  No GPU."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as oa
from oracle import attention_ref, attention_ref_rect


def _rand(shape, seed, mult=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * mult


@pytest.mark.parametrize("causal", [False, True])
def test_square_case_is_the_square_oracle(causal):
    q, k, v = _rand((2, 2, 37, 8), 1), _rand((2, 2, 37, 8), 2), _rand((2, 2, 37, 8), 3)
    a = attention_ref_rect(q, k, v, causal=causal, scale=0.3)
    b = attention_ref(q, k, v, causal=causal, scale=0.3)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("nq", [1, 5, 40])
def test_last_rows_of_a_causal_sequence(nq):
    # Decoding the last nq positions equals the last nq rows of full causal
    # attention over the whole sequence (the same queries at those positions).
    N = 40
    q, k, v = _rand((1, 3, N, 8), 4), _rand((1, 3, N, 8), 5), _rand((1, 3, N, 8), 6)
    full_o, full_l = attention_ref(q, k, v, causal=True, scale=0.35)
    o, l = attention_ref_rect(q[:, :, N - nq:], k, v, causal=True, scale=0.35)
    assert np.allclose(o, full_o[:, :, N - nq:], atol=1e-13)
    assert np.allclose(l, full_l[:, :, N - nq:], atol=1e-13)


def test_single_query_sees_every_key_even_when_causal():
    q, k, v = _rand((1, 2, 1, 16), 7), _rand((1, 2, 50, 16), 8), _rand((1, 2, 50, 16), 9)
    a = attention_ref_rect(q, k, v, causal=True, scale=0.25)
    b = attention_ref_rect(q, k, v, causal=False, scale=0.25)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_zero_query_rectangular_closed_form():
    # q = 0: O_i is the mean of the values at keys 0..Nk-Nq+i, LSE_i = ln(count).
    Nq, Nk = 3, 10
    q = np.zeros((1, 1, Nq, 4))
    k, v = _rand((1, 1, Nk, 4), 10), _rand((1, 1, Nk, 4), 11)
    o, l = attention_ref_rect(q, k, v, causal=True, scale=1.0)
    for i in range(Nq):
        cnt = Nk - Nq + i + 1
        assert np.allclose(o[0, 0, i], v[0, 0, :cnt].mean(axis=0), atol=1e-13)
        assert abs(l[0, 0, i] - math.log(cnt)) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_rectangular_against_torch_sdpa_with_explicit_mask(causal):
    Nq, Nk, d, scale = 7, 29, 16, 0.2
    q, k, v = _rand((2, 2, Nq, d), 12, 3.0), _rand((2, 2, Nk, d), 13, 3.0), _rand((2, 2, Nk, d), 14)
    o, l = attention_ref_rect(q, k, v, causal=causal, scale=scale)
    mask = torch.ones(Nq, Nk, dtype=torch.bool)
    if causal:
        mask = torch.arange(Nk)[None, :] <= (Nk - Nq + torch.arange(Nq))[:, None]
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    o_t = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    s = (scale * (tq @ tk.transpose(-1, -2))).masked_fill(~mask, float("-inf"))
    assert np.allclose(o, o_t.numpy(), atol=1e-10)
    assert np.allclose(l, torch.logsumexp(s, dim=-1).numpy(), atol=1e-10)


def test_rejects_more_queries_than_keys():
    with pytest.raises(ValueError):
        attention_ref_rect(np.zeros((1, 1, 5, 4)), np.zeros((1, 1, 4, 4)), np.zeros((1, 1, 4, 4)))


def test_planted_offset_mistake_is_caught(monkeypatch):
    # A top-left-aligned causal mask (the offset dropped) must fail the
    # decode-prefix pin above.
    orig = oa._allowed_mask
    monkeypatch.setattr(oa, "_allowed_mask", lambda rows, n, causal, offset=0: orig(rows, n, causal, 0))
    with pytest.raises(AssertionError):
        test_last_rows_of_a_causal_sequence(5)
