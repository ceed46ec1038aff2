"""Pins for the fp64 CPU oracle (no GPU).

The oracle is checked against things other than itself: hand-computed
fixtures, closed forms, invariants the mathematics fixes, a library routine
the problem reduces to (torch's float64 scaled-dot-product attention), brute
force on tiny inputs, and a mutation test showing that each plausible mistake
planted in the oracle fails at least one pin.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle.attention as oa
from oracle import attention_ref, attention_ref_rows, attention_probs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_fixture(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rhs = line.split("=", 1)
            vals[key.strip()] = [float(x) for x in rhs.split()]
    B, H, N, d = (int(x) for x in vals["shape"])
    out = {"shape": (B, H, N, d), "scale": vals["scale"][0]}
    for key in ("q", "k", "v"):
        out[key] = np.array(vals[key]).reshape(B, H, N, d)
    for key in ("o_full", "o_causal"):
        if key in vals:
            out[key] = np.array(vals[key]).reshape(B, H, N, d)
    for key in ("lse_full", "lse_causal"):
        if key in vals:
            out[key] = np.array(vals[key]).reshape(B, H, N)
    return out


FIXTURES = ["two_keys_d1.txt", "three_keys_d2.txt", "causal_zero_q_d1.txt"]


def _rand(shape, seed, mult=1.0):
    r = np.random.default_rng(seed)
    return r.standard_normal(shape) * mult


# --------------------------------------------------------------------------
# Pins, written as checks on any attention function f(q, k, v, causal, scale)
# -> (O, LSE).  Each returns None when it holds, or a short failure message.
# --------------------------------------------------------------------------

def pin_golden(f):
    for name in FIXTURES:
        fx = _read_fixture(name)
        for causal, ok, lk in ((False, "o_full", "lse_full"), (True, "o_causal", "lse_causal")):
            if ok not in fx:
                continue
            o, lse = f(fx["q"], fx["k"], fx["v"], causal, fx["scale"])
            if not np.allclose(o, fx[ok], rtol=0, atol=1e-12):
                return f"{name} causal={causal}: O {o.ravel()} != {fx[ok].ravel()}"
            if not np.allclose(lse, fx[lk], rtol=0, atol=1e-12):
                return f"{name} causal={causal}: LSE {lse.ravel()} != {fx[lk].ravel()}"
    return None


def pin_single_key(f):
    # N = 1: the only key gets probability 1, O = v_0 and LSE = scale * q.k.
    q, k, v = _rand((2, 3, 1, 8), 1), _rand((2, 3, 1, 8), 2), _rand((2, 3, 1, 8), 3)
    for causal in (False, True):
        o, lse = f(q, k, v, causal, 0.37)
        if not np.allclose(o, v, atol=1e-12):
            return "N=1: O != V"
        if not np.allclose(lse, 0.37 * np.sum(q * k, axis=-1), atol=1e-12):
            return "N=1: LSE != scale*q.k"
    return None


def pin_zero_query(f):
    # q = 0: every allowed score is 0, P is uniform, O is the mean of the
    # allowed values and LSE = ln(#allowed keys).
    N, d = 9, 4
    q = np.zeros((1, 2, N, d))
    k, v = _rand((1, 2, N, d), 4), _rand((1, 2, N, d), 5)
    o, lse = f(q, k, v, False, 0.8)
    if not np.allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), atol=1e-12):
        return "q=0 non-causal: O != mean(V)"
    if not np.allclose(lse, math.log(N), atol=1e-12):
        return "q=0 non-causal: LSE != ln N"
    o, lse = f(q, k, v, True, 0.8)
    prefix_mean = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    if not np.allclose(o, prefix_mean, atol=1e-12):
        return "q=0 causal: O != prefix mean(V)"
    if not np.allclose(lse, np.log(np.arange(1, N + 1))[None, None, :], atol=1e-12):
        return "q=0 causal: LSE != ln(i+1)"
    return None


def pin_constant_v(f):
    q, k = _rand((1, 2, 17, 8), 6, 3.0), _rand((1, 2, 17, 8), 7, 3.0)
    v = np.full((1, 2, 17, 8), -1.25)
    for causal in (False, True):
        o, _ = f(q, k, v, causal, 0.5)
        if not np.allclose(o, -1.25, atol=1e-12):
            return f"constant V causal={causal}: O not constant"
    return None


def pin_causal_row0(f):
    q, k, v = _rand((2, 2, 13, 8), 8), _rand((2, 2, 13, 8), 9), _rand((2, 2, 13, 8), 10)
    o, lse = f(q, k, v, True, 0.35)
    if not np.array_equal(o[:, :, 0], v[:, :, 0]):
        return "causal row 0 != V[0] exactly"
    if not np.allclose(lse[:, :, 0], 0.35 * np.sum(q[:, :, 0] * k[:, :, 0], axis=-1), atol=1e-12):
        return "causal row 0 LSE != scale q0.k0"
    return None


def pin_causal_prefix(f):
    # Causal row i equals non-causal attention over the prefix 0..i.
    q, k, v = _rand((1, 1, 12, 8), 11), _rand((1, 1, 12, 8), 12), _rand((1, 1, 12, 8), 13)
    oc, lc = f(q, k, v, True, 0.4)
    for i in (1, 5, 11):
        on, ln = f(q[:, :, : i + 1], k[:, :, : i + 1], v[:, :, : i + 1], False, 0.4)
        if not np.allclose(oc[:, :, i], on[:, :, i], atol=1e-12):
            return f"causal row {i} != prefix attention"
        if not np.allclose(lc[:, :, i], ln[:, :, i], atol=1e-12):
            return f"causal LSE row {i} != prefix LSE"
    return None


def pin_affine_v(f):
    q, k, v = _rand((1, 2, 10, 8), 14), _rand((1, 2, 10, 8), 15), _rand((1, 2, 10, 8), 16)
    for causal in (False, True):
        o, lse = f(q, k, v, causal, 0.3)
        o2, lse2 = f(q, k, 2.5 * v - 0.75, causal, 0.3)
        if not np.allclose(o2, 2.5 * o - 0.75, atol=1e-12):
            return f"affine V causal={causal}"
        if not np.allclose(lse2, lse, atol=1e-12):
            return f"LSE depends on V causal={causal}"
    return None


def pin_permutation(f):
    q, k, v = _rand((1, 2, 11, 8), 17), _rand((1, 2, 11, 8), 18), _rand((1, 2, 11, 8), 19)
    perm = np.random.default_rng(20).permutation(11)
    o, lse = f(q, k, v, False, 0.3)
    o2, lse2 = f(q, k[:, :, perm], v[:, :, perm], False, 0.3)
    if not (np.allclose(o, o2, atol=1e-12) and np.allclose(lse, lse2, atol=1e-12)):
        return "non-causal result changes under a joint K/V row permutation"
    return None


def pin_score_shift(f):
    # An extra feature with q_extra = t and k_extra = 1 adds scale*t to every
    # score: O unchanged, LSE shifted by scale*t.
    q, k, v = _rand((1, 2, 10, 8), 21), _rand((1, 2, 10, 8), 22), _rand((1, 2, 10, 8), 23)
    t, scale = 3.0, 0.3
    qx = np.concatenate([q, np.full((1, 2, 10, 1), t)], axis=-1)
    kx = np.concatenate([k, np.ones((1, 2, 10, 1))], axis=-1)
    vx = np.concatenate([v, np.zeros((1, 2, 10, 1))], axis=-1)
    for causal in (False, True):
        o, lse = f(q, k, v, causal, scale)
        o2, lse2 = f(qx, kx, vx, causal, scale)
        if not np.allclose(o2[..., :8], o, atol=1e-12):
            return f"score shift changed O causal={causal}"
        if not np.allclose(lse2, lse + scale * t, atol=1e-12):
            return f"score shift: LSE not shifted by scale*t causal={causal}"
    return None


def pin_sdpa(f):
    # Library special case: torch's float64 CPU scaled_dot_product_attention
    # (O) and torch.logsumexp of the masked scaled scores (LSE).
    for causal, (N, d, scale, mult) in [(False, (33, 16, 0.25, 1.0)), (True, (33, 16, 0.25, 1.0)),
                                         (False, (40, 8, 0.5, 4.0)), (True, (40, 8, 0.5, 4.0))]:
        q, k, v = _rand((2, 3, N, d), 24, mult), _rand((2, 3, N, d), 25, mult), _rand((2, 3, N, d), 26)
        o, lse = f(q, k, v, causal, scale)
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
        o_t = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        s = scale * (tq @ tk.transpose(-1, -2))
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        lse_t = torch.logsumexp(s, dim=-1)
        if not np.allclose(o, o_t.numpy(), atol=1e-10, rtol=0):
            return f"O != torch SDPA (causal={causal}, x{mult})"
        if not np.allclose(lse, lse_t.numpy(), atol=1e-10, rtol=0):
            return f"LSE != torch.logsumexp (causal={causal}, x{mult})"
    return None


def pin_brute_force(f):
    # Tiny inputs, element by element with math.exp / math.fsum.
    B, H, N, d = 1, 2, 5, 3
    q, k, v = _rand((B, H, N, d), 27), _rand((B, H, N, d), 28), _rand((B, H, N, d), 29)
    scale = 0.7
    for causal in (False, True):
        o, lse = f(q, k, v, causal, scale)
        for b in range(B):
            for h in range(H):
                for i in range(N):
                    keys = range(i + 1) if causal else range(N)
                    s = [scale * math.fsum(q[b, h, i, c] * k[b, h, j, c] for c in range(d)) for j in keys]
                    w = [math.exp(x) for x in s]
                    tot = math.fsum(w)
                    if abs(lse[b, h, i] - math.log(tot)) > 1e-12:
                        return f"brute force LSE mismatch causal={causal}"
                    for c in range(d):
                        oc = math.fsum(w[jj] * v[b, h, j, c] for jj, j in enumerate(keys)) / tot
                        if abs(o[b, h, i, c] - oc) > 1e-12:
                            return f"brute force O mismatch causal={causal}"
    return None


def pin_large_logits(f):
    # Q, K x16 (logit std ~ 180 at d=8): exact result still finite, O a convex
    # combination of the values, LSE between the row max and max + ln(#keys).
    q, k, v = _rand((1, 2, 64, 8), 30, 16.0), _rand((1, 2, 64, 8), 31, 16.0), _rand((1, 2, 64, 8), 32)
    for causal in (False, True):
        o, lse = f(q, k, v, causal, 1 / math.sqrt(8))
        if not (np.all(np.isfinite(o)) and np.all(np.isfinite(lse))):
            return f"large logits: non-finite output causal={causal}"
        s = (q @ np.swapaxes(k, -1, -2)) / math.sqrt(8)
        if causal:
            s = np.where(np.tri(64, dtype=bool), s, -np.inf)
        m = s.max(axis=-1)
        cnt = np.isfinite(s).sum(axis=-1)
        if np.any(lse < m - 1e-9) or np.any(lse > m + np.log(cnt) + 1e-9):
            return f"large logits: LSE outside [max, max+ln n] causal={causal}"
        if np.any(o > v.max(axis=2, keepdims=True) + 1e-9) or np.any(o < v.min(axis=2, keepdims=True) - 1e-9):
            return f"large logits: O outside the value hull causal={causal}"
    return None


PINS = [pin_golden, pin_single_key, pin_zero_query, pin_constant_v, pin_causal_row0,
        pin_causal_prefix, pin_affine_v, pin_permutation, pin_score_shift, pin_sdpa,
        pin_brute_force, pin_large_logits]


def pin_failures(f):
    out = []
    for pin in PINS:
        try:
            msg = pin(f)
        except Exception as e:  # a crash is a failure too
            msg = f"raised {type(e).__name__}: {e}"
        if msg:
            out.append(f"{pin.__name__}: {msg}")
    return out


def _oracle(q, k, v, causal, scale):
    return attention_ref(q, k, v, causal=causal, scale=scale)


# --------------------------------------------------------------------------
# The oracle against its pins
# --------------------------------------------------------------------------

@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    assert pin(_oracle) is None


def test_rows_of_p_sum_to_one():
    q, k = _rand((1, 2, 20, 8), 40, 4.0), _rand((1, 2, 20, 8), 41, 4.0)
    for causal in (False, True):
        p = attention_probs(q, k, causal=causal, scale=0.5)
        assert np.allclose(p.sum(-1), 1.0, atol=1e-12)
        assert np.all(p >= 0)
        if causal:
            assert np.all(p[..., np.triu_indices(20, 1)[0], np.triu_indices(20, 1)[1]] == 0)


def test_rows_sample_matches_full():
    q, k, v = _rand((2, 2, 50, 8), 42), _rand((2, 2, 50, 8), 43), _rand((2, 2, 50, 8), 44)
    for causal in (False, True):
        o, lse = attention_ref(q, k, v, causal=causal, scale=0.3)
        rows = [0, 7, 49]
        o_r, l_r = attention_ref_rows(q, k, v, 1, 0, rows, causal=causal, scale=0.3)
        assert np.allclose(o_r, o[1, 0, rows], atol=1e-13)
        assert np.allclose(l_r, lse[1, 0, rows], atol=1e-13)


def test_row_block_does_not_change_values():
    q, k, v = _rand((1, 1, 70, 8), 45), _rand((1, 1, 70, 8), 46), _rand((1, 1, 70, 8), 47)
    a = attention_ref(q, k, v, causal=True, scale=0.3)
    b = attention_ref(q, k, v, causal=True, scale=0.3, row_block=16)
    assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-14)


def test_default_scale_is_inverse_sqrt_d():
    q, k, v = _rand((1, 1, 6, 16), 48), _rand((1, 1, 6, 16), 49), _rand((1, 1, 6, 16), 50)
    a = attention_ref(q, k, v)
    b = attention_ref(q, k, v, scale=0.25)
    assert np.allclose(a[0], b[0]) and np.allclose(a[1], b[1])


def test_bf16_inputs_taken_exactly():
    from exact_tiled_attention_45_b200.inputs import make_qkv
    q, k, v = make_qkv(1, 2, 16, 8, seed=0)
    o, lse = attention_ref(q.float().numpy(), k.float().numpy(), v.float().numpy())
    o2, lse2 = attention_ref(q.double().numpy(), k.double().numpy(), v.double().numpy())
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


# --------------------------------------------------------------------------
# Mutation test: plausible mistakes planted in the oracle fail a pin
# --------------------------------------------------------------------------

def _flipped_mask(rows, n_keys, causal, offset=0):
    j = np.arange(n_keys)[None, :]
    return (j >= rows[:, None] + offset) if causal else np.ones((rows.shape[0], n_keys), bool)


def _strict_mask(rows, n_keys, causal, offset=0):
    j = np.arange(n_keys)[None, :]
    return (j < rows[:, None] + offset) if causal else np.ones((rows.shape[0], n_keys), bool)


def _make_rows(bug, block=4):
    """A copy of the oracle's per-head kernel with one planted mistake."""

    def rows_fn(q_rows, k, v, rows, causal, scale):
        s = scale * (q_rows @ k.T)
        if bug == "transpose_s":
            if q_rows.shape[0] != k.shape[0]:
                raise ValueError("transposed scores need a square block")
            s = scale * (k @ q_rows.T)
        if bug == "no_scale":
            s = q_rows @ k.T
        if bug == "sign":
            s = -s
        if bug == "kv_swap":
            v = k
        allowed = oa._allowed_mask(rows, k.shape[0], causal)
        s = np.where(allowed, s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        if bug == "no_max_sub":
            m = np.zeros_like(m)
        e = np.exp(s - m)
        if bug == "col_norm":
            l = np.sum(e, axis=0, keepdims=True)
            p = e / l
            lse = m[:, 0] + np.log(np.sum(e, axis=1))
        elif bug == "block_norm":
            # per-block normalisation, added up (what the tiled method must
            # not do: each block of keys normalised on its own)
            p = np.zeros_like(e)
            for j0 in range(0, e.shape[1], block):
                blk = e[:, j0:j0 + block]
                tot = blk.sum(axis=1, keepdims=True)
                p[:, j0:j0 + block] = np.where(tot > 0, blk / np.where(tot > 0, tot, 1), 0)
            lse = m[:, 0] + np.log(np.sum(e, axis=1))
        else:
            l = np.sum(e, axis=1, keepdims=True)
            p = e / l
            lse = m[:, 0] + np.log(l[:, 0])
            if bug == "lse_no_max":
                lse = np.log(l[:, 0])
            if bug == "lse_log2":
                lse = lse / math.log(2)
        o = p @ v
        return o, lse

    return rows_fn


ARITH_BUGS = ["no_scale", "sign", "kv_swap", "no_max_sub", "col_norm", "block_norm",
              "lse_no_max", "lse_log2", "transpose_s"]


@pytest.mark.parametrize("bug", ARITH_BUGS)
def test_planted_arithmetic_mistake_is_caught(bug, monkeypatch):
    monkeypatch.setattr(oa, "_rows_one_head", _make_rows(bug))
    assert pin_failures(_oracle), f"mutant {bug} passed every pin"


@pytest.mark.parametrize("mask", [_flipped_mask, _strict_mask], ids=["flipped", "strict"])
def test_planted_mask_mistake_is_caught(mask, monkeypatch):
    monkeypatch.setattr(oa, "_allowed_mask", mask)
    with np.errstate(all="ignore"):
        assert pin_failures(_oracle), "mask mutant passed every pin"


def test_negative_control_block_normalisation_fails_tolerance():
    # The tiled method must reach the global softmax; normalising each key
    # block on its own (iplexlaw blog, "Tiling preserves the attention
    # calculation") is wrong, and the parity tolerance is tight enough to see
    # it on the tiny workload (B1 H2 N128 d64).
    from exact_tiled_attention_45_b200.inputs import make_qkv
    q, k, v = (t.double().numpy() for t in make_qkv(1, 2, 128, 64, seed=0))
    o, lse = attention_ref(q, k, v, causal=False, scale=1 / 8)
    orig = oa._rows_one_head
    try:
        oa._rows_one_head = _make_rows("block_norm", block=64)
        o_bad, _ = attention_ref(q, k, v, causal=False, scale=1 / 8)
    finally:
        oa._rows_one_head = orig
    assert np.max(np.abs(o_bad - o)) > 1e-2
