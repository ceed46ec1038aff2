"""GPU parity of the backward (dQ, dK, dV) against the fp64 oracle.

The kernels take O and LSE from the forward kernel (as a training step
would) and dO drawn like the inputs.  Tolerance, per gradient tensor G (the
pages give none for gradients; derived from the arithmetic): the kernel
rounds P and dS to bf16 before the tensor-core products (relative error
2^-9 each), reads D = rowsum(dO o O) from the bf16 forward output (2^-9),
accumulates in fp32 and rounds the result to bf16 (2^-9).  Every element is
a sum of such terms, so its error is bounded relative to the magnitude of
the tensor's entries rather than its own (dS = P (dP - D) cancels):
    max |dG| <= 2^-6 * max |G|   and   ||dG|| / ||G|| <= 2^-7.
"""
import numpy as np
import pytest
import torch

from exact_tiled_attention_45_b200 import bwd, fwd, sync_status
from exact_tiled_attention_45_b200.inputs import make_qkv
from oracle import attention_bwd_ref

pytestmark = pytest.mark.gpu

MAX_TOL = 2.0 ** -6
FRO_TOL = 2.0 ** -7


def make_dout(B, H, N, d, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 + seed)
    return torch.randn(B, H, N, d, generator=g, dtype=torch.float32).to(torch.bfloat16)


def run(q, k, v, do, causal, scale=None):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = bwd(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    sync_status()
    return [t.double().cpu().numpy() for t in (dq, dk, dv)]


def check(got, ref, what):
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        assert np.isfinite(g).all(), f"{what} {name}: non-finite"
        err = np.abs(g - r)
        scale = np.abs(r).max()
        fro = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
        assert err.max() <= MAX_TOL * scale + 1e-6, (f"{what} {name}: max |d| {err.max():.3e} > "
                                                     f"{MAX_TOL:.3e} * {scale:.3e}; rel fro {fro:.3e}")
        # Relative to ||G||, with the max check's absolute 1e-6 per element
        # (a gradient can be exactly zero: one key gives dS = dP - D = 0).
        assert np.linalg.norm(g - r) <= FRO_TOL * np.linalg.norm(r) + 1e-6 * np.sqrt(r.size), (
            f"{what} {name}: relative Frobenius error {fro:.3e}")


CASES = [
    # (B, H, N, d, causal, mult)
    (1, 2, 128, 64, False, 1.0),
    (1, 2, 128, 64, True, 1.0),
    (2, 2, 256, 128, False, 1.0),
    (2, 2, 256, 128, True, 1.0),
    (1, 2, 640, 128, True, 1.0),
    (1, 3, 512, 64, False, 1.0),
    # ragged sequence lengths
    (1, 1, 1, 128, False, 1.0),
    (1, 1, 1, 64, True, 1.0),
    (1, 2, 130, 64, True, 1.0),
    (1, 2, 300, 128, False, 1.0),
    (2, 1, 1000, 64, True, 1.0),
    (1, 2, 777, 128, True, 1.0),
    # large logits
    (1, 2, 512, 128, True, 4.0),
    (1, 2, 384, 64, False, 4.0),
    # zero-padded head dims
    (1, 2, 256, 32, False, 1.0),
    (1, 2, 130, 32, True, 1.0),
    (1, 2, 300, 96, True, 1.0),
    (2, 1, 256, 96, False, 1.0),
    # d = 256: 64-key tiles in the dQ kernel, dV and dK passes over 64-query tiles
    (1, 2, 256, 256, False, 1.0),
    (1, 2, 256, 256, True, 1.0),
    (2, 1, 129, 256, True, 1.0),
    (1, 1, 1, 256, False, 1.0),
    (1, 2, 333, 256, False, 1.0),
    (1, 2, 700, 256, True, 1.0),
    (1, 2, 384, 256, True, 4.0),
]


@pytest.mark.parametrize("B,H,N,d,causal,mult", CASES,
                         ids=[f"B{b}H{h}N{n}d{d}{'c' if c else 'f'}x{int(m)}" for b, h, n, d, c, m in CASES])
def test_bwd_elementwise(B, H, N, d, causal, mult):
    q, k, v = make_qkv(B, H, N, d, seed=21, qk_mult=mult)
    do = make_dout(B, H, N, d, 21)
    got = run(q, k, v, do, causal)
    ref = attention_bwd_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                            causal=causal, scale=d ** -0.5)
    check(got, ref, f"B{B}H{H}N{N}d{d} causal={causal} x{mult}")


def test_bwd_non_default_scale():
    q, k, v = make_qkv(1, 2, 333, 128, seed=22)
    do = make_dout(1, 2, 333, 128, 22)
    got = run(q, k, v, do, True, scale=0.05)
    ref = attention_bwd_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                            causal=True, scale=0.05)
    check(got, ref, "scale 0.05")


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_full_size_sampled_heads(causal):
    # The benchmark shape B=8, H=16, N=2048, d=128; whole heads checked.
    B, H, N, d = 8, 16, 2048, 128
    q, k, v = make_qkv(B, H, N, d, seed=0)
    do = make_dout(B, H, N, d, 0)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fwd(qd, kd, vd, causal=causal)
    dq, dk, dv = bwd(qd, kd, vd, o, lse, dod, causal=causal)
    sync_status()
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all().item()
    rng = np.random.default_rng(3)
    heads = {(0, 0), (B - 1, H - 1), (int(rng.integers(B)), int(rng.integers(H)))}
    for b, h in sorted(heads):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = attention_bwd_ref(q[sl].double().numpy(), k[sl].double().numpy(), v[sl].double().numpy(),
                                do[sl].double().numpy(), causal=causal, scale=d ** -0.5)
        got = [t[sl].double().cpu().numpy() for t in (dq, dk, dv)]
        check(got, ref, f"head ({b},{h}) causal={causal}")


def test_bwd_d256_full_size_sampled_heads():
    # A long d = 256 sequence (B=1, H=8, N=4096, causal): whole heads checked.
    B, H, N, d = 1, 8, 4096, 256
    q, k, v = make_qkv(B, H, N, d, seed=5)
    do = make_dout(B, H, N, d, 5)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fwd(qd, kd, vd, causal=True)
    dq, dk, dv = bwd(qd, kd, vd, o, lse, dod, causal=True)
    sync_status()
    for h in (0, H - 1):
        sl = (slice(0, 1), slice(h, h + 1))
        ref = attention_bwd_ref(q[sl].double().numpy(), k[sl].double().numpy(), v[sl].double().numpy(),
                                do[sl].double().numpy(), causal=True, scale=d ** -0.5)
        got = [t[sl].double().cpu().numpy() for t in (dq, dk, dv)]
        check(got, ref, f"d256 head {h}")


def test_bwd_repeatable_bitwise():
    q, k, v = (t.cuda() for t in make_qkv(2, 2, 700, 128, seed=23))
    do = make_dout(2, 2, 700, 128, 23).cuda()
    o, lse = fwd(q, k, v, causal=True)
    a = bwd(q, k, v, o, lse, do, causal=True)
    b = bwd(q, k, v, o, lse, do, causal=True)
    sync_status()
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def test_bwd_constant_v_gives_zero_dq_dk():
    # V constant over keys: O does not depend on Q or K (oracle pin); the
    # kernel's dQ and dK must vanish up to the rounding of D.
    q, k, _ = make_qkv(1, 2, 384, 64, seed=24)
    v = torch.full_like(q, 0.5)
    do = make_dout(1, 2, 384, 64, 24)
    for causal in (False, True):
        dq, dk, _ = run(q, k, v, do, causal)
        assert np.abs(dq).max() < 2e-3 and np.abs(dk).max() < 2e-3
