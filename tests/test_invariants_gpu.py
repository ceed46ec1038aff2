"""GPU checks of properties the exact result must have, and an input that
forces the online softmax's rescale on every key tile.

* Forced rescale.  The kernels keep a running row maximum m (log2 units) and
  rescale the output accumulator only when a key tile raises it by more than
  8.  Here the scores grow linearly with the key position, by 16 log2 units
  per key tile (64 keys at d = 256, 128 otherwise), so every full key tile a
  row sees triggers the rescale; the test first checks that on the inputs
  themselves (in fp64), then compares the kernel element by element with the
  fp64 oracle.  A rescale that was skipped, applied twice or applied with the
  wrong factor leaves the output off by factors of 2^16.
* Affine V: O(alpha V + beta) = alpha O(V) + beta, since each row of P sums to
  one.  V is drawn on a grid on which alpha V + beta is exact in bf16.
* Joint K/V permutation (non-causal): reordering keys and values together
  leaves O and LSE unchanged (up to the rounding of a different summation
  order).
* Causal row i equals non-causal attention over the prefix of length i + 1.

Tolerances are the parity tests' (|dO| <= 1e-2 plus half a bf16 spacing of
the exact value, |dLSE| <= 1e-3) against the oracle; comparisons of two kernel
results allow the sum of both sides' bounds.
"""
import numpy as np
import pytest
import torch

from exact_tiled_attention_45_b200 import fwd, sync_status
from exact_tiled_attention_45_b200.inputs import make_qkv
from oracle import attention_ref

from test_parity_gpu import LSE_TOL, O_TOL, assert_close, bf16_half_spacing

pytestmark = pytest.mark.gpu

RESCALE_THRESHOLD_LOG2 = 8.0
LOG2E = 1.4426950408889634


def tile_keys(d):
    return 64 if d > 128 else 128


def ramp_inputs(B, H, N, d, seed, growth_per_tile=16.0):
    """Q, K, V (bf16, CPU) whose scores rise by ~growth_per_tile log2 units per
    key tile: q_i = A e_0 + noise (noise only off column 0), k_j = r j e_0 +
    noise, V standard normal."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    scale = d ** -0.5
    A = 8.0
    r = growth_per_tile / (A * tile_keys(d) * scale * LOG2E)
    q = 0.5 * torch.randn(B, H, N, d, generator=g)
    k = 0.5 * torch.randn(B, H, N, d, generator=g)
    v = torch.randn(B, H, N, d, generator=g)
    q[..., 0] = A
    k[..., 0] = r * torch.arange(N, dtype=torch.float32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def assert_rescale_forced_on_every_full_tile(q, k, causal):
    """Per row, in fp64: each key tile's max of scale*log2(e)*s over the keys
    the row may see exceeds the maximum over all earlier tiles by more than
    the threshold, for every tile but a causal row's last (partial) one."""
    d, N = q.shape[-1], q.shape[2]
    T = tile_keys(d)
    c = d ** -0.5 * LOG2E
    qn, kn = q.double().numpy(), k.double().numpy()
    s = c * np.einsum("bhid,bhjd->bhij", qn, kn)
    n_tiles = (N + T - 1) // T
    checked = 0
    for i in range(N):
        visible = i + 1 if causal else N
        full = visible // T if causal else n_tiles  # a causal row's diagonal tile may hold few keys
        run = s[:, :, i, 0:min(T, visible)].max(axis=-1)
        for t in range(1, full):
            tmax = s[:, :, i, t * T:min((t + 1) * T, visible)].max(axis=-1)
            assert (tmax > run + RESCALE_THRESHOLD_LOG2).all(), (i, t)
            run = np.maximum(run, tmax)
            checked += 1
    assert checked > 0


@pytest.mark.parametrize("d", [32, 64, 96, 128, 256])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("N", [1024, 1000])
def test_rescale_forced_on_every_key_tile(d, causal, N):
    q, k, v = ramp_inputs(1, 2, N, d, seed=20 + d)
    assert_rescale_forced_on_every_full_tile(q, k, causal)
    o, lse = fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    sync_status()
    o_ref, lse_ref = attention_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                                   scale=d ** -0.5)
    assert_close(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref,
                 f"forced rescale d={d} N={N} causal={causal}")


def grid_v(shape, seed):
    """V on multiples of 1/16 in [-3.9375, 3.9375]: 2 V + 0.5 stays exact in bf16."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    v = torch.round(16 * torch.randn(shape, generator=g).clamp(-3.9, 3.9)) / 16
    return v.to(torch.bfloat16)


@pytest.mark.parametrize("d,causal", [(64, False), (128, True), (256, False), (96, True)])
def test_affine_v(d, causal):
    alpha, beta = 2.0, 0.5
    q, k, _ = make_qkv(2, 2, 700, d, seed=21)
    v = grid_v(q.shape, 22)
    v2 = (alpha * v.float() + beta).to(torch.bfloat16)
    assert torch.equal(v2.float(), alpha * v.float() + beta)  # exact on the grid
    qd, kd = q.cuda(), k.cuda()
    o1, l1 = fwd(qd, kd, v.cuda(), causal=causal)
    o2, l2 = fwd(qd, kd, v2.cuda(), causal=causal)
    sync_status()
    o1, o2 = o1.double().cpu().numpy(), o2.double().cpu().numpy()
    # LSE does not depend on V at all
    assert np.array_equal(l1.cpu().numpy(), l2.cpu().numpy())
    # the kernel on the transformed V against the oracle ...
    o_ref, lse_ref = attention_ref(q.double().numpy(), k.double().numpy(), v2.double().numpy(), causal=causal,
                                   scale=d ** -0.5)
    assert_close(o2, l2.double().cpu().numpy(), o_ref, lse_ref, f"affine V d={d}")
    # ... and against the transformed kernel output on V
    pred = alpha * o1 + beta
    bound = (1 + alpha) * O_TOL + alpha * bf16_half_spacing(o1) + bf16_half_spacing(pred)
    assert (np.abs(o2 - pred) <= bound).all(), np.abs(o2 - pred).max()


@pytest.mark.parametrize("d,N", [(64, 1000), (128, 777), (256, 300), (32, 513)])
def test_joint_kv_permutation_non_causal(d, N):
    q, k, v = make_qkv(1, 3, N, d, seed=23, qk_mult=2.0)
    perm = torch.from_numpy(np.random.default_rng(24).permutation(N))
    kp, vp = k[:, :, perm].contiguous(), v[:, :, perm].contiguous()
    qd = q.cuda()
    o1, l1 = fwd(qd, k.cuda(), v.cuda(), causal=False)
    o2, l2 = fwd(qd, kp.cuda(), vp.cuda(), causal=False)
    sync_status()
    o1, o2 = o1.double().cpu().numpy(), o2.double().cpu().numpy()
    l1, l2 = l1.double().cpu().numpy(), l2.double().cpu().numpy()
    o_ref, lse_ref = attention_ref(q.double().numpy(), kp.double().numpy(), vp.double().numpy(), causal=False,
                                   scale=d ** -0.5)
    assert_close(o2, l2, o_ref, lse_ref, f"permuted keys d={d}")
    assert (np.abs(o1 - o2) <= 2 * (O_TOL + bf16_half_spacing(o_ref))).all()
    assert np.abs(l1 - l2).max() <= 2 * LSE_TOL


@pytest.mark.parametrize("d", [64, 128, 256])
def test_causal_row_equals_attention_over_its_prefix(d):
    N = 520
    q, k, v = make_qkv(1, 2, N, d, seed=25)
    oc, lc = fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    sync_status()
    oc, lc = oc.double().cpu().numpy(), lc.double().cpu().numpy()
    for i in (0, 63, 64, 127, 128, 129, 255, 256, 300, 511, 519):
        qs, ks, vs = (t[:, :, :i + 1].contiguous() for t in (q, k, v))
        of, lf = fwd(qs.cuda(), ks.cuda(), vs.cuda(), causal=False)
        sync_status()
        of, lf = of.double().cpu().numpy(), lf.double().cpu().numpy()
        # row i of the causal run against the last row of the prefix run
        assert (np.abs(oc[:, :, i] - of[:, :, i]) <= 2 * O_TOL + 2 * bf16_half_spacing(of[:, :, i])).all(), i
        assert np.abs(lc[:, :, i] - lf[:, :, i]).max() <= 2 * LSE_TOL, i
