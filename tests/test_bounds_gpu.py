"""GPU checks that every kernel writes inside its output buffers and nowhere else.

Each output (O, LSE, dQ, dK, dV) and each workspace is a view into the middle
of a larger byte buffer whose bytes before and after the view hold a fixed
pattern.  After the call the pattern must be intact, and the values inside
the views must equal, bit for bit, those of a call that allocated its own
outputs (the kernels are deterministic; an element the kernels failed to
write would still hold the pattern).  The shapes put rows past N into the
last tile (ragged N, N = 1), columns past d into a tile (d = 32 and 96 run on
64- and 128-column tiles), and cover d = 256 and the split-K/V ranges and
merge.
"""
import pytest
import torch

from exact_tiled_attention_45_b200 import bwd, bwd_workspace_bytes, fwd, fwd_splitkv, splitkv_workspace_bytes, \
    sync_status
from exact_tiled_attention_45_b200.inputs import make_q_kv, make_qkv

from test_bwd_gpu import make_dout

pytestmark = pytest.mark.gpu

PAD_BYTES = 64 * 1024
PATTERN = 0xA5


class Guarded:
    """A view of `nbytes` (as dtype, shape) with PAD_BYTES of pattern on each side."""

    def __init__(self, nbytes, dtype, shape):
        self.nbytes = nbytes
        self.buf = torch.full((PAD_BYTES + nbytes + PAD_BYTES,), PATTERN, dtype=torch.uint8, device="cuda")
        raw = self.buf[PAD_BYTES:PAD_BYTES + nbytes]
        self.view = raw if dtype is torch.uint8 else raw.view(dtype).view(shape)

    def assert_intact(self, name):
        head, tail = self.buf[:PAD_BYTES], self.buf[PAD_BYTES + self.nbytes:]
        bad_head = int((head != PATTERN).sum())
        bad_tail = int((tail != PATTERN).sum())
        assert bad_head == 0 and bad_tail == 0, f"{name}: {bad_head} bytes before and {bad_tail} after were written"


def bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def assert_same_bits(a, b, name):
    assert torch.equal(bits(a), bits(b)), f"{name} differs from the unguarded call"


FWD_CASES = [
    (1, 2, 200, 128, True),
    (1, 2, 200, 128, False),
    (2, 1, 333, 96, True),
    (1, 2, 77, 32, False),
    (1, 2, 300, 256, True),
    (1, 1, 1, 64, False),
    (1, 2, 513, 64, True),
]


@pytest.mark.parametrize("B,H,N,d,causal", FWD_CASES,
                         ids=[f"B{b}H{h}N{n}d{d}{'c' if c else 'f'}" for b, h, n, d, c in FWD_CASES])
def test_fwd_writes_only_its_outputs(B, H, N, d, causal):
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=31))
    o_ref, l_ref = fwd(q, k, v, causal=causal)
    go = Guarded(B * H * N * d * 2, torch.bfloat16, (B, H, N, d))
    gl = Guarded(B * H * N * 4, torch.float32, (B, H, N))
    o, l = fwd(q, k, v, causal=causal, out=go.view, lse=gl.view)
    sync_status()
    go.assert_intact("O")
    gl.assert_intact("LSE")
    assert_same_bits(o, o_ref, "O")
    assert_same_bits(l, l_ref, "LSE")


SKV_CASES = [
    (1, 2, 1, 1000, 128, True, 4),
    (2, 2, 5, 777, 64, True, 3),
    (1, 2, 40, 600, 96, False, 2),
    (1, 1, 1, 300, 256, True, 2),
    (1, 2, 130, 900, 128, True, 0),
    (1, 2, 20, 2000, 32, False, 5),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,n_splits", SKV_CASES,
                         ids=[f"B{b}H{h}Nq{nq}Nk{nk}d{d}{'c' if c else 'f'}s{s}"
                              for b, h, nq, nk, d, c, s in SKV_CASES])
def test_splitkv_writes_only_its_outputs(B, H, Nq, Nk, d, causal, n_splits):
    q, k, v = (t.cuda() for t in make_q_kv(B, H, Nq, Nk, d, seed=32))
    o_ref, l_ref = fwd_splitkv(q, k, v, causal=causal, n_splits=n_splits)
    need = splitkv_workspace_bytes(B, H, Nq, Nk, d, n_splits)
    go = Guarded(B * H * Nq * d * 2, torch.bfloat16, (B, H, Nq, d))
    gl = Guarded(B * H * Nq * 4, torch.float32, (B, H, Nq))
    gw = Guarded(need, torch.uint8, None) if need > 0 else None
    o, l = fwd_splitkv(q, k, v, causal=causal, n_splits=n_splits, out=go.view, lse=gl.view,
                       workspace=gw.view if gw is not None else None)
    sync_status()
    go.assert_intact("O")
    gl.assert_intact("LSE")
    if gw is not None:
        gw.assert_intact("workspace")
    assert_same_bits(o, o_ref, "O")
    assert_same_bits(l, l_ref, "LSE")


BWD_CASES = [
    (1, 2, 200, 128, True),
    (2, 1, 333, 96, False),
    (1, 2, 77, 32, True),
    (1, 2, 300, 256, True),
    (1, 1, 1, 64, False),
    (1, 2, 130, 64, True),
    (1, 1, 129, 256, False),
]


@pytest.mark.parametrize("B,H,N,d,causal", BWD_CASES,
                         ids=[f"B{b}H{h}N{n}d{d}{'c' if c else 'f'}" for b, h, n, d, c in BWD_CASES])
def test_bwd_writes_only_its_outputs(B, H, N, d, causal):
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=33))
    do = make_dout(B, H, N, d, seed=33).cuda()
    o, lse = fwd(q, k, v, causal=causal)
    ref = bwd(q, k, v, o, lse, do, causal=causal)
    nbytes = B * H * N * d * 2
    grads = [Guarded(nbytes, torch.bfloat16, (B, H, N, d)) for _ in range(3)]
    gw = Guarded(bwd_workspace_bytes(B, H, N, d), torch.uint8, None)
    out = bwd(q, k, v, o, lse, do, causal=causal, dq=grads[0].view, dk=grads[1].view, dv=grads[2].view,
              workspace=gw.view)
    sync_status()
    for g, name in zip(grads, ("dQ", "dK", "dV")):
        g.assert_intact(name)
    gw.assert_intact("workspace")
    for a, b, name in zip(out, ref, ("dQ", "dK", "dV")):
        assert_same_bits(a, b, name)
