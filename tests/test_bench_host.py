"""Host-side pieces of bench.py that need no GPU: the sweep's points and the
input equivalence that lets the sweep draw once per head dimension."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from exact_tiled_attention_45_b200.inputs import WORKLOADS, make_qkv  # noqa: E402


def test_grid_covers_the_16k_token_sweep():
    pts = bench.grid_points()
    names = [p[0] for p in pts]
    assert len(names) == len(set(names)) == 30
    for name, B, H, N, d, causal, mult in pts:
        assert B * N == 16384 and H * d == 2048
        if mult == 1.0:
            w = WORKLOADS[name]
            assert (w.B, w.H, w.N, w.d, w.causal) == (B, H, N, d, causal)
    x1 = {(N, d, c) for _, _, _, N, d, c, m in pts if m == 1.0}
    assert x1 == {(N, d, c) for N in (512, 1024, 2048, 4096, 8192, 16384) for d in (64, 128) for c in (False, True)}
    # the headline shape is one of the points
    assert "grid_N2048_d128_causal" in names


def test_one_draw_per_head_dim_equals_the_per_shape_draw():
    # make_qkv fills [B, H, N, d] from one flat sequence of the generator, so
    # equal element counts give equal data whatever the shape.
    for B, H, N, d in ((4, 3, 16, 8), (1, 6, 64, 8), (16, 2, 12, 4)):
        flat = make_qkv(1, 1, B * H * N, d, seed=0)
        shaped = make_qkv(B, H, N, d, seed=0)
        for a, b in zip(flat, shaped):
            assert torch.equal(a.view(B, H, N, d), b)


def test_tensor_pipe_record_is_keyed_by_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "tensor_pipe.txt").write_text("# header\nabc grid_N512_d64_full 41.5 44.0 2.7e8\n"
                                          "def grid_N512_d64_full 10 11 1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = bench.recorded_tensor_pipe("abc")
    assert rec == {"grid_N512_d64_full": {"tensor_pipe_pct": 41.5, "tensor_pipe_active_pct": 44.0,
                                          "traffic": 2.7e8}}
    assert bench.recorded_tensor_pipe("zzz") == {}


def test_source_hash_covers_every_kernel_source():
    # The ncu records in profiles/ are trusted only while this hash matches,
    # so every file the library is compiled from must be part of it, and
    # the rebuild check must watch the same files.
    import glob
    from exact_tiled_attention_45_b200 import build
    csrc = os.path.join(bench.ROOT, "exact_tiled_attention_45_b200", "csrc")
    kernel_files = sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh")))
    hashed = sorted(os.path.join(bench.ROOT, rel) for rel in bench.KERNEL_SOURCES)
    assert kernel_files == hashed
    assert set(kernel_files) <= {os.path.abspath(p) for p in build.DEPS}
