"""C-ABI library checks that need no GPU: it builds, loads, exports every
symbol ``include/fa2.h`` declares, and rejects bad arguments on the host
before touching CUDA (fake device pointers are never dereferenced)."""
import ctypes
import os
import re
import subprocess

import pytest

from exact_tiled_attention_45_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa2.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(fa2_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_expected_entry_points():
    assert sorted(binding.EXPORTS) == _declared_symbols()


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (fa2_\w+)", out))
    for sym in _declared_symbols():
        assert sym in exported, sym
        assert hasattr(lib, sym)


def test_library_is_built_for_sm100a():
    assert any("arch=compute_100a,code=sm_100a" in f for f in build.NVCC_FLAGS)


def test_version_and_strerror(lib):
    assert lib.fa2_version() >= 100
    for code, word in ((0, b"ok"), (1, b"invalid"), (2, b"unsupported"), (3, b"CUDA"), (4, b"timed out")):
        assert word in lib.fa2_strerror(code)
    assert b"unknown" in lib.fa2_strerror(99)


FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced by the host


def _call(lib, q=FAKE, k=FAKE + (1 << 32), v=FAKE + (2 << 32), o=FAKE + (3 << 32), lse=FAKE + (4 << 32),
          B=1, H=1, N=128, d=64, causal=0, scale=0.125):
    return lib.fa2_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), binding.FA2_ERR_INVALID_ARG),
    (dict(lse=0), binding.FA2_ERR_INVALID_ARG),
    (dict(N=0), binding.FA2_ERR_INVALID_ARG),
    (dict(B=0), binding.FA2_ERR_INVALID_ARG),
    (dict(H=-1), binding.FA2_ERR_INVALID_ARG),
    (dict(B=70000), binding.FA2_ERR_INVALID_ARG),
    (dict(B=65535, H=65535), binding.FA2_ERR_INVALID_ARG),   # B*H >= 2^31
    (dict(B=1024, H=1024, N=2048 * 256), binding.FA2_ERR_INVALID_ARG),  # 2^31 CTAs
    (dict(d=80), binding.FA2_ERR_UNSUPPORTED),
    (dict(d=512), binding.FA2_ERR_UNSUPPORTED),
    (dict(d=16), binding.FA2_ERR_UNSUPPORTED),
    (dict(q=FAKE + 8), binding.FA2_ERR_INVALID_ARG),
    (dict(lse=FAKE + (4 << 32) + 2), binding.FA2_ERR_INVALID_ARG),
    (dict(o=FAKE), binding.FA2_ERR_INVALID_ARG),                   # o aliases q
    (dict(lse=FAKE + (3 << 32) + 64), binding.FA2_ERR_INVALID_ARG),  # lse inside o
    (dict(scale=float("inf")), binding.FA2_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.FA2_ERR_INVALID_ARG),
])
def test_bad_arguments_rejected_before_launch(lib, kw, expect):
    assert _call(lib, **kw) == expect
    assert lib.fa2_last_error_detail()  # a reason is recorded


def test_host_entry_validates_workspace(lib):
    need = lib.fa2_fwd_host_workspace_bytes(1, 2, 128, 64)
    t = 1 * 2 * 128 * 64 * 2
    assert need == 4 * t + 1024
    assert lib.fa2_fwd_host_workspace_bytes(1, 1, 0, 64) == 0
    assert lib.fa2_fwd_host_workspace_bytes(1, 1, 8, 80) == 0
    rc = lib.fa2_fwd_host(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 128, 64, 0, 0.125, FAKE, need - 1, None)
    assert rc == binding.FA2_ERR_INVALID_ARG
    rc = lib.fa2_fwd_host(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 128, 80, 0, 0.125, FAKE, 1 << 30, None)
    assert rc == binding.FA2_ERR_UNSUPPORTED


def test_inject_hook_validates_timeout(lib):
    rc = lib.fa2_fwd_inject_timeout(FAKE, FAKE + (1 << 32), FAKE + (2 << 32), FAKE + (3 << 32), FAKE + (4 << 32),
                                    1, 1, 128, 64, 0, 0.125, ctypes.c_ulonglong(0), None)
    assert rc == binding.FA2_ERR_INVALID_ARG


def test_splitkv_and_backward_hooks_validate_on_the_host(lib):
    p = [FAKE + (i << 32) for i in range(10)]
    rc = lib.fa2_fwd_splitkv_inject_timeout(*p[:5], 1, 2, 1, 1000, 128, 0, 0.088, 2, p[5], 1 << 30,
                                            ctypes.c_ulonglong(0), None)
    assert rc == binding.FA2_ERR_INVALID_ARG and b"timeout" in lib.fa2_last_error_detail()
    rc = lib.fa2_fwd_splitkv_inject_timeout(*p[:5], 1, 2, 1, 1000, 128, 0, 0.088, 2, p[5], 1 << 30,
                                            ctypes.c_ulonglong(3_000_000_000), None)
    assert rc == binding.FA2_ERR_INVALID_ARG
    for kernel, timeout in ((2, 1000), (-1, 1000), (0, 0)):
        rc = lib.fa2_bwd_inject_timeout(*p[:9], 1, 2, 200, 128, 0, 0.088, p[9], 1 << 20, kernel,
                                        ctypes.c_ulonglong(timeout), None)
        assert rc == binding.FA2_ERR_INVALID_ARG, (kernel, timeout)


def test_python_wrapper_rejects_wrong_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        binding._check_qkv(q.float(), q, q, "cpu")
    with pytest.raises(ValueError):
        binding._check_qkv(q, q[..., :32], q, "cpu")
    with pytest.raises(ValueError):
        binding._check_qkv(q.transpose(2, 3), q, q, "cpu")
    with pytest.raises(ValueError):
        binding._check_qkv(q, q, q, "cuda")


@pytest.mark.parametrize("scale", [0.0, -0.125])
def test_non_positive_scale_rejected(lib, scale):
    # Masked scores are -inf before scaling; a scale <= 0 would turn them into
    # NaN or +inf, so the library refuses it.
    assert _call(lib, scale=scale) == binding.FA2_ERR_INVALID_ARG


# ---------------------------------------------------------------- split-K/V

def _skv(lib, q=FAKE, k=FAKE + (1 << 32), v=FAKE + (2 << 32), o=FAKE + (3 << 32), lse=FAKE + (4 << 32),
         B=1, H=2, Nq=1, Nk=1000, d=128, causal=0, scale=0.125, n_splits=0, ws=FAKE + (5 << 32), ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = 1 << 30
    return lib.fa2_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, n_splits, ws, ws_bytes, None)


def test_splitkv_split_count_and_workspace(lib):
    n_kv = 8  # Nk = 1000 -> 8 key tiles of 128
    for req, want in ((1, 1), (2, 2), (3, 3), (5, 4), (7, 4), (8, 8), (9, 8), (500, 8)):
        # a request of s ranges means ceil(8/s) tiles per range, which may
        # cover the 8 tiles with fewer ranges (5 -> 2 tiles each -> 4 ranges)
        got = lib.fa2_fwd_splitkv_splits(1, 2, 1, 1000, 128, req)
        assert got == want, (req, got)
    assert lib.fa2_fwd_splitkv_splits(1, 2, 1, 1000, 128, 1) == 1
    auto = lib.fa2_fwd_splitkv_splits(1, 2, 1, 1000, 128, 0)
    assert 1 <= auto <= n_kv
    # workspace: fp32 partial O then fp32 partial LSE, each rounded to 256 bytes
    s = lib.fa2_fwd_splitkv_splits(2, 3, 5, 1000, 64, 3)
    assert s == 3
    rows = s * 2 * 3 * 5
    r256 = lambda x: (x + 255) // 256 * 256
    assert lib.fa2_fwd_splitkv_workspace_bytes(2, 3, 5, 1000, 64, 3) == r256(rows * 64 * 4) + r256(rows * 4)
    for bad in ((1, 1, 0, 10, 64, 0), (1, 1, 11, 10, 64, 0), (1, 1, 1, 10, 80, 0), (1, 1, 1, 10, 64, -1),
                (300, 300, 1, 10, 64, 0)):
        assert lib.fa2_fwd_splitkv_workspace_bytes(*bad) == 0
        assert lib.fa2_fwd_splitkv_splits(*bad) == 0


def test_splitkv_auto_split_choice(lib):
    # The choice assumes a B200 (148 SMs) when no device can be queried, and a
    # B200 is what the library targets: the fewest ranges giving >= 119 CTAs,
    # with at least 4 key tiles per range.
    assert lib.fa2_fwd_splitkv_splits(8, 16, 1, 16384, 128, 0) == 1      # 128 heads fill the GPU
    assert lib.fa2_fwd_splitkv_splits(1, 16, 1, 65536, 128, 0) == 8      # 16 heads x 8 ranges
    assert lib.fa2_fwd_splitkv_splits(1, 1, 1, 65536, 128, 0) == 103    # ceil(512 / ceil(512 / 119))
    assert lib.fa2_fwd_splitkv_splits(1, 1, 1, 1000, 128, 0) == 2        # only 8 tiles: >= 4 per range
    assert lib.fa2_fwd_splitkv_splits(1, 16, 512, 16384, 128, 0) == 2    # 4 query tiles x 16 heads
    # one range: no workspace, the kernel writes O and LSE itself
    assert lib.fa2_fwd_splitkv_workspace_bytes(8, 16, 1, 16384, 128, 0) == 0
    assert lib.fa2_fwd_splitkv_workspace_bytes(8, 16, 1, 16384, 128, 1) == 0
    assert lib.fa2_fwd_splitkv_workspace_bytes(8, 16, 1, 16384, 128, 2) > 0


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), binding.FA2_ERR_INVALID_ARG),
    (dict(ws=0, n_splits=2), binding.FA2_ERR_INVALID_ARG),          # two ranges need a workspace
    (dict(Nq=0), binding.FA2_ERR_INVALID_ARG),
    (dict(Nq=1001), binding.FA2_ERR_INVALID_ARG),          # Nq > Nk
    (dict(B=300, H=300), binding.FA2_ERR_INVALID_ARG),     # B*H > 65535
    (dict(n_splits=-1), binding.FA2_ERR_INVALID_ARG),
    (dict(scale=0.0), binding.FA2_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.FA2_ERR_INVALID_ARG),
    (dict(d=80), binding.FA2_ERR_UNSUPPORTED),
    (dict(ws=FAKE + (5 << 32) + 128), binding.FA2_ERR_INVALID_ARG),  # workspace not 256-aligned
    (dict(ws_bytes=1024), binding.FA2_ERR_INVALID_ARG),              # workspace too small
    (dict(o=FAKE + (1 << 32)), binding.FA2_ERR_INVALID_ARG),         # o aliases k
    (dict(ws=FAKE + (2 << 32)), binding.FA2_ERR_INVALID_ARG),        # workspace aliases v
])
def test_splitkv_bad_arguments_rejected_before_launch(lib, kw, expect):
    assert _skv(lib, **kw) == expect
    assert lib.fa2_last_error_detail()


def test_splitkv_wrapper_shape_checks():
    import torch
    q = torch.zeros(1, 2, 4, 64, dtype=torch.bfloat16)
    kv = torch.zeros(1, 2, 9, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):  # tensors on the CPU
        binding._check_q_kv(q, kv, kv)


def test_static_scratch_entry_rejects_on_the_host(lib):
    # beyond the 16 MiB scratch: 32 ranges x 16 heads x 4096 rows x (128 + 1) floats
    rc = lib.fa2_fwd_splitkv_static(FAKE, FAKE + (1 << 32), FAKE + (2 << 32), FAKE + (3 << 32), FAKE + (4 << 32),
                                    1, 16, 4096, 4096, 128, 1, 0.088, 32, None)
    assert rc == binding.FA2_ERR_INVALID_ARG
    assert b"static scratch" in lib.fa2_last_error_detail()
    rc = lib.fa2_fwd_splitkv_static(0, FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 128, 64, 0, 0.125, 0, None)
    assert rc == binding.FA2_ERR_INVALID_ARG


@pytest.mark.parametrize("d", [32, 96, 256])
def test_static_scratch_sizes_every_head_dim(lib, d):
    # The scratch need is computed for every supported head dimension (the
    # zero-padded 32 and 96, and 256 with its 64-key tiles), so an oversized
    # request is refused for the scratch's size, not for a missing workspace.
    assert lib.fa2_fwd_splitkv_workspace_bytes(1, 16, 4096, 4096, d, 32) > binding.SPLITKV_STATIC_SCRATCH_BYTES
    rc = lib.fa2_fwd_splitkv_static(FAKE, FAKE + (1 << 32), FAKE + (2 << 32), FAKE + (3 << 32), FAKE + (4 << 32),
                                    1, 16, 4096, 4096, d, 1, 0.088, 32, None)
    assert rc == binding.FA2_ERR_INVALID_ARG
    assert b"static scratch" in lib.fa2_last_error_detail()


# ---------------------------------------------------------------- backward

def _bwd(lib, B=1, H=2, N=200, d=128, causal=0, scale=0.088, ws=FAKE + (9 << 32), ws_bytes=1 << 20, **ptrs):
    names = ["q", "k", "v", "o", "do", "lse", "dq", "dk", "dv"]
    p = {n: FAKE + (i << 32) for i, n in enumerate(names)}
    p.update(ptrs)
    return lib.fa2_bwd(*(p[n] for n in names), B, H, N, d, causal, scale, ws, ws_bytes, None)


def test_bwd_workspace_size(lib):
    # lse2 and D, fp32, rows padded to 128 per head, each rounded to 256 bytes
    assert lib.fa2_bwd_workspace_bytes(2, 3, 200, 128) == 2 * (2 * 3 * 256 * 4)
    assert lib.fa2_bwd_workspace_bytes(1, 1, 1, 64) == 2 * 512
    assert lib.fa2_bwd_workspace_bytes(1, 1, 0, 64) == 0
    assert lib.fa2_bwd_workspace_bytes(1, 1, 8, 80) == 0
    assert lib.fa2_bwd_workspace_bytes(1, 1, 8, 256) == 2 * 512  # d = 256 too (64-key / 64-query tiles)
    assert lib.fa2_bwd_workspace_bytes(1, 1, 8, 96) == 2 * 512  # d = 96 runs on zero-padded 128-column tiles


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), binding.FA2_ERR_INVALID_ARG),
    (dict(dv=0), binding.FA2_ERR_INVALID_ARG),
    (dict(ws=0), binding.FA2_ERR_INVALID_ARG),
    (dict(N=0), binding.FA2_ERR_INVALID_ARG),
    (dict(d=80), binding.FA2_ERR_UNSUPPORTED),
    (dict(d=512), binding.FA2_ERR_UNSUPPORTED),
    (dict(scale=0.0), binding.FA2_ERR_INVALID_ARG),
    (dict(scale=float("inf")), binding.FA2_ERR_INVALID_ARG),
    (dict(ws=FAKE + (9 << 32) + 64), binding.FA2_ERR_INVALID_ARG),   # workspace not 256-aligned
    (dict(ws_bytes=1024), binding.FA2_ERR_INVALID_ARG),              # too small (needs 4096)
    (dict(dq=FAKE), binding.FA2_ERR_INVALID_ARG),                    # dq aliases q
    (dict(dk=FAKE + (6 << 32)), binding.FA2_ERR_INVALID_ARG),        # dk aliases dq
    (dict(ws=FAKE + (8 << 32)), binding.FA2_ERR_INVALID_ARG),        # workspace aliases dv
    (dict(o=FAKE + (1 << 32) + 8), binding.FA2_ERR_INVALID_ARG),     # misaligned o
])
def test_bwd_bad_arguments_rejected_before_launch(lib, kw, expect):
    assert _bwd(lib, **kw) == expect
    assert lib.fa2_last_error_detail()


def test_padded_head_dims_size_like_the_wider_kernel(lib):
    # d = 32 and 96 run on the 64- and 128-column kernels; the split-K/V
    # partials are kept at the padded width, the user tensors at d.
    assert lib.fa2_fwd_splitkv_workspace_bytes(1, 2, 3, 1000, 96, 2) == lib.fa2_fwd_splitkv_workspace_bytes(
        1, 2, 3, 1000, 128, 2)
    assert lib.fa2_fwd_splitkv_workspace_bytes(1, 2, 3, 1000, 32, 2) == lib.fa2_fwd_splitkv_workspace_bytes(
        1, 2, 3, 1000, 64, 2)
    assert lib.fa2_fwd_host_workspace_bytes(1, 2, 128, 96) == 4 * (2 * 128 * 96 * 2) + 1024


def test_head_dim_256_uses_64_key_tiles(lib):
    # d = 256 runs on the one-tile kernel with 64-key tiles: 1000 keys are 16
    # tiles (8 at 128 keys), so up to 16 ranges and >= 4 tiles per range.
    assert lib.fa2_fwd_splitkv_splits(1, 1, 1, 1000, 256, 500) == 16
    assert lib.fa2_fwd_splitkv_splits(1, 1, 1, 1000, 128, 500) == 8
    assert lib.fa2_fwd_splitkv_splits(1, 1, 1, 1000, 256, 0) == 4
    rows = 2 * 1 * 2 * 3
    assert lib.fa2_fwd_splitkv_workspace_bytes(1, 2, 3, 1000, 256, 2) == (rows * 256 * 4 + 255) // 256 * 256 + 256


def test_output_buffer_checks_reject_wrong_buffers():
    # Caller-provided outputs and workspaces are checked before the library
    # sees their pointers (a short or misshapen buffer would be written past
    # its end by the kernels).
    import torch
    ok = torch.empty((2, 3, 5, 64), dtype=torch.bfloat16)
    binding._check_buffer("out", ok, (2, 3, 5, 64), torch.bfloat16, "cpu")
    with pytest.raises(TypeError):
        binding._check_buffer("out", ok.float(), (2, 3, 5, 64), torch.bfloat16, "cpu")
    with pytest.raises(ValueError):
        binding._check_buffer("out", ok[:, :, :4], (2, 3, 5, 64), torch.bfloat16, "cpu")
    with pytest.raises(ValueError):
        binding._check_buffer("out", ok.transpose(2, 3).contiguous().transpose(2, 3), (2, 3, 5, 64),
                              torch.bfloat16, "cpu")
    with pytest.raises(ValueError):
        binding._check_buffer("out", ok, (2, 3, 5, 64), torch.bfloat16, "cuda")
    lse = torch.empty((2, 3, 5), dtype=torch.float32)
    with pytest.raises(ValueError):
        binding._check_buffer("lse", lse, (2, 3, 6), torch.float32, "cpu")
    with pytest.raises(ValueError):
        binding._check_workspace(torch.empty(16, dtype=torch.uint8), 16)  # host memory, not device
