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
    (dict(d=96), binding.FA2_ERR_UNSUPPORTED),
    (dict(d=256), binding.FA2_ERR_UNSUPPORTED),
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
