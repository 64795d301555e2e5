"""The C ABI library loads and exports every symbol include/nvfp4.h declares;
host-side argument checks reject bad calls before any launch (no GPU needed:
each call below fails its checks before touching the device)."""
import ctypes
import os
import re

import pytest

from nvfp4_w4a4_gemm_quantize_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")

OK, INVALID, SHAPE, MISALIGNED, DEVICE, CUDA, TIMEOUT, WORKSPACE, NONFINITE = range(9)
A = 0x10000          # fake, 16-byte aligned device addresses (never dereferenced)
B = 0x20000
C = 0x30000


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) == 24, names
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.SIGNATURES, n


def test_sf_bytes_and_workspace(L):
    assert L.nvfp4_sf_bytes(128, 256) == 128 * 16
    assert L.nvfp4_sf_bytes(600, 4096) == 640 * 256
    assert L.nvfp4_sf_bytes(0, 64) == 0
    assert L.nvfp4_sf_bytes(5, 32) == 0          # k not a multiple of 64
    assert L.nvfp4_sf_bytes(-1, 64) == 0
    assert L.nvfp4_quantize_workspace_bytes(32768, 12288) >= 1024


def test_status_strings(L):
    for s in range(9):
        assert L.nvfp4_status_string(s)
        assert b"unknown" not in L.nvfp4_status_string(s)
    assert b"unknown" in L.nvfp4_status_string(99)


def test_debug_wait_rejects_bad_arguments(L):
    w = L.nvfp4_debug_wait_timeout
    assert w(None, 1000, None) == INVALID
    assert w(A, 0, None) == INVALID
    assert w(A, 2000001, None) == INVALID
    assert w(A + 2, 1000, None) == MISALIGNED


def test_shutdown_runs_without_a_device(L):
    L.nvfp4_shutdown()
    L.nvfp4_shutdown()


def test_quantize_rejects_bad_arguments(L):
    q = L.nvfp4_quantize
    # k not a multiple of 64
    assert q(A, 128, 96, 96, B, C, A, 1, None, 0, None, None) == SHAPE
    # null input
    assert q(None, 128, 256, 256, B, C, A, 1, None, 0, None, None) == INVALID
    # null tensor scale
    assert q(A, 128, 256, 256, B, C, None, 1, None, 0, None, None) == INVALID
    # ld_x < k
    assert q(A, 128, 256, 128, B, C, A, 1, None, 0, None, None) == INVALID
    # unknown flag
    assert q(A, 128, 256, 256, B, C, A, 4, None, 0, None, None) == INVALID
    # dynamic scale without workspace
    assert q(A, 128, 256, 256, B, C, A, 0, None, 0, None, None) == WORKSPACE
    assert q(A, 128, 256, 256, B, C, A, 0, A, 16, None, None) == WORKSPACE
    # misaligned pointers / row stride
    assert q(A + 2, 128, 256, 256, B, C, A, 1, None, 0, None, None) == MISALIGNED
    assert q(A, 128, 256, 260, B, C, A, 1, None, 0, None, None) == MISALIGNED
    assert q(A, 128, 256, 256, B + 8, C, A, 1, None, 0, None, None) == MISALIGNED
    # more rows than the tile grid can hold (65535 row blocks of 128): rejected
    # before any launch, by every quantize entry point that takes that grid
    big = 65535 * 128 + 1
    assert q(A, big, 64, 64, B, C, A, 1, None, 0, None, None) == SHAPE
    assert L.nvfp4_quantize_block(A, big, 64, 64, 32, B, C, A, 1, None, 0, None, None) == SHAPE
    assert L.nvfp4_fake_quantize(A, big, 64, 64, B, 0, None, A, 1, None, 0, None, None) == SHAPE
    assert L.nvfp4_quantize_noalloc(A, big, 64, 64, B, C, A, 0, None, None) == SHAPE


def test_layernorm_quantize_rejects_bad_arguments(L):
    f = L.nvfp4_layernorm_quantize
    # (x, rows, k, ld, gamma, beta, rows_per_group, eps, codes, sf, scale, flags, ws, ws_bytes, dev_status, stream)
    assert f(A, 128, 96, 96, None, None, 0, 1e-6, B, C, A, 1, None, 0, None, None) == SHAPE
    assert f(A, 128, 256, 256, None, None, 0, 0.0, B, C, A, 1, None, 0, None, None) == INVALID     # eps <= 0
    assert f(A, 128, 256, 256, None, None, -1, 1e-6, B, C, A, 1, None, 0, None, None) == INVALID   # group size
    assert f(None, 128, 256, 256, None, None, 0, 1e-6, B, C, A, 1, None, 0, None, None) == INVALID
    assert f(A, 128, 256, 256, None, None, 0, 1e-6, B, C, None, 1, None, 0, None, None) == INVALID
    assert f(A, 128, 256, 256, None, None, 0, 1e-6, B, C, A, 0, None, 0, None, None) == WORKSPACE
    assert f(A, 128, 256, 256, A + 4, None, 0, 1e-6, B, C, A, 1, None, 0, None, None) == MISALIGNED
    assert f(A, 128, 256, 260, None, None, 0, 1e-6, B, C, A, 1, None, 0, None, None) == MISALIGNED


def test_dequantize_rejects_bad_arguments(L):
    d = L.nvfp4_dequantize
    assert d(A, B, C, 128, 256, A, 7, None) == INVALID
    assert d(A, B, C, 128, 100, A, 0, None) == SHAPE
    assert d(None, B, C, 128, 256, A, 0, None) == INVALID
    assert d(A + 4, B, C, 128, 256, A, 0, None) == MISALIGNED


def test_gemm_rejects_bad_arguments(L):
    g = L.nvfp4_gemm_w4a4
    args = [A, B, C, A, B, C]
    # K not multiple of 64
    assert g(*args, 128, 256, 96, A, 0, None, None, None, None, 0, None, None) == SHAPE
    # N not multiple of 8 for bf16 output
    assert g(*args, 128, 260, 256, A, 0, None, None, None, None, 0, None, None) == SHAPE
    # fused NVFP4 output needs N % 64 == 0
    assert g(*args, 128, 96, 256, None, 0, A, B, C, None, 0, None, None) == SHAPE
    # both outputs given
    assert g(*args, 128, 256, 256, A, 0, A, B, C, None, 0, None, None) == INVALID
    # no output at all
    assert g(*args, 128, 256, 256, None, 0, None, None, None, None, 0, None, None) == INVALID
    # bad dtype
    assert g(*args, 128, 256, 256, A, 5, None, None, None, None, 0, None, None) == INVALID
    # null scale
    assert g(A, B, None, A, B, C, 128, 256, 256, A, 0, None, None, None, None, 0, None, None) == INVALID
    # misaligned operand
    assert g(A + 1, B, C, A, B, C, 128, 256, 256, A, 0, None, None, None, None, 0, None, None) == MISALIGNED
    # unknown activation
    assert g(*args, 128, 256, 256, A, 0, None, None, None, None, 2, None, None) == INVALID
    # negative M
    assert g(*args, -1, 256, 256, A, 0, None, None, None, None, 0, None, None) == INVALID


def test_fake_quantize_rejects_bad_arguments(L):
    f = L.nvfp4_fake_quantize
    # (x, rows, k, ld, y, y_dtype, mask, scale, flags, ws, ws_bytes, dev_status, stream)
    assert f(A, 128, 96, 96, B, 0, C, A, 1, None, 0, None, None) == SHAPE
    assert f(None, 128, 256, 256, B, 0, C, A, 1, None, 0, None, None) == INVALID
    assert f(A, 128, 256, 256, None, 0, C, A, 1, None, 0, None, None) == INVALID
    assert f(A, 128, 256, 256, B, 3, C, A, 1, None, 0, None, None) == INVALID
    assert f(A, 128, 256, 256, B, 0, C, None, 1, None, 0, None, None) == INVALID
    assert f(A, 128, 256, 128, B, 0, C, A, 1, None, 0, None, None) == INVALID
    assert f(A, 128, 256, 256, B, 0, C, A, 2, None, 0, None, None) == INVALID
    assert f(A, 128, 256, 256, B, 0, C, A, 0, None, 0, None, None) == WORKSPACE
    assert f(A, 128, 256, 256, B + 8, 0, C, A, 1, None, 0, None, None) == MISALIGNED
    assert f(A, 128, 256, 256, B, 0, C + 2, A, 1, None, 0, None, None) == MISALIGNED
    assert f(A, 128, 256, 260, B, 0, None, A, 1, None, 0, None, None) == MISALIGNED


def test_ste_backward_rejects_bad_arguments(L):
    s = L.nvfp4_ste_backward
    assert s(A, B, 128, 24, 0, C, None) == SHAPE
    assert s(A, B, 128, 256, 2, C, None) == INVALID
    assert s(None, B, 128, 256, 0, C, None) == INVALID
    assert s(A, None, 128, 256, 0, C, None) == INVALID
    assert s(A, B, -1, 256, 0, C, None) == INVALID
    assert s(A, B + 2, 128, 256, 0, C, None) == MISALIGNED


def _problems(n, over=None):
    arr = (_lib.NVFP4GemmProblem * n)()
    for i in range(n):
        pr = arr[i]
        pr.a_codes, pr.a_sf, pr.a_scale, pr.b_codes, pr.b_sf, pr.b_scale = A, B, C, A, B, C
        pr.M, pr.N, pr.K, pr.y = 128, 256, 256, A
        for k, v in (over or {}).get(i, {}).items():
            setattr(pr, k, v)
    return arr


def test_grouped_gemm_rejects_bad_arguments(L):
    g = L.nvfp4_gemm_w4a4_grouped
    addr = ctypes.addressof
    assert g(None, 1, 0, None, None) == INVALID
    arr = _problems(9)
    assert g(addr(arr), 0, 0, None, None) == INVALID
    assert g(addr(arr), 9, 0, None, None) == INVALID
    assert g(addr(arr), 2, 7, None, None) == INVALID                                 # bad dtype
    # mixed output kinds in one launch
    arr = _problems(2, {1: dict(y=None, y_codes=A, y_sf=B, y_scale=C)})
    assert g(addr(arr), 2, 0, None, None) == INVALID
    arr = _problems(3, {2: dict(K=96)})
    assert g(addr(arr), 3, 0, None, None) == SHAPE
    arr = _problems(2, {1: dict(N=260)})
    assert g(addr(arr), 2, 0, None, None) == SHAPE
    arr = _problems(2, {0: dict(a_codes=A + 4)})
    assert g(addr(arr), 2, 0, None, None) == MISALIGNED
    arr = _problems(2, {1: dict(b_scale=None)})
    assert g(addr(arr), 2, 0, None, None) == INVALID
    arr = _problems(2, {0: dict(M=-1)})
    assert g(addr(arr), 2, 0, None, None) == INVALID
    arr = _problems(2, {1: dict(act=1)})                                              # mixed activations
    assert g(addr(arr), 2, 0, None, None) == INVALID


def test_mx_calls_reject_bad_arguments(L):
    assert L.nvfp4_mx_sf_bytes(128, 256) == 128 * 8
    assert L.nvfp4_mx_sf_bytes(130, 384) == 256 * 12
    assert L.nvfp4_mx_sf_bytes(128, 64) == 0                    # k not a multiple of 128
    q = L.nvfp4_mx_quantize
    assert q(A, 128, 192, 192, B, C, None) == SHAPE
    assert q(None, 128, 256, 256, B, C, None) == INVALID
    assert q(A, 128, 256, 128, B, C, None) == INVALID
    assert q(A + 2, 128, 256, 256, B, C, None) == MISALIGNED
    assert q(A, 128, 256, 260, B, C, None) == MISALIGNED
    assert q(A, 65535 * 64 + 1, 256, 256, B, C, None) == SHAPE
    d = L.nvfp4_mx_dequantize
    assert d(A, B, 128, 256, C, 4, None) == INVALID
    assert d(A, B, 128, 64, C, 0, None) == SHAPE
    g = L.nvfp4_mx_gemm
    assert g(A, B, A, B, 128, 256, 192, C, 0, 0, None, None) == SHAPE
    assert g(A, B, A, B, 128, 260, 256, C, 0, 0, None, None) == SHAPE
    assert g(A, B, A, B, 128, 256, 256, None, 0, 0, None, None) == INVALID
    assert g(A, B, A, B, 128, 256, 256, C, 0, 3, None, None) == INVALID
    assert g(A, B + 4, A, B, 128, 256, 256, C, 0, 0, None, None) == MISALIGNED
    assert g(A, B, A, B, -2, 256, 256, C, 0, 0, None, None) == INVALID


def test_block_size_calls(L):
    qb = L.nvfp4_quantize_block
    assert qb(A, 128, 256, 256, 48, B, C, A, 1, None, 0, None, None) == INVALID     # block not 16/32/64
    assert qb(A, 128, 96, 96, 32, B, C, A, 1, None, 0, None, None) == SHAPE
    assert qb(A, 128, 256, 256, 64, B, C, A, 0, None, 0, None, None) == WORKSPACE
    assert qb(A + 2, 128, 256, 256, 32, B, C, A, 1, None, 0, None, None) == MISALIGNED
    e = L.nvfp4_block_size_errors
    assert e(A, 128, 96, 96, B, C, None) == SHAPE
    assert e(A, 128, 256, 256, None, C, None) == INVALID
    assert e(A, 128, 256, 256, B, C + 4, None) == MISALIGNED
    sel = L.nvfp4_select_block_size
    err = (ctypes.c_double * 8)(1.0, 1.0, 1.0, 0.10, 0.15, 1.0, 1.0, 1.0)
    assert sel(ctypes.addressof(err), 0.0) == 8
    assert sel(ctypes.addressof(err), 2.0) == 16
    assert sel(ctypes.addressof(err), 1e6) == 64
    assert sel(None, 1.0) == 0 and sel(ctypes.addressof(err), -1.0) == 0


def test_attention_rejects_bad_arguments(L):
    a = L.nvfp4_attention
    ops = [A, B, C] * 3
    assert a(*ops, None, 2, 128, 256, 64, A, C, 1 << 30, None, None) == SHAPE          # d != 128
    assert a(*ops, None, 2, 100, 256, 128, A, C, 1 << 30, None, None) == SHAPE         # Lq % 128
    assert a(*ops, None, 2, 128, 200, 128, A, C, 1 << 30, None, None) == SHAPE         # Lk % 128
    assert a(*ops, None, 0, 128, 256, 128, A, C, 1 << 30, None, None) == INVALID
    assert a(None, B, C, A, B, C, A, B, C, None, 2, 128, 256, 128, A, C, 1 << 30, None, None) == INVALID
    assert a(*ops, None, 2, 128, 256, 128, None, C, 1 << 30, None, None) == INVALID
    assert a(A + 8, B, C, A, B, C, A, B, C, None, 2, 128, 256, 128, A, C, 1 << 30, None, None) == MISALIGNED
    assert a(*ops, C + 2, 2, 128, 256, 128, A, C, 1 << 30, None, None) == MISALIGNED
    assert a(*ops, None, 2, 128, 256, 128, A, C, 100, None, None) == WORKSPACE
    assert a(*ops, None, 2, 128, 256, 128, A, None, 1 << 30, None, None) == WORKSPACE
    # room for the decoded V but not for the heads' decode slots
    assert a(*ops, None, 2, 128, 256, 128, A, C, 2 * 128 * 256 * 2, None, None) == WORKSPACE
    assert L.nvfp4_attention_workspace_bytes(2, 256, 128) == 2 * 128 * 256 * 2 + 2 * 128


def test_w4a16_rejects_bad_arguments(L):
    g = L.nvfp4_gemm_w4a16
    assert g(A, B, C, A, 128, 256, 96, A, 0, None, None) == SHAPE
    assert g(A, B, C, A, 128, 250, 256, A, 0, None, None) == SHAPE
    assert g(None, B, C, A, 128, 256, 256, A, 0, None, None) == INVALID
    assert g(A, B, C, A, 128, 256, 256, None, 0, None, None) == INVALID
    assert g(A + 2, B, C, A, 128, 256, 256, A, 0, None, None) == MISALIGNED


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(_lib, "_LIB", None)
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()
