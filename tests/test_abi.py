"""CPU tests of the C ABI: the library loads, exports every entry point the
header declares, sizes buffers as documented, and rejects bad arguments on
the host before touching a device."""

from __future__ import annotations

import ctypes as C
import os
import re

import pytest

from reference_sliding_window_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rswa.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(rswa_[a-z_]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    return _native.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("rswa_init", "rswa_load_reference", "rswa_append", "rswa_decode",
                 "rswa_append_decode", "rswa_masked_forward", "rswa_cache_len",
                 "rswa_cache_positions", "rswa_reset", "rswa_destroy", "rswa_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in _native._PROTOS, f"binding lacks a prototype for {name}"


def test_version(lib):
    assert lib.rswa_version().decode().startswith("rswa ")


def test_cache_bytes(lib):
    # [B][H][L_m_cap + window][d] elements
    assert lib.rswa_cache_bytes(2592, 128, 10, 128, 1, _native.BF16) == 1 * 10 * 2720 * 128 * 2
    assert lib.rswa_cache_bytes(272, 128, 2, 64, 1, _native.F32) == 2 * 400 * 64 * 4
    assert lib.rswa_cache_bytes(12832, 100000, 10, 128, 8, _native.BF16) == 8 * 10 * 112832 * 128 * 2
    assert lib.rswa_cache_bytes(10, 4, 2, 96, 1, _native.BF16) == 0      # d unsupported
    assert lib.rswa_cache_bytes(0, 4, 2, 64, 1, _native.BF16) == 0
    assert lib.rswa_cache_bytes(10, 0, 2, 64, 1, _native.BF16) == 0
    assert lib.rswa_cache_bytes(10, 4, 2, 64, 1, 7) == 0


def test_workspace_bytes(lib):
    ws = lib.rswa_workspace_bytes(2592, 128, 10, 128, 1)
    assert ws > 0 and ws % 256 == 0
    # grows with batch*heads (per-(b,h) tickets and partial slots)
    assert lib.rswa_workspace_bytes(2592, 128, 10, 128, 64) > ws
    assert lib.rswa_workspace_bytes(2592, 128, 10, 96, 1) == 0


def _err(lib):
    return lib.rswa_last_error().decode()


def test_init_rejects_bad_arguments_before_device(lib):
    h = C.c_void_p()
    buf = C.create_string_buffer(64)
    p = C.cast(buf, C.c_void_p).value
    p16 = (p + 15) // 16 * 16
    assert lib.rswa_init(None, 0, 10, 4, 0, 2, 64, 1, _native.BF16, p16, p16, p16, 1 << 20, None) == _native.ERR_ARG
    assert lib.rswa_init(C.byref(h), 0, 10, 4, 0, 2, 96, 1, _native.BF16, p16, p16, p16, 1 << 20, None) == _native.ERR_UNSUPPORTED
    assert "head dim" in _err(lib)
    assert lib.rswa_init(C.byref(h), 0, 10, 0, 0, 2, 64, 1, _native.BF16, p16, p16, p16, 1 << 20, None) == _native.ERR_ARG
    assert "window" in _err(lib)
    assert lib.rswa_init(C.byref(h), 1, 10, 4, 0, 2, 64, 1, _native.BF16, p16, p16, p16, 1 << 20, None) == _native.ERR_ARG
    assert "T_cap" in _err(lib)
    assert lib.rswa_init(C.byref(h), 0, 10, 4, 0, 2, 64, 1, _native.BF16, None, p16, p16, 1 << 20, None) == _native.ERR_ARG
    assert lib.rswa_init(C.byref(h), 0, 10, 4, 0, 256, 64, 257, _native.BF16, p16, p16, p16, 1 << 20, None) == _native.ERR_ARG
    assert "65535" in _err(lib)
    assert lib.rswa_init(C.byref(h), 0, 10, 4, 0, 2, 64, 1, _native.BF16, p16 + 8, p16, p16, 1 << 20, None) == _native.ERR_ARG
    assert "aligned" in _err(lib)
    assert lib.rswa_init(C.byref(h), 0, 10, 4, 0, 2, 64, 1, _native.BF16, p16, p16, p16, 16, None) == _native.ERR_ARG
    assert "workspace" in _err(lib)
    assert lib.rswa_init(C.byref(h), 5, 10, 4, 0, 2, 64, 1, _native.BF16, p16, p16, p16, 1 << 20, None) == _native.ERR_ARG
    assert h.value is None


def test_null_handle_is_an_argument_error(lib):
    assert lib.rswa_append(None, None, None) == _native.ERR_ARG
    assert lib.rswa_load_packed(None, None, None, 1, None, 0) == _native.ERR_ARG
    assert lib.rswa_decode(None, None, None, 0.0) == _native.ERR_ARG
    assert lib.rswa_append_decode(None, None, None, None, None, 0.0) == _native.ERR_ARG
    assert lib.rswa_reset(None) == _native.ERR_ARG
    assert lib.rswa_check(None) == _native.ERR_ARG
    assert lib.rswa_cache_len(None, None) == _native.ERR_ARG
    assert lib.rswa_load_reference_chunk(None, None, None, 1, None) == _native.ERR_ARG
    assert lib.rswa_masked_forward_fill(None, None, None, None, None, 8, 4, 0.0, 0) == _native.ERR_ARG
    lib.rswa_destroy(None)  # no-op


def test_layers_call_rejects_bad_arguments_before_device(lib):
    P = C.c_void_p * 2
    buf = C.create_string_buffer(256)
    p = (C.cast(buf, C.c_void_p).value + 15) // 16 * 16
    ptrs = P(p, p)
    f = lib.rswa_append_decode_layers
    assert f(None, 2, ptrs, ptrs, ptrs, ptrs, 0.0) == _native.ERR_ARG
    assert f(P(None, None), 2, ptrs, ptrs, ptrs, ptrs, 0.0) == _native.ERR_ARG   # null handles
    assert f(P(None, None), 0, ptrs, ptrs, ptrs, ptrs, 0.0) == _native.ERR_ARG   # R < 1
    assert f(P(None, None), 2, ptrs, ptrs, ptrs, ptrs, float("inf")) == _native.ERR_ARG
    assert f(P(None, None), 2, None, ptrs, ptrs, ptrs, 0.0) == _native.ERR_ARG


def test_masked_forward_rejects_bad_arguments_before_device(lib):
    buf = C.create_string_buffer(256)
    p = (C.cast(buf, C.c_void_p).value + 15) // 16 * 16
    mf = lib.rswa_masked_forward
    assert mf(None, p, p, p, 8, 2, 2, 1, 64, _native.F32, 0.0, None) == _native.ERR_ARG
    assert mf(p, p, p, p + 4, 8, 2, 2, 1, 64, _native.F32, 0.0, None) == _native.ERR_ARG
    assert mf(p, p, p, p, 8, 2, 2, 1, 80, _native.F32, 0.0, None) == _native.ERR_UNSUPPORTED
    assert mf(p, p, p, p, 8, -1, 2, 1, 64, _native.F32, 0.0, None) == _native.ERR_ARG  # L_m = 0 is the plain window
    assert mf(p, p, p, p, 8, 9, 2, 1, 64, _native.F32, 0.0, None) == _native.ERR_ARG
    assert mf(p, p, p, p, 8, 2, 0, 1, 64, _native.F32, 0.0, None) == _native.ERR_ARG
    assert mf(p, p, p, p, 8, 2, 2, 1, 64, _native.F32, float("nan"), None) == _native.ERR_ARG
    assert mf(p, p, p, p, 8, 2, 2, 1, 64, 3, 0.0, None) == _native.ERR_UNSUPPORTED


def test_masked_forward_ex_rejects_unknown_flags(lib):
    buf = C.create_string_buffer(256)
    p = (C.cast(buf, C.c_void_p).value + 15) // 16 * 16
    mfx = lib.rswa_masked_forward_ex
    assert mfx(p, p, p, p, 8, 2, 2, 1, 64, _native.F32, 0.0, 2, None) == _native.ERR_ARG
    assert mfx(p, p, p, p, 8, 2, 2, 1, 64, _native.F32, 0.0, -1, None) == _native.ERR_ARG
    assert mfx(None, p, p, p, 8, 2, 2, 1, 64, _native.F32, 0.0, _native.FLAG_BIDIR_PREFIX, None) == _native.ERR_ARG


def test_masked_forward_varlen_rejects_bad_arguments_before_device(lib):
    # Every case fails the host checks, so nothing is launched.
    buf = C.create_string_buffer(256)
    p = (C.cast(buf, C.c_void_p).value + 15) // 16 * 16
    mv = lib.rswa_masked_forward_varlen

    def call(cu, refs, n_docs=None, n=2, H=1, d=64, dtype=_native.F32, scale=0.0, flags=0, Q=p, O=p):
        cu_a = (C.c_int32 * len(cu))(*cu)
        refs_a = (C.c_int32 * max(len(refs), 1))(*refs)
        nd = len(refs) if n_docs is None else n_docs
        return mv(Q, p, p, O, cu_a, refs_a, nd, n, H, d, dtype, scale, flags, None)

    assert call([0, 4], [1], Q=None) == _native.ERR_ARG
    assert call([0, 4], [1], O=p + 4) == _native.ERR_ARG
    assert call([0], [], n_docs=0) == _native.ERR_ARG
    assert call([0, 4], [1], flags=2) == _native.ERR_ARG
    assert call([1, 4], [1]) == _native.ERR_ARG          # must start at 0
    assert call([0, 4, 4], [1, 0]) == _native.ERR_ARG    # empty document
    assert call([0, 4, 3], [1, 0]) == _native.ERR_ARG    # decreasing
    assert call([0, 4], [5]) == _native.ERR_ARG          # more reference rows than rows
    assert call([0, 4, 6], [1, -1]) == _native.ERR_ARG
    assert call([0, 4], [1], n=0) == _native.ERR_ARG
    assert call([0, 4], [1], H=0) == _native.ERR_ARG
    assert call([0, 4], [1], d=80) == _native.ERR_UNSUPPORTED
    assert call([0, 4], [1], dtype=3) == _native.ERR_UNSUPPORTED
    assert call([0, 4], [1], scale=float("inf")) == _native.ERR_ARG
    assert call([0, 1 << 30], [0], H=4) == _native.ERR_ARG  # 2^31 elements or more


def test_product_path_has_no_oracle_dependency():
    # The package must never import the oracle (or any CPU fallback).
    pkg = os.path.join(ROOT, "reference_sliding_window_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", src, re.M), f
                assert "rswa_oracle" not in src, f
