"""Host-side checks of the C-ABI library (no GPU needed): it builds, loads,
exports every symbol include/kata.h declares, and rejects bad arguments on the
host before touching a device."""

import ctypes
import os
import re

import pytest

from kernelized_linear_attention_kata_b200 import build as kbuild
from kernelized_linear_attention_kata_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return L.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"KATA_API\s+[\w\s\*]+?\b(kata_\w+)\s*\(", text))
    return names


def test_header_declares_the_abi():
    names = declared_symbols()
    for required in ("kata_fwd_chunked", "kata_fwd_quadratic", "kata_decode_step",
                     "kata_state_dim", "kata_fwd_chunked_workspace_bytes",
                     "kata_workspace_status", "kata_status_string", "kata_bwd_chunked",
                     "kata_bwd_chunked_workspace_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(L.SIGNATURES) == declared_symbols()


def test_library_has_no_torch_dependency():
    """The .so is a plain C ABI: it must not link against libtorch/libc10."""
    text = open(L.LIB_PATH, "rb").read()
    assert b"libtorch" not in text and b"libc10" not in text


def test_state_dim(lib):
    assert lib.kata_state_dim(32, L.KATA_FEATURE_PSD) == 528
    assert lib.kata_state_dim(16, L.KATA_FEATURE_PSD) == 136
    assert lib.kata_state_dim(64, L.KATA_FEATURE_FIRST_ORDER) == 65
    assert lib.kata_state_dim(0, L.KATA_FEATURE_PSD) == 0
    assert lib.kata_state_dim(32, 7) == 0


def test_status_strings(lib):
    for code in range(7):
        assert lib.kata_status_string(code).decode().startswith("KATA_")
    assert lib.kata_status_string(99) == b"KATA_ERR_UNKNOWN"
    assert lib.kata_version() >= 100


def _fwd(lib, fn="kata_fwd_chunked", d_k=32, d_v=64, C=64, dtype=L.KATA_DTYPE_BF16,
         feature=L.KATA_FEATURE_PSD, B=1, H=1, T=16, ws=None, ws_bytes=1 << 20, ptr=256):
    p = ctypes.c_void_p(ptr)
    return getattr(lib, fn)(p, p, p, p, B, H, T, d_k, d_v, C, dtype, feature, None, None,
                            ws if ws is not None else p, ws_bytes, None)


def test_host_rejects_unsupported_shapes(lib):
    assert _fwd(lib, d_k=24) == L.KATA_ERR_UNSUPPORTED
    assert _fwd(lib, d_k=64) == L.KATA_ERR_UNSUPPORTED          # PSD d_k=64 not built
    assert _fwd(lib, d_v=48) == L.KATA_ERR_UNSUPPORTED
    assert _fwd(lib, C=96) == L.KATA_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=5) == L.KATA_ERR_UNSUPPORTED
    assert _fwd(lib, feature=7) == L.KATA_ERR_UNSUPPORTED
    # the two-factor variants need an even d_k the library builds (16 or 32)
    assert _fwd(lib, feature=L.KATA_FEATURE_MULTI_PSD2, d_k=64) == L.KATA_ERR_UNSUPPORTED
    assert _fwd(lib, feature=L.KATA_FEATURE_SUMMED_PSD2, d_k=24) == L.KATA_ERR_UNSUPPORTED
    assert _fwd(lib, fn="kata_fwd_chunked_sequential", d_k=8) == L.KATA_ERR_UNSUPPORTED
    p = ctypes.c_void_p(256)
    assert lib.kata_fwd_quadratic(p, p, p, p, 1, 1, 8, 24, 64, 1, 0, None) == L.KATA_ERR_UNSUPPORTED
    assert lib.kata_decode_step(p, p, p, p, p, p, 1, 1, 32, 40, 1, 0, None) == L.KATA_ERR_UNSUPPORTED


def test_variant_state_dims(lib):
    assert lib.kata_state_dim(32, L.KATA_FEATURE_MULTI_PSD2) == 2 * 136
    assert lib.kata_state_dim(32, L.KATA_FEATURE_SUMMED_PSD2) == 136
    assert lib.kata_state_dim(16, L.KATA_FEATURE_MULTI_PSD2) == 2 * 36
    assert lib.kata_state_dim(15, L.KATA_FEATURE_SUMMED_PSD2) == 0


def test_delta_host_checks(lib):
    p = ctypes.c_void_p(256)

    def delta(feature=L.KATA_FEATURE_PSD, d_k=32, d_v=64, B=1, ws=p, ws_bytes=256):
        return lib.kata_fwd_delta(p, p, p, p, p, B, 1, 16, d_k, d_v, L.KATA_DTYPE_BF16, feature,
                                  None, None, ws, ws_bytes, None)
    assert delta(feature=L.KATA_FEATURE_FIRST_ORDER) == L.KATA_ERR_UNSUPPORTED
    assert delta(feature=L.KATA_FEATURE_MULTI_PSD2) == L.KATA_ERR_UNSUPPORTED
    assert delta(d_k=24) == L.KATA_ERR_UNSUPPORTED
    assert delta(B=-1) == L.KATA_ERR_INVALID_ARGUMENT
    assert delta(ws=ctypes.c_void_p(0)) == L.KATA_ERR_WORKSPACE
    assert delta(ws_bytes=100) == L.KATA_ERR_WORKSPACE
    assert delta(ws=ctypes.c_void_p(256 + 16)) == L.KATA_ERR_WORKSPACE


def test_backward_rejects_the_variants(lib):
    assert lib.kata_bwd_chunked_workspace_bytes(1, 1, 16, 32, 64, 64, L.KATA_DTYPE_BF16,
                                                L.KATA_FEATURE_MULTI_PSD2) == 0


def test_host_rejects_bad_arguments(lib):
    assert _fwd(lib, B=-1) == L.KATA_ERR_INVALID_ARGUMENT
    assert _fwd(lib, T=-5) == L.KATA_ERR_INVALID_ARGUMENT
    assert _fwd(lib, C=0) == L.KATA_ERR_INVALID_ARGUMENT
    assert _fwd(lib, ws=ctypes.c_void_p(0)) == L.KATA_ERR_WORKSPACE
    assert _fwd(lib, ws=ctypes.c_void_p(256 + 8)) == L.KATA_ERR_WORKSPACE     # unaligned
    p = ctypes.c_void_p(256)
    assert lib.kata_fwd_quadratic(p, p, p, p, -1, 1, 8, 32, 64, 1, 0, None) == L.KATA_ERR_INVALID_ARGUMENT
    assert lib.kata_decode_step(p, p, p, p, p, p, 1, -2, 32, 64, 1, 0, None) == L.KATA_ERR_INVALID_ARGUMENT
    assert lib.kata_workspace_status(None, None) == L.KATA_ERR_WORKSPACE


def _bwd(lib, d_k=32, d_v=64, C=64, dtype=L.KATA_DTYPE_BF16, feature=L.KATA_FEATURE_PSD, B=1, H=1,
         T=16, ws=None):
    p = ctypes.c_void_p(256)
    return lib.kata_bwd_chunked(p, p, p, p, p, p, p, B, H, T, d_k, d_v, C, dtype, feature,
                                ws if ws is not None else p, 1 << 20, None)


def test_backward_host_checks(lib):
    assert _bwd(lib, d_k=24) == L.KATA_ERR_UNSUPPORTED
    assert _bwd(lib, d_k=64) == L.KATA_ERR_UNSUPPORTED           # PSD d_k = 64 not built
    assert _bwd(lib, d_v=48) == L.KATA_ERR_UNSUPPORTED
    assert _bwd(lib, feature=3) == L.KATA_ERR_UNSUPPORTED
    assert _bwd(lib, dtype=5) == L.KATA_ERR_UNSUPPORTED
    assert _bwd(lib, B=-1) == L.KATA_ERR_INVALID_ARGUMENT
    assert _bwd(lib, T=-3) == L.KATA_ERR_INVALID_ARGUMENT
    assert _bwd(lib, C=0) == L.KATA_ERR_INVALID_ARGUMENT
    assert _bwd(lib, ws=ctypes.c_void_p(0)) == L.KATA_ERR_WORKSPACE
    assert _bwd(lib, ws=ctypes.c_void_p(256 + 8)) == L.KATA_ERR_WORKSPACE
    assert lib.kata_bwd_chunked_workspace_bytes(1, 1, 16, 24, 64, 64, 1, 0) == 0
    assert lib.kata_bwd_chunked_workspace_bytes(-1, 1, 16, 32, 64, 64, 1, 0) == 0


def test_state_and_from_state_host_checks(lib):
    p = ctypes.c_void_p(256)
    st = lib.kata_chunked_state
    assert st(p, p, 1, 1, 16, 24, 64, 64, 1, 0, p, p, p, 1 << 20, None) == L.KATA_ERR_UNSUPPORTED
    assert st(p, p, -1, 1, 16, 32, 64, 64, 1, 0, p, p, p, 1 << 20, None) == L.KATA_ERR_INVALID_ARGUMENT
    assert st(p, p, 1, 1, 16, 32, 64, 0, 1, 0, p, p, p, 1 << 20, None) == L.KATA_ERR_INVALID_ARGUMENT
    assert st(p, p, 1, 1, 16, 32, 64, 64, 1, 0, p, p, None, 1 << 20, None) == L.KATA_ERR_WORKSPACE
    fs = lib.kata_fwd_chunked_from_state
    assert fs(p, p, p, p, 1, 1, 16, 24, 64, 64, 1, 0, p, p, p, p, p, 1 << 20, None) == L.KATA_ERR_UNSUPPORTED
    assert fs(p, p, p, p, 1, 1, -2, 32, 64, 64, 1, 0, p, p, p, p, p, 1 << 20, None) == L.KATA_ERR_INVALID_ARGUMENT
    assert fs(p, p, p, p, 1, 1, 16, 32, 64, 64, 1, 0, p, p, p, p, ctypes.c_void_p(264), 1 << 20,
              None) == L.KATA_ERR_WORKSPACE


def test_selftest_rejects_a_missing_or_short_workspace(lib):
    """The device-timeout self-test checks its workspace on the host and
    launches nothing when it is null or shorter than the status header."""
    assert lib.kata_selftest_device_timeout(None, 0, None) == L.KATA_ERR_WORKSPACE
    assert lib.kata_selftest_device_timeout(ctypes.c_void_p(256), 255, None) == L.KATA_ERR_WORKSPACE


def test_empty_problems_launch_nothing(lib):
    p = ctypes.c_void_p(256)
    assert lib.kata_fwd_quadratic(p, p, p, p, 0, 4, 8, 32, 64, 1, 0, None) == L.KATA_OK
    assert lib.kata_fwd_quadratic(p, p, p, p, 2, 4, 0, 32, 64, 1, 0, None) == L.KATA_OK
    assert lib.kata_decode_step(p, p, p, p, p, p, 0, 3, 32, 64, 1, 0, None) == L.KATA_OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    """No CPU fallback: a missing library is an ImportError, not a silent path."""
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        L.lib()
