"""Python binding of the C ABI: argument marshalling only.

Each function takes CUDA torch tensors, checks their dtype / device /
contiguity, reads the shapes and forwards raw device pointers and sizes to the
entry point of the same name in libkata.so, on the current torch CUDA stream.
Every step of the computation runs in the library's CUDA kernels; PyTorch
only provides device memory and streams.
"""

from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (KATA_DTYPE_BF16, KATA_DTYPE_F32, KATA_FEATURE_FIRST_ORDER, KATA_FEATURE_PSD,
                   check, lib)

_DTYPES = {torch.float32: KATA_DTYPE_F32, torch.bfloat16: KATA_DTYPE_BF16}
_FEATURES = {"psd": KATA_FEATURE_PSD, "first_order": KATA_FEATURE_FIRST_ORDER,
             "mg2": _lib.KATA_FEATURE_MULTI_PSD2, "sigma_g2": _lib.KATA_FEATURE_SUMMED_PSD2}


def _feature(feature: str) -> int:
    try:
        return _FEATURES[feature]
    except KeyError:
        raise ValueError(f"feature must be one of {sorted(_FEATURES)}, got {feature!r}") from None


def _dtype(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16") from None


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _opt(t, name, dtype=torch.float32):
    return None if t is None else _dev(t, name, dtype)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def state_dim(d_k: int, feature: str = "psd") -> int:
    return int(lib().kata_state_dim(d_k, _feature(feature)))


def chunked_workspace_bytes(B, H, T, d_k, d_v, C, dtype=torch.bfloat16, feature="psd") -> int:
    return int(lib().kata_fwd_chunked_workspace_bytes(B, H, T, d_k, d_v, C, _DTYPES[dtype],
                                                      _feature(feature)))


def fwd_chunked_plan(B, H, T, d_k, d_v, C, dtype=torch.bfloat16, feature="psd",
                     sequential=False) -> dict:
    """How kata_fwd_chunked runs this problem on the current device (16-byte
    aligned buffers): {"path", "segments", "segment_tokens", "chunk_tokens"}."""
    p = _lib.KataPlan()
    check("kata_fwd_chunked_plan",
          lib().kata_fwd_chunked_plan(B, H, T, d_k, d_v, C, _DTYPES[dtype], _feature(feature),
                                      1 if sequential else 0, ctypes.byref(p)))
    return {"path": _lib.PATH_NAMES.get(p.path, str(p.path)), "segments": p.segments,
            "segment_tokens": p.segment_tokens, "chunk_tokens": p.chunk_tokens}


def alloc_workspace(B, H, T, d_k, d_v, C, dtype=torch.bfloat16, feature="psd", device=None):
    n = chunked_workspace_bytes(B, H, T, d_k, d_v, C, dtype, feature)
    if n == 0:
        raise ValueError("unsupported shape for kata_fwd_chunked")
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _shapes(q, k, v, o, o_name="o"):
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError(f"expected q, k [B,H,T,d_k] and v [B,H,T,d_v]; got {tuple(q.shape)}, "
                         f"{tuple(k.shape)}, {tuple(v.shape)}")
    if o.shape != v.shape or o.dtype != q.dtype:
        raise ValueError(f"{o_name} must have v's shape and q's dtype")
    if not (k.dtype == v.dtype == q.dtype):
        raise TypeError("q, k, v must share one dtype")
    B, H, T, d_k = q.shape
    return B, H, T, d_k, v.shape[3]


def _state_shapes(B, H, d_k, d_v, feature, S, z, names):
    D = state_dim(d_k, feature)
    if S is not None and tuple(S.shape) != (B, H, D, d_v):
        raise ValueError(f"{names[0]} must be [B,H,{D},{d_v}] fp32")
    if z is not None and tuple(z.shape) != (B, H, D):
        raise ValueError(f"{names[1]} must be [B,H,{D}] fp32")


def kata_fwd_chunked(q, k, v, o, C, feature="psd", S_out=None, z_out=None, workspace=None,
                     stream=None, sequential=False, S0=None, z0=None):
    """Chunked-state causal forward into `o` (see include/kata.h); with S0 / z0
    it starts from that state (kata_fwd_chunked_from_state)."""
    B, H, T, d_k, d_v = _shapes(q, k, v, o)
    _state_shapes(B, H, d_k, d_v, feature, S_out, z_out, ("S_out", "z_out"))
    if workspace is None:
        workspace = alloc_workspace(B, H, T, d_k, d_v, C, q.dtype, feature, q.device)
    ws = (_dev(workspace, "workspace"), workspace.numel() * workspace.element_size())
    if S0 is not None or z0 is not None:
        if sequential:
            raise ValueError("the sequential-carry entry point takes no initial state")
        _state_shapes(B, H, d_k, d_v, feature, S0, z0, ("S0", "z0"))
        fn = "kata_fwd_chunked_from_state"
        st = lib().kata_fwd_chunked_from_state(
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, d_k, d_v, C, _dtype(q),
            _feature(feature), _opt(S0, "S0"), _opt(z0, "z0"), _opt(S_out, "S_out"),
            _opt(z_out, "z_out"), *ws, _stream(stream))
    else:
        fn = "kata_fwd_chunked_sequential" if sequential else "kata_fwd_chunked"
        st = getattr(lib(), fn)(
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, d_k, d_v, C, _dtype(q),
            _feature(feature), _opt(S_out, "S_out"), _opt(z_out, "z_out"), *ws, _stream(stream))
    check(fn, st)
    return o


def kata_chunked_state(k, v, S_out, z_out, C, feature="psd", workspace=None, stream=None):
    """State after all tokens of k, v (no outputs) into S_out, z_out."""
    if k.dim() != 4 or v.dim() != 4 or v.shape[:3] != k.shape[:3] or k.dtype != v.dtype:
        raise ValueError("expected k [B,H,T,d_k] and v [B,H,T,d_v] of one dtype")
    B, H, T, d_k = k.shape
    d_v = v.shape[3]
    _state_shapes(B, H, d_k, d_v, feature, S_out, z_out, ("S_out", "z_out"))
    if workspace is None:
        workspace = alloc_workspace(B, H, T, d_k, d_v, C, k.dtype, feature, k.device)
    st = lib().kata_chunked_state(
        _dev(k, "k"), _dev(v, "v"), B, H, T, d_k, d_v, C, _dtype(k), _feature(feature),
        _opt(S_out, "S_out"), _opt(z_out, "z_out"), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    check("kata_chunked_state", st)
    return S_out, z_out


def kata_fwd_chunked_sequential(q, k, v, o, C, feature="psd", S_out=None, z_out=None,
                                workspace=None, stream=None):
    return kata_fwd_chunked(q, k, v, o, C, feature, S_out, z_out, workspace, stream, sequential=True)


def kata_fwd_quadratic(q, k, v, o, feature="psd", stream=None):
    B, H, T, d_k, d_v = _shapes(q, k, v, o)
    st = lib().kata_fwd_quadratic(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T,
                                  d_k, d_v, _dtype(q), _feature(feature), _stream(stream))
    check("kata_fwd_quadratic", st)
    return o


def kata_decode_step(q, k, v, S, z, y, feature="psd", stream=None):
    """In-place decode step: S, z updated; y [B,H,d_v] written."""
    if q.dim() != 3 or k.shape != q.shape or v.shape[:2] != q.shape[:2] or y.shape != v.shape:
        raise ValueError("expected q, k [B,H,d_k], v, y [B,H,d_v]")
    B, H, d_k = q.shape
    d_v = v.shape[2]
    D = state_dim(d_k, feature)
    if S.shape != (B, H, D, d_v) or z.shape != (B, H, D):
        raise ValueError(f"expected S [B,H,{D},{d_v}] and z [B,H,{D}] fp32")
    st = lib().kata_decode_step(_dev(q, "q"), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype),
                                _dev(S, "S", torch.float32), _dev(z, "z", torch.float32),
                                _dev(y, "y", q.dtype), B, H, d_k, d_v, _dtype(q), _feature(feature),
                                _stream(stream))
    check("kata_decode_step", st)
    return y


def bwd_chunked_workspace_bytes(B, H, T, d_k, d_v, C, dtype=torch.bfloat16, feature="psd") -> int:
    return int(lib().kata_bwd_chunked_workspace_bytes(B, H, T, d_k, d_v, C, _DTYPES[dtype],
                                                      _feature(feature)))


def kata_bwd_chunked(q, k, v, dout, dq, dk, dv, C, feature="psd", workspace=None, stream=None):
    """Gradient of the chunked forward into dq, dk, dv (see include/kata.h)."""
    B, H, T, d_k, d_v = _shapes(q, k, v, dout, "dout")
    if dq.shape != q.shape or dk.shape != k.shape or dv.shape != v.shape:
        raise ValueError("dq, dk, dv must have the shapes of q, k, v")
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} must be {q.dtype}")
    if workspace is None:
        n = bwd_chunked_workspace_bytes(B, H, T, d_k, d_v, C, q.dtype, feature)
        if n == 0:
            raise ValueError("unsupported shape for kata_bwd_chunked")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    st = lib().kata_bwd_chunked(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dq, "dq"),
        _dev(dk, "dk"), _dev(dv, "dv"), B, H, T, d_k, d_v, C, _dtype(q), _feature(feature),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream))
    check("kata_bwd_chunked", st)
    return dq, dk, dv


def kata_fwd_delta(q, k, v, beta, o, feature="psd", S0=None, S_out=None, workspace=None,
                   stream=None):
    """DeltaKATA forward into `o` (see include/kata.h): beta [B, H, T] fp32
    write strengths; S0 / S_out optional [B, H, D, d_v + 1] fp32 states."""
    B, H, T, d_k, d_v = _shapes(q, k, v, o)
    if tuple(beta.shape) != (B, H, T):
        raise ValueError("beta must be [B, H, T] fp32")
    D = state_dim(d_k, feature)
    for t, name in ((S0, "S0"), (S_out, "S_out")):
        if t is not None and tuple(t.shape) != (B, H, D, d_v + 1):
            raise ValueError(f"{name} must be [B, H, {D}, {d_v + 1}] fp32")
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=q.device)
    st = lib().kata_fwd_delta(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
                              _dev(beta, "beta", torch.float32), _dev(o, "o"), B, H, T, d_k, d_v,
                              _dtype(q), _feature(feature), _opt(S0, "S0"), _opt(S_out, "S_out"),
                              _dev(workspace, "workspace"),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    check("kata_fwd_delta", st)
    return o


def fwd_delta(q, k, v, beta, feature="psd", return_state=False, S0=None):
    """(o) or (o, S') of the DeltaKATA forward, allocated with torch."""
    o = torch.empty_like(v)
    S = None
    if return_state:
        B, H, _, d_k = q.shape
        S = torch.empty((B, H, state_dim(d_k, feature), v.shape[3] + 1), dtype=torch.float32,
                        device=q.device)
    kata_fwd_delta(q, k, v, beta, o, feature, S0=S0, S_out=S)
    return (o, S) if return_state else o


def kata_workspace_status(workspace, stream=None) -> int:
    """Synchronises the stream and returns the status code left in the workspace."""
    return int(lib().kata_workspace_status(_dev(workspace, "workspace"), _stream(stream)))


def kata_selftest_device_timeout(workspace, stream=None) -> None:
    """Launch the device-timeout self-test into `workspace` (>= 256 bytes);
    kata_workspace_status(workspace) then reports KATA_ERR_DEVICE_TIMEOUT."""
    st = lib().kata_selftest_device_timeout(_dev(workspace, "workspace"),
                                            workspace.numel() * workspace.element_size(),
                                            _stream(stream))
    check("kata_selftest_device_timeout", st)


def profile_enable(on: bool = True) -> None:
    """Start (and clear) or stop per-kernel CUDA-event timing inside the library."""
    check("kata_profile_enable", lib().kata_profile_enable(1 if on else 0))


def profile_read() -> dict:
    """{kernel name: (launches, total device ms)} since profile_enable(True)."""
    out = {}
    n = lib().kata_profile_count()
    for i in range(n):
        name = ctypes.c_char_p()
        launches = ctypes.c_longlong()
        ms = ctypes.c_double()
        check("kata_profile_get", lib().kata_profile_get(i, ctypes.byref(name), ctypes.byref(launches),
                                                         ctypes.byref(ms)))
        out[name.value.decode()] = (int(launches.value), float(ms.value))
    return out


# Convenience wrappers that allocate the outputs with torch.

def fwd_chunked(q, k, v, C, feature="psd", return_state=False, sequential=False):
    o = torch.empty_like(v)
    if return_state:
        B, H = q.shape[:2]
        D = state_dim(q.shape[3], feature)
        S = torch.empty((B, H, D, v.shape[3]), dtype=torch.float32, device=q.device)
        z = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
        kata_fwd_chunked(q, k, v, o, C, feature, S, z, sequential=sequential)
        return o, S, z
    kata_fwd_chunked(q, k, v, o, C, feature, sequential=sequential)
    return o


def chunked_state(k, v, C, feature="psd"):
    """(S, z): the state after all tokens, allocated with torch."""
    B, H, _, d_k = k.shape
    D = state_dim(d_k, feature)
    S = torch.empty((B, H, D, v.shape[3]), dtype=torch.float32, device=k.device)
    z = torch.empty((B, H, D), dtype=torch.float32, device=k.device)
    return kata_chunked_state(k, v, S, z, C, feature)


def fwd_quadratic(q, k, v, feature="psd"):
    o = torch.empty_like(v)
    return kata_fwd_quadratic(q, k, v, o, feature)


def bwd_chunked(q, k, v, dout, C, feature="psd"):
    """(dq, dk, dv) of sum(dout * y) for y = fwd_chunked(q, k, v)."""
    return kata_bwd_chunked(q, k, v, dout, torch.empty_like(q), torch.empty_like(k),
                            torch.empty_like(v), C, feature)


def decode_step(q, k, v, S, z, feature="psd"):
    y = torch.empty_like(v)
    return kata_decode_step(q, k, v, S, z, y, feature)


__all__ = [
    "state_dim", "chunked_workspace_bytes", "alloc_workspace", "kata_fwd_chunked",
    "kata_fwd_chunked_sequential", "kata_fwd_quadratic", "kata_decode_step",
    "kata_workspace_status", "profile_enable", "profile_read", "fwd_chunked", "fwd_quadratic", "decode_step", "_lib",
    "bwd_chunked_workspace_bytes", "kata_bwd_chunked", "bwd_chunked", "kata_chunked_state",
    "chunked_state", "kata_selftest_device_timeout", "fwd_chunked_plan", "kata_fwd_delta",
    "fwd_delta",
]
