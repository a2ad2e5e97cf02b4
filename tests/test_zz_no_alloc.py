"""kata_fwd_chunked_noalloc: the chunked forward for callers that cannot
allocate device memory (their device memory belongs to another runtime's
pool, or they must not trigger the synchronisation cudaMalloc can cause).

Called through the C ABI and compared with kata_fwd_chunked (the caller-
workspace entry point) on the same inputs, on two calls in a row, because
every call reuses the library's one fixed scratch array. This file sorts last
so that a run stopping at its first failure has run everything else first.
"""

import ctypes

import numpy as np
import pytest
import torch

from kernelized_linear_attention_kata_b200 import api
from kernelized_linear_attention_kata_b200 import build as kbuild
from kernelized_linear_attention_kata_b200 import workloads as W
from kernelized_linear_attention_kata_b200._lib import (KATA_DTYPE_BF16, KATA_ERR_WORKSPACE,
                                                        KATA_FEATURE_PSD, KATA_OK, lib)

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
SCRATCH_BYTES = 32 * 1024 * 1024


def rel_err(y, ref):
    num = np.max(np.abs(y - ref), axis=-1)
    den = np.maximum(np.max(np.abs(ref), axis=-1), 1e-6)
    return float(np.max(num / den))


def call_noalloc(q, k, v, o, C, S=None, z=None):
    B, H, T, d_k = q.shape
    d_v = v.shape[3]
    return lib().kata_fwd_chunked_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), B, H, T, d_k, d_v, C,
        KATA_DTYPE_BF16, KATA_FEATURE_PSD, None if S is None else S.data_ptr(),
        None if z is None else z.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_entry_point_twice():
    assert torch.cuda.is_available()
    kbuild.build()
    # 4 heads leave room for many segments per head, so the segment
    # increments (the scratch) are really used.
    w = W.Workload("noalloc", B=1, H=4, T=4000, d_k=32, d_v=64, C=64, dtype="bf16",
                   feature="psd", seed=21, recipe="unit")
    assert api.chunked_workspace_bytes(w.B, w.H, w.T, w.d_k, w.d_v, w.C) > 1 << 20
    q, k, v = (t.cuda() for t in W.make_inputs(w))
    ref, S_ref, z_ref = api.fwd_chunked(q, k, v, w.C, w.feature, return_state=True)
    ref = ref.float().cpu().numpy().astype(np.float64)
    for call in range(2):
        o = torch.full_like(v, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        z = torch.full_like(z_ref, float("nan"))
        assert call_noalloc(q, k, v, o, w.C, S, z) == KATA_OK
        torch.cuda.synchronize()
        assert rel_err(o.float().cpu().numpy(), ref) <= TOL_BF16, call
        torch.testing.assert_close(S, S_ref, rtol=1e-5, atol=1e-4)
        torch.testing.assert_close(z, z_ref, rtol=1e-5, atol=1e-4)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 256 heads, one segment each: 256 x 528 x 65 fp32 > 32 MiB
    B, H, T = 4, 64, 64
    need = api.chunked_workspace_bytes(B, H, T, 32, 64, 64)
    assert need > SCRATCH_BYTES
    p = ctypes.c_void_p(256)
    st = lib().kata_fwd_chunked_noalloc(p, p, p, p, B, H, T, 32, 64, 64, KATA_DTYPE_BF16,
                                        KATA_FEATURE_PSD, None, None, None)
    assert st == KATA_ERR_WORKSPACE
