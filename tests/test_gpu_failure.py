"""Failure detection on the GPU without a fault.

The bounded wait that every tensor-core kernel uses is made to run out: the
self-test kernel waits on an mbarrier that nothing completes. After the
wait's 2 s limit it frees its tensor memory and returns, the host reads
KATA_ERR_DEVICE_TIMEOUT from the workspace, and the same CUDA context then
runs a tensor-core forward that is clean and matches the fp64 oracle. No
trap, assert, invalid address or endless loop is involved.
"""

import numpy as np
import pytest
import torch

import oracle as O
from kernelized_linear_attention_kata_b200 import api
from kernelized_linear_attention_kata_b200 import build as kbuild
from kernelized_linear_attention_kata_b200 import workloads as W
from kernelized_linear_attention_kata_b200._lib import KATA_ERR_DEVICE_TIMEOUT, KATA_OK

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kbuild.build()
    api.lib()


def max_row_rel_err(y, ref):
    y = np.asarray(y, dtype=np.float64).reshape(-1, ref.shape[-1])
    ref = ref.reshape(-1, ref.shape[-1])
    num = np.max(np.abs(y - ref), axis=1)
    den = np.maximum(np.max(np.abs(ref), axis=1), 1e-6)
    return float(np.max(num / den))


def test_device_wait_timeout_is_reported_and_the_context_survives():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    api.kata_selftest_device_timeout(ws)
    end.record()
    assert api.kata_workspace_status(ws) == KATA_ERR_DEVICE_TIMEOUT
    ms = start.elapsed_time(end)
    assert 1900.0 <= ms <= 10000.0, ms      # it waited for the 2 s limit, then returned

    # the context is still usable: a bf16 tensor-core forward runs clean and
    # matches the oracle (B = 1, H = 2, T = 300: three chunks, a ragged tail)
    w = W.Workload("after_timeout", B=1, H=2, T=300, d_k=32, d_v=64, C=128, dtype="bf16",
                   feature="psd", seed=5, recipe="unit")
    q, k, v = W.make_inputs(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.empty_like(vd)
    ws2 = api.alloc_workspace(w.B, w.H, w.T, w.d_k, w.d_v, w.C, qd.dtype, w.feature, qd.device)
    api.kata_fwd_chunked(qd, kd, vd, o, w.C, w.feature, workspace=ws2)
    assert api.kata_workspace_status(ws2) == KATA_OK
    ref = O.per_head(O.forward_brute_force, W.to_f64_numpy(q), W.to_f64_numpy(k),
                     W.to_f64_numpy(v), w.feature)
    assert max_row_rel_err(o.float().cpu().numpy(), ref) <= 2e-2

    # the self-test resets the status word each time
    api.kata_selftest_device_timeout(ws)
    assert api.kata_workspace_status(ws) == KATA_ERR_DEVICE_TIMEOUT
