"""GPU parity of DeltaKATA (the delta-rule state update the KATA explainer's
section 4 names; the library's reading is stated in include/kata.h) through
the C ABI, against the fp64 oracle of oracle/variants.py (recurrent and
chunked forms) on the same seeded inputs and write strengths.

Tolerances are the forward's (per output row, max relative error): 1e-4 for
fp32, 2e-2 for bf16 inputs (the kernel computes in fp32 either way).
"""

import numpy as np
import pytest
import torch

from oracle import variants as V
from kernelized_linear_attention_kata_b200 import api
from kernelized_linear_attention_kata_b200 import build as kbuild
from kernelized_linear_attention_kata_b200 import workloads as W
from kernelized_linear_attention_kata_b200._lib import KATA_ERR_NONPOSITIVE_NORMALISER, KATA_OK

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
f64 = W.to_f64_numpy


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kbuild.build()
    api.lib()


def rel_err(y, ref):
    y = np.asarray(y, dtype=np.float64)
    return float(np.max(np.max(np.abs(y - ref), -1) / np.maximum(np.max(np.abs(ref), -1), 1e-6)))


def case(B, H, T, d_k, d_v, dtype, seed, recipe="unit"):
    w = W.Workload("delta", B=B, H=H, T=T, d_k=d_k, d_v=d_v, C=64, dtype=dtype, feature="psd",
                   seed=seed, recipe=recipe)
    q, k, v = W.make_inputs(w)
    return q, k, v, W.make_delta_beta(B, H, T, seed)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d_k,d_v", [(16, 16), (32, 64), (32, 32)])
def test_delta_ragged_against_recurrent_oracle(dtype, d_k, d_v):
    """Outputs and final augmented state against the token-by-token rule,
    for lengths below, at and across the kernel's 32-token chunks."""
    for T, B, H in ((1, 1, 2), (31, 2, 1), (32, 1, 1), (33, 1, 3), (200, 2, 2)):
        q, k, v, beta = case(B, H, T, d_k, d_v, dtype, seed=T * 3 + d_k)
        y, S = api.fwd_delta(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), return_state=True)
        qn, kn, vn, bn = f64(q), f64(k), f64(v), beta.double().numpy()
        for b in range(B):
            for h in range(H):
                ref, S_ref = V.forward_delta(qn[b, h], kn[b, h], vn[b, h], bn[b, h],
                                             return_state=True)
                assert rel_err(y[b, h].float().cpu().numpy(), ref) <= TOL[dtype], (T, b, h)
                err = np.max(np.abs(S[b, h].cpu().numpy() - S_ref)) / max(np.max(np.abs(S_ref)), 1e-6)
                assert err <= 1e-4, (T, b, h, err)


def test_delta_continues_from_a_state():
    """Two calls, the second starting from the first's state, equal one call."""
    q, k, v, beta = case(1, 2, 300, 32, 64, "f32", seed=5)
    qd, kd, vd, bd = q.cuda(), k.cuda(), v.cuda(), beta.cuda()
    y, S = api.fwd_delta(qd, kd, vd, bd, return_state=True)
    y1, S1 = api.fwd_delta(qd[:, :, :130].contiguous(), kd[:, :, :130].contiguous(),
                           vd[:, :, :130].contiguous(), bd[:, :, :130].contiguous(), return_state=True)
    y2, S2 = api.fwd_delta(qd[:, :, 130:].contiguous(), kd[:, :, 130:].contiguous(),
                           vd[:, :, 130:].contiguous(), bd[:, :, 130:].contiguous(),
                           return_state=True, S0=S1)
    assert rel_err(torch.cat([y1, y2], dim=2).cpu().numpy(), y.cpu().numpy().astype(np.float64)) <= 1e-5
    assert torch.allclose(S2, S, rtol=1e-5, atol=1e-6)


def test_delta_overwrites_a_repeated_key():
    """beta = 1 at a repeated unit key replaces its binding: querying that key
    right after returns the new value (up to the other keys' interference)."""
    T, d_k, d_v = 64, 32, 64
    q, k, v, beta = case(1, 1, T, d_k, d_v, "f32", seed=17)
    k[0, 0, 40] = k[0, 0, 10]
    q[0, 0, 40] = k[0, 0, 10]
    beta[:] = 1.0
    y = api.fwd_delta(q.cuda(), k.cuda(), v.cuda(), beta.cuda()).cpu().numpy()
    ref = V.forward_delta(f64(q)[0, 0], f64(k)[0, 0], f64(v)[0, 0], beta.double().numpy()[0, 0])
    assert rel_err(y[0, 0], ref) <= 1e-4


def test_delta_mid_bf16_against_chunked_oracle():
    """The mid-size workload's shapes (B=4, H=8, T=4096, d_k=32, d_v=64, V ~
    N(0, 0.5^2)) with seeded write strengths, every head in full, against
    the oracle's chunked delta rule (C = 64)."""
    w = W.MID
    q, k, v = W.make_inputs(w)
    beta = W.make_delta_beta(w.B, w.H, w.T, w.seed)
    y = api.fwd_delta(q.cuda(), k.cuda(), v.cuda(), beta.cuda()).float().cpu().numpy()
    qn, kn, vn, bn = f64(q), f64(k), f64(v), beta.double().numpy()
    for b in range(w.B):
        for h in range(w.H):
            ref = V.forward_delta_chunked(qn[b, h], kn[b, h], vn[b, h], bn[b, h], 64)
            assert rel_err(y[b, h], ref) <= TOL["bf16"], (b, h)


def test_delta_long131k_two_heads():
    """The long workload (T=131072, MQAR-like repeated keys) on all 16 heads;
    two heads in full against the oracle's chunked rule."""
    w = W.LONG
    q, k, v = W.make_inputs(w)
    beta = W.make_delta_beta(w.B, w.H, w.T, w.seed)
    y = api.fwd_delta(q.cuda(), k.cuda(), v.cuda(), beta.cuda()).float().cpu().numpy()
    qn, kn, vn, bn = f64(q), f64(k), f64(v), beta.double().numpy()
    for h in (0, 9):
        ref = V.forward_delta_chunked(qn[0, h], kn[0, h], vn[0, h], bn[0, h], 256)
        assert rel_err(y[0, h], ref) <= TOL["bf16"], h


def test_delta_reports_nonpositive_normaliser_and_rejects_shapes():
    q, k, v, beta = case(1, 1, 40, 32, 64, "f32", seed=3)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(v).cuda()
    api.kata_fwd_delta(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), o, workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_OK
    q2 = q.clone()
    q2[0, 0, 20] = 0
    api.kata_fwd_delta(q2.cuda(), k.cuda(), v.cuda(), beta.cuda(), o, workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_ERR_NONPOSITIVE_NORMALISER
    with pytest.raises(Exception):
        api.fwd_delta(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), feature="first_order")
