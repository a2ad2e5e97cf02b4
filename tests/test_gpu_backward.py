"""GPU parity of the gradient of the chunked forward (kata_bwd_chunked),
called through the C ABI, against the fp64 oracle (oracle/backward.py) on the
same seeded inputs.

Tolerance per gradient tensor (dq, dk, dv), measured against the tensor's
largest entry because single gradient rows can cancel to near zero, with a
floor of 1e-3 of the largest entry of the three (a tensor whose exact value
is zero, such as dq at T = 1, is held to that):
    max |g - g_ref| / max(max |g_ref|, 1e-3 max_all |ref|)
        <= 1e-4 (fp32), <= 2e-2 (bf16 inputs, fp32 arithmetic, bf16 outputs).
A single token (T = 1) is the one case whose exact dq and dk are zero by
cancellation: e_00 = g_0 . v_0 + c_0 = g_0 . (v_0 - y_0) with y_0 = v_0, so
fp32 rounding of the two terms, amplified by 1 / d_0, is all that remains.
There dq and dk are held to the size of the cancelling terms,
|dy_0| (|v_0| + |y_0|) / d_0 times |dw/dq| (|dw/dk|).
"""

import numpy as np
import pytest
import torch

import oracle as O
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


def normwise(g, ref, scale_all):
    g = np.asarray(g, dtype=np.float64)
    return float(np.max(np.abs(g - ref)) / max(np.max(np.abs(ref)), 1e-3 * scale_all))


def run_gpu(w):
    q, k, v = W.make_inputs(w)
    dy = W.make_grad_output(w)
    qd, kd, vd, dyd = (t.cuda() for t in (q, k, v, dy))
    dq, dk, dv = api.bwd_chunked(qd, kd, vd, dyd, w.C, w.feature)
    torch.cuda.synchronize()
    return (q, k, v, dy), (dq.float().cpu().numpy(), dk.float().cpu().numpy(),
                           dv.float().cpu().numpy())


# (feature, dtype, B, H, T, d_k, d_v, C): chunk tails, several segments per
# head, one segment per head (B*H >= the SM count), every d_k / d_v built.
CASES = [
    ("psd", "f32", 1, 1, 1, 32, 64, 64),
    ("psd", "f32", 1, 2, 200, 32, 64, 64),
    ("psd", "f32", 2, 3, 257, 16, 16, 16),
    ("psd", "f32", 1, 2, 130, 32, 32, 128),
    ("psd", "bf16", 1, 2, 300, 32, 64, 128),
    ("psd", "bf16", 2, 2, 129, 16, 64, 64),
    ("psd", "bf16", 2, 80, 70, 32, 64, 64),
    # the tensor-core kernels (bf16, d_k = 32, d_v = 64): one-chunk segments
    # with a ragged last chunk, and segments of several chunks
    ("psd", "bf16", 1, 3, 1000, 32, 64, 128),
    ("psd", "bf16", 2, 20, 2000, 32, 64, 128),
    ("psd", "bf16", 1, 1, 1, 32, 64, 128),
    ("psd", "bf16", 1, 2, 129, 32, 64, 64),
    ("first_order", "f32", 1, 1, 1, 64, 64, 64),
    ("first_order", "f32", 1, 2, 191, 64, 64, 64),
    ("first_order", "f32", 2, 2, 100, 16, 32, 32),
    ("first_order", "bf16", 1, 3, 257, 64, 64, 64),
    ("first_order", "bf16", 2, 2, 150, 32, 16, 128),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_oracle(case):
    feature, dtype, B, H, T, d_k, d_v, C = case
    w = W.Workload(f"bwd_{feature}_{dtype}", B=B, H=H, T=T, d_k=d_k, d_v=d_v, C=C, dtype=dtype,
                   feature=feature, seed=100 + T + d_k + d_v, recipe="unit")
    (q, k, v, dy), got = run_gpu(w)
    qn, kn, vn, dyn = f64(q), f64(k), f64(v), f64(dy)
    ref = [np.empty_like(qn), np.empty_like(kn), np.empty_like(vn)]
    for b in range(B):
        for h in range(H):
            for r, x in zip(ref, O.backward_brute_force(qn[b, h], kn[b, h], vn[b, h], dyn[b, h],
                                                        feature)):
                r[b, h] = x
    scale = max(float(np.max(np.abs(r))) for r in ref)
    if T == 1:
        for b in range(B):
            for h in range(H):
                qv, kv, vv, dv0 = qn[b, h, 0], kn[b, h, 0], vn[b, h, 0], dyn[b, h, 0]
                dot = qv @ kv
                w00 = dot * dot if feature == "psd" else 1.0 + dot
                fac = 2.0 * abs(dot) if feature == "psd" else 1.0
                term = np.abs(dv0) @ (2.0 * np.abs(vv)) / w00 * fac
                assert np.max(np.abs(got[0][b, h])) <= TOL[dtype] * term * np.max(np.abs(kv))
                assert np.max(np.abs(got[1][b, h])) <= TOL[dtype] * term * np.max(np.abs(qv))
        assert normwise(got[2], ref[2], scale) <= TOL[dtype]
        return
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        err = normwise(g, r, scale)
        assert err <= TOL[dtype], f"{name}: {err:.3e} > {TOL[dtype]}"


def test_backward_empty_problem():
    q = torch.empty((1, 2, 0, 32), device="cuda", dtype=torch.bfloat16)
    v = torch.empty((1, 2, 0, 64), device="cuda", dtype=torch.bfloat16)
    dq, dk, dv = api.bwd_chunked(q, q, v, v, 64, "psd")
    assert dq.numel() == 0 and dv.numel() == 0


def test_backward_reports_nonpositive_normaliser():
    """First-order weight 1 + q.k with q_0 = -2 k_0 (unit k_0): w_00 = -1."""
    w = W.Workload("bwd_bad", B=1, H=1, T=40, d_k=64, d_v=64, C=64, dtype="f32",
                   feature="first_order", seed=3, recipe="unit")
    q, k, v = (t.cuda() for t in W.make_inputs(w))
    q[0, 0, 0] = -2.0 * k[0, 0, 0]
    dy = W.make_grad_output(w).cuda()
    n = api.bwd_chunked_workspace_bytes(1, 1, 40, 64, 64, 64, torch.float32, "first_order")
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    dq, dk, dv = (torch.empty_like(t) for t in (q, k, v))
    api.kata_bwd_chunked(q, k, v, dy, dq, dk, dv, 64, "first_order", workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_ERR_NONPOSITIVE_NORMALISER
    # a clean problem leaves the status word at zero
    q2, k2, v2 = (t.cuda() for t in W.make_inputs(w))
    api.kata_bwd_chunked(q2, k2, v2, dy, dq, dk, dv, 64, "first_order", workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_OK


def test_backward_long_workload_sampled_rows():
    """The long workload at full size (B = 1, H = 16, T = 131072, bf16, C =
    128), the launch the benchmark times: sampled rows of two heads against
    the oracle's per-row gradient."""
    w = W.LONG
    (q, k, v, dy), (dq, dk, dv) = run_gpu(w)
    rng = np.random.default_rng(17)
    # segment starts of the tensor-core split (9 segments of 114 chunks per
    # head on 148 SMs) and the rows just before them, where the carried
    # prefix and suffix states change hands
    seg = 114 * 128
    bounds = set(x for gi in range(1, 9) for x in (gi * seg - 1, gi * seg))
    rows = np.array(sorted(set([0, 1, 127, 128, 4095, w.T // 2, w.T - 2, w.T - 1]) | bounds
                           | set(int(x) for x in rng.integers(0, w.T, size=24))))
    for h in (0, w.H - 1):
        ref = O.backward_rows(f64(q)[0, h], f64(k)[0, h], f64(v)[0, h], f64(dy)[0, h], rows, w.feature)
        scale = max(float(np.max(np.abs(r))) for r in ref)
        for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            err = normwise(g[0, h, rows], r, scale)
            assert err <= TOL["bf16"], f"head {h} {name}: {err:.3e}"
