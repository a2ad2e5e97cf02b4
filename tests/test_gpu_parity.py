"""GPU parity: the CUDA library, called through its C ABI (ctypes binding),
against the fp64 oracle on the same seeded inputs.

Tolerance (per output row, maximised over all compared rows):
    ||y - y_ref||_inf / max(||y_ref||_inf, 1e-6)
    <= 1e-4 for the fp32 path, <= 2e-2 for bf16 inputs with fp32 accumulation.
"""

import numpy as np
import pytest
import torch

import oracle as O
from kernelized_linear_attention_kata_b200 import api
from kernelized_linear_attention_kata_b200 import build as kbuild
from kernelized_linear_attention_kata_b200 import workloads as W
from kernelized_linear_attention_kata_b200._lib import (KATA_ERR_NONPOSITIVE_NORMALISER, KATA_OK,
                                                        KataError)

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
    num = np.max(np.abs(y - ref), axis=-1)
    den = np.maximum(np.max(np.abs(ref), axis=-1), 1e-6)
    return float(np.max(num / den))


def dev(*ts):
    return [t.cuda() for t in ts]


def oracle_heads(fn, q, k, v, *args, **kw):
    return O.per_head(fn, f64(q), f64(k), f64(v), *args, **kw)


def sample_rows(T, C, n, seed):
    r = np.random.default_rng(seed)
    fixed = [0, 1, C - 1, C, T // 2, T - 2, T - 1]
    rows = set(t for t in fixed if 0 <= t < T)
    rows |= set(int(x) for x in r.integers(0, T, size=n))
    return np.array(sorted(rows))


def check_rows(y_gpu, q, k, v, feature, rows, tol, label):
    """Compare sampled rows of every head with the definition at those rows."""
    y = y_gpu.float().cpu().numpy()
    qn, kn, vn = f64(q), f64(k), f64(v)
    B, H = qn.shape[:2]
    worst = 0.0
    for b in range(B):
        for h in range(H):
            ref = O.forward_rows(qn[b, h], kn[b, h], vn[b, h], rows, feature)
            worst = max(worst, rel_err(y[b, h, rows], ref))
    assert worst <= tol, f"{label}: max rel err {worst:.3e} > {tol}"
    return worst


# ---------------------------------------------------------------------------
# Workload 1: tiny fp32 case, every entry point
# ---------------------------------------------------------------------------

def test_tiny_f32_all_forms():
    w = W.TINY
    q, k, v = W.make_inputs(w)
    ref = oracle_heads(O.forward_brute_force, q, k, v, w.feature)
    ref_rec = oracle_heads(O.forward_recurrent_unpacked, q, k, v)
    ref_chk = oracle_heads(O.forward_chunked, q, k, v, w.C, w.feature)
    assert rel_err(ref_rec, ref) < 1e-12 and rel_err(ref_chk, ref) < 1e-12
    qd, kd, vd = dev(q, k, v)
    for seq in (False, True):
        y = api.fwd_chunked(qd, kd, vd, w.C, w.feature, sequential=seq)
        assert rel_err(y.cpu().numpy(), ref) <= TOL["f32"], seq
    y = api.fwd_quadratic(qd, kd, vd, w.feature)
    assert rel_err(y.cpu().numpy(), ref) <= TOL["f32"]
    # decode replay from the zero state, one token at a time
    D = api.state_dim(w.d_k, w.feature)
    S = torch.zeros((1, 1, D, w.d_v), device="cuda")
    z = torch.zeros((1, 1, D), device="cuda")
    ys = []
    for t in range(w.T):
        ys.append(api.decode_step(qd[:, :, t].contiguous(), kd[:, :, t].contiguous(),
                                  vd[:, :, t].contiguous(), S, z, w.feature))
    yd = torch.stack(ys, dim=2).cpu().numpy()
    assert rel_err(yd, ref) <= TOL["f32"]


# ---------------------------------------------------------------------------
# Ragged lengths, every chunk size, every supported (feature, d_k, d_v), both dtypes
# ---------------------------------------------------------------------------

SHAPES = [("psd", 16, 16), ("psd", 16, 64), ("psd", 32, 32), ("psd", 32, 64),
          ("first_order", 16, 16), ("first_order", 32, 64), ("first_order", 64, 64),
          ("first_order", 64, 32)]


@pytest.mark.parametrize("feature,d_k,d_v", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_shapes_ragged(feature, d_k, d_v, dtype):
    for T, C, B, H in ((1, 64, 1, 2), (63, 16, 2, 1), (65, 64, 1, 1), (200, 32, 1, 3),
                       (300, 128, 2, 2), (517, 64, 1, 1)):
        w = W.Workload("ragged", B=B, H=H, T=T, d_k=d_k, d_v=d_v, C=C, dtype=dtype,
                       feature=feature, seed=T * 7 + C, recipe="unit")
        q, k, v = W.make_inputs(w)
        ref = oracle_heads(O.forward_brute_force, q, k, v, feature)
        qd, kd, vd = dev(q, k, v)
        for seq in (False, True):
            y = api.fwd_chunked(qd, kd, vd, C, feature, sequential=seq)
            e = rel_err(y.float().cpu().numpy(), ref)
            assert e <= TOL[dtype], (T, C, seq, e)
        y = api.fwd_quadratic(qd, kd, vd, feature)
        e = rel_err(y.float().cpu().numpy(), ref)
        assert e <= TOL[dtype], (T, "quadratic", e)


# ---------------------------------------------------------------------------
# Workload 2: mid-size bf16, chunked and quadratic, full outputs; final state
# ---------------------------------------------------------------------------

def test_mid_bf16_chunked_quadratic_and_state():
    w = W.MID
    q, k, v = W.make_inputs(w)
    ref, S_ref, z_ref = [], [], []
    qn, kn, vn = f64(q), f64(k), f64(v)
    for b in range(w.B):
        for h in range(w.H):
            y_, S_, z_ = O.forward_chunked(qn[b, h], kn[b, h], vn[b, h], w.C, w.feature,
                                           return_state=True)
            ref.append(y_), S_ref.append(S_), z_ref.append(z_)
    ref = np.stack(ref).reshape(w.B, w.H, w.T, w.d_v)
    qd, kd, vd = dev(q, k, v)
    y, S, z = api.fwd_chunked(qd, kd, vd, w.C, w.feature, return_state=True)
    assert rel_err(y.float().cpu().numpy(), ref) <= TOL["bf16"]
    yq = api.fwd_quadratic(qd, kd, vd, w.feature)
    assert rel_err(yq.float().cpu().numpy(), ref) <= TOL["bf16"]
    # chunked vs quadratic on the GPU (two independent paths)
    assert rel_err(y.float().cpu().numpy(), yq.float().cpu().numpy().astype(np.float64)) <= TOL["bf16"]
    S_ref = np.stack(S_ref).reshape(S.shape)
    z_ref = np.stack(z_ref).reshape(z.shape)
    # this shape runs on the tensor cores, whose update multiplies the feature
    # products k_i k_j rounded to bf16 (relative 2^-9 per term): the state is
    # held to 1e-2 of its largest entry; z comes from K^T K with exact products
    assert np.max(np.abs(S.cpu().numpy() - S_ref)) <= 1e-2 * np.abs(S_ref).max()
    np.testing.assert_allclose(z.cpu().numpy(), z_ref, rtol=1e-4, atol=1e-3)


# ---------------------------------------------------------------------------
# Workload 3: 340M-LM-shaped layer (projected inputs), full outputs
# ---------------------------------------------------------------------------

def test_layer340m_bf16():
    w = W.LAYER
    q, k, v = W.make_inputs(w)
    ref = oracle_heads(O.forward_chunked, q, k, v, w.C, w.feature)
    qd, kd, vd = dev(q, k, v)
    y = api.fwd_chunked(qd, kd, vd, w.C, w.feature)
    assert rel_err(y.float().cpu().numpy(), ref) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# Workload 4: T = 131072 chunked (sampled rows) and the quadratic at 16384
# ---------------------------------------------------------------------------

def test_long131k_chunked_sampled_rows():
    w = W.LONG
    q, k, v = W.make_inputs(w)
    qd, kd, vd = dev(q, k, v)
    y = api.fwd_chunked(qd, kd, vd, w.C, w.feature)
    rows = sample_rows(w.T, w.C, 40, seed=4)
    check_rows(y, q, k, v, w.feature, rows, TOL["bf16"], "long131k chunked")
    # the first 16384 outputs of the causal forward are the 16384-token
    # problem's outputs: compare with the quadratic form on that prefix
    Tq = W.LONG_QUADRATIC_T
    qp, kp, vp = (t[:, :, :Tq].contiguous() for t in (qd, kd, vd))
    yq = api.fwd_quadratic(qp, kp, vp, w.feature)
    rows_q = sample_rows(Tq, w.C, 40, seed=44)
    check_rows(yq, q[:, :, :Tq], k[:, :, :Tq], v[:, :, :Tq], w.feature, rows_q, TOL["bf16"],
               "long quadratic 16k")
    e = rel_err(y[:, :, :Tq].float().cpu().numpy(), yq.float().cpu().numpy().astype(np.float64))
    assert e <= TOL["bf16"], e


# ---------------------------------------------------------------------------
# Workload 5a: first-order feature, scanned carry vs sequential carry
# ---------------------------------------------------------------------------

def test_first_order_scan_and_sequential():
    w = W.FIRST
    q, k, v = W.make_inputs(w)
    qd, kd, vd = dev(q, k, v)
    y = api.fwd_chunked(qd, kd, vd, w.C, w.feature)
    ys = api.fwd_chunked(qd, kd, vd, w.C, w.feature, sequential=True)
    rows = sample_rows(w.T, w.C, 24, seed=5)
    check_rows(y, q, k, v, w.feature, rows, TOL["bf16"], "first-order scanned")
    check_rows(ys, q, k, v, w.feature, rows, TOL["bf16"], "first-order sequential")


# ---------------------------------------------------------------------------
# Workload 5b: batched decode step (batch 256 x 16 heads)
# ---------------------------------------------------------------------------

def test_decode_batch256():
    B, H, d_k, d_v = W.DECODE_BATCH, W.DECODE_HEADS, W.DECODE_DK, W.DECODE_DV
    # One prior state per head, accumulated by the oracle from 4096 seeded
    # tokens and shared by every sequence of the batch.
    kp, vp = W.make_decode_prior_tokens(1, H)
    S1, z1 = [], []
    for h in range(H):
        S_, z_ = O.final_state(f64(kp[0, h]), f64(vp[0, h]), O.PSD)
        S1.append(S_), z1.append(z_)
    S0 = np.broadcast_to(np.stack(S1)[None], (B, H) + S1[0].shape).astype(np.float32)
    z0 = np.broadcast_to(np.stack(z1)[None], (B, H) + z1[0].shape).astype(np.float32)
    q, k, v = W.make_decode_inputs()
    y_ref, S_ref, z_ref = O.decode_step_batched(f64(q), f64(k), f64(v), S0.astype(np.float64),
                                                z0.astype(np.float64))
    S = torch.from_numpy(np.ascontiguousarray(S0)).cuda()
    z = torch.from_numpy(np.ascontiguousarray(z0)).cuda()
    qd, kd, vd = dev(q, k, v)
    y = api.decode_step(qd, kd, vd, S, z)
    assert rel_err(y.float().cpu().numpy(), y_ref) <= TOL["bf16"]
    np.testing.assert_allclose(S.cpu().numpy(), S_ref, rtol=1e-6, atol=1e-4)
    np.testing.assert_allclose(z.cpu().numpy(), z_ref, rtol=1e-6, atol=1e-4)


# ---------------------------------------------------------------------------
# Cross-checks and edge cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_prefill_then_decode_equals_one_call(dtype):
    w = W.Workload("pd", B=2, H=3, T=700, d_k=32, d_v=64, C=64, dtype=dtype, feature="psd",
                   seed=77, recipe="unit")
    q, k, v = dev(*W.make_inputs(w))
    T1 = 650
    y_all = api.fwd_chunked(q, k, v, w.C, w.feature)
    y1, S, z = api.fwd_chunked(q[:, :, :T1].contiguous(), k[:, :, :T1].contiguous(),
                               v[:, :, :T1].contiguous(), w.C, w.feature, return_state=True)
    ys = []
    for t in range(T1, w.T):
        ys.append(api.decode_step(q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                  v[:, :, t].contiguous(), S, z, w.feature))
    y2 = torch.stack(ys, dim=2)
    ref = y_all.float().cpu().numpy().astype(np.float64)
    assert rel_err(torch.cat([y1, y2], dim=2).float().cpu().numpy(), ref) <= TOL[dtype]


def test_nonpositive_normaliser_is_reported():
    w = W.Workload("z", B=1, H=2, T=300, d_k=32, d_v=64, C=64, dtype="bf16", feature="psd",
                   seed=9, recipe="unit")
    q, k, v = dev(*W.make_inputs(w))
    ws = api.alloc_workspace(1, 2, 300, 32, 64, 64)
    o = torch.empty_like(v)
    api.kata_fwd_chunked(q, k, v, o, 64, "psd", workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_OK
    q2 = q.clone()
    q2[0, 1, 200] = 0          # a zero query: every weight of that row is 0
    api.kata_fwd_chunked(q2, k, v, o, 64, "psd", workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_ERR_NONPOSITIVE_NORMALISER
    api.kata_fwd_chunked(q, k, v, o, 64, "psd", workspace=ws)     # status is reset per call
    assert api.kata_workspace_status(ws) == KATA_OK


def test_empty_problems():
    q = torch.empty((1, 2, 0, 32), dtype=torch.bfloat16, device="cuda")
    v = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device="cuda")
    o, S, z = api.fwd_chunked(q, q, v, 64, "psd", return_state=True)
    assert o.shape == v.shape and torch.all(S == 0) and torch.all(z == 0)
    api.fwd_quadratic(q, q, v)
    qb = torch.empty((0, 2, 10, 32), dtype=torch.bfloat16, device="cuda")
    vb = torch.empty((0, 2, 10, 64), dtype=torch.bfloat16, device="cuda")
    api.fwd_chunked(qb, qb, vb, 64)


def test_unsupported_shape_raises():
    q = torch.zeros((1, 1, 8, 24), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises((KataError, ValueError)):
        api.fwd_chunked(q, q, v, 64)


# ---------------------------------------------------------------------------
# Tensor-core chunked path (bf16, PSD, d_k = 32, d_v = 64, C = 128)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,T", [(1, 1, 1), (1, 2, 127), (1, 3, 128), (2, 2, 129), (1, 4, 1000),
                                   (1, 2, 5000), (2, 80, 300)])
def test_tc_chunked_c128_shapes_and_state(B, H, T):
    w = W.Workload("tc", B=B, H=H, T=T, d_k=32, d_v=64, C=128, dtype="bf16", feature="psd",
                   seed=1000 + T + H, recipe="unit")
    q, k, v = W.make_inputs(w)
    qn, kn, vn = f64(q), f64(k), f64(v)
    ref = np.empty((B, H, T, 64))
    S_ref = np.empty((B, H, 528, 64))
    z_ref = np.empty((B, H, 528))
    for b in range(B):
        for h in range(H):
            ref[b, h], S_ref[b, h], z_ref[b, h] = O.forward_chunked(qn[b, h], kn[b, h], vn[b, h], 128,
                                                                    return_state=True)
    qd, kd, vd = dev(q, k, v)
    for seq in (False, True):
        y, S, z = api.fwd_chunked(qd, kd, vd, 128, "psd", return_state=True, sequential=seq)
        e = rel_err(y.float().cpu().numpy(), ref)
        assert e <= TOL["bf16"], (seq, e)
        # the update MMA takes the feature products k_i k_j in bf16 (relative
        # rounding 2^-9 per term); the state is held to 1e-2 of its largest
        # entry. z comes from K^T K with exact fp32 products.
        assert np.max(np.abs(S.cpu().numpy() - S_ref)) <= 1e-2 * np.abs(S_ref).max(), seq
        assert np.max(np.abs(z.cpu().numpy() - z_ref)) <= 1e-4 * np.abs(z_ref).max(), seq


def test_tc_chunked_reports_nonpositive_normaliser():
    w = W.Workload("tcz", B=1, H=2, T=600, d_k=32, d_v=64, C=128, dtype="bf16", feature="psd",
                   seed=8, recipe="unit")
    q, k, v = dev(*W.make_inputs(w))
    ws = api.alloc_workspace(1, 2, 600, 32, 64, 128)
    o = torch.empty_like(v)
    api.kata_fwd_chunked(q, k, v, o, 128, "psd", workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_OK
    q2 = q.clone()
    q2[0, 0, 300] = 0
    api.kata_fwd_chunked(q2, k, v, o, 128, "psd", workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_ERR_NONPOSITIVE_NORMALISER


# ---------------------------------------------------------------------------
# Tensor-core chunked path, first-order feature (bf16, d_k = d_v = 64)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,T,C", [(1, 1, 1, 64), (1, 2, 127, 64), (1, 3, 128, 128), (2, 2, 129, 64),
                                     (1, 4, 1000, 128), (1, 2, 5000, 64), (2, 40, 300, 64)])
def test_tc_first_order_shapes_and_state(B, H, T, C):
    w = W.Workload("tcfo", B=B, H=H, T=T, d_k=64, d_v=64, C=C, dtype="bf16", feature="first_order",
                   seed=2000 + T + H, recipe="unit")
    q, k, v = W.make_inputs(w)
    qn, kn, vn = f64(q), f64(k), f64(v)
    ref = np.empty((B, H, T, 64))
    S_ref = np.empty((B, H, 65, 64))
    z_ref = np.empty((B, H, 65))
    for b in range(B):
        for h in range(H):
            ref[b, h], S_ref[b, h], z_ref[b, h] = O.forward_chunked(
                qn[b, h], kn[b, h], vn[b, h], C, "first_order", return_state=True)
    qd, kd, vd = dev(q, k, v)
    for seq in (False, True):
        y, S, z = api.fwd_chunked(qd, kd, vd, C, "first_order", return_state=True, sequential=seq)
        e = rel_err(y.float().cpu().numpy(), ref)
        assert e <= TOL["bf16"], (seq, e)
        # the state's products of bf16 inputs are exact; only fp32 summation rounds
        assert np.max(np.abs(S.cpu().numpy() - S_ref)) <= 1e-4 * np.abs(S_ref).max(), seq
        assert np.max(np.abs(z.cpu().numpy() - z_ref)) <= 1e-4 * np.abs(z_ref).max(), seq


def test_tc_first_order_reports_nonpositive_normaliser():
    w = W.Workload("tcfoz", B=1, H=1, T=300, d_k=64, d_v=64, C=64, dtype="bf16",
                   feature="first_order", seed=9, recipe="unit")
    q, k, v = dev(*W.make_inputs(w))
    ws = api.alloc_workspace(1, 1, 300, 64, 64, 64, feature="first_order")
    o = torch.empty_like(v)
    api.kata_fwd_chunked(q, k, v, o, 64, "first_order", workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_OK
    # q_0 = -2 k_0 gives the first token the weight 1 + q.k = -1
    q2 = q.clone()
    q2[0, 0, 0] = -2 * k[0, 0, 0]
    api.kata_fwd_chunked(q2, k, v, o, 64, "first_order", workspace=ws)
    assert api.kata_workspace_status(ws) == KATA_ERR_NONPOSITIVE_NORMALISER
