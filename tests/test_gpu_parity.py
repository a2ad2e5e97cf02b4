"""GPU parity: the CUDA library, called through its C ABI (ctypes binding),
against the fp64 oracle on the same seeded inputs.

Tolerance (per output row, maximised over all compared rows):
    ||y - y_ref||_inf / max(||y_ref||_inf, 1e-6)
    <= 1e-4 for the fp32 path, <= 2e-2 for bf16 inputs with fp32 accumulation.
"""

import os

import numpy as np
import pytest
import torch

import oracle as O
from kernelized_linear_attention_kata_b200 import api
from kernelized_linear_attention_kata_b200 import build as kbuild
from kernelized_linear_attention_kata_b200 import workloads as W
from kernelized_linear_attention_kata_b200._lib import (KATA_ERR_NONPOSITIVE_NORMALISER, KATA_OK,
                                                        KataError)
from state_bounds import assert_state_close, tc_psd_path

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


def sample_rows(T, C, n, seed, extra=()):
    r = np.random.default_rng(seed)
    fixed = [0, 1, C - 1, C, T // 2, T - 2, T - 1, *extra]
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
    qn, kn, vn = f64(q), f64(k), f64(v)
    ref = O.per_head(O.forward_chunked, qn, kn, vn, w.C, w.feature)
    qd, kd, vd = dev(q, k, v)
    y, S, z = api.fwd_chunked(qd, kd, vd, w.C, w.feature, return_state=True)
    assert rel_err(y.float().cpu().numpy(), ref) <= TOL["bf16"]
    yq = api.fwd_quadratic(qd, kd, vd, w.feature)
    assert rel_err(yq.float().cpu().numpy(), ref) <= TOL["bf16"]
    # chunked vs quadratic on the GPU (two independent paths)
    assert rel_err(y.float().cpu().numpy(), yq.float().cpu().numpy().astype(np.float64)) <= TOL["bf16"]
    # element by element, within the bounds of the tensor-core path's
    # arithmetic (bf16 key products, fp32 accumulation; tests/state_bounds.py)
    assert_state_close(S.cpu().numpy(), z.cpu().numpy(), kn, vn, w.feature,
                       tc_psd_path(w.dtype, w.feature, w.d_k, w.d_v, w.C), "mid_bf16")


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
    # the rows on either side of every segment boundary of the parallel carry
    # (where a segment's carry-in starts), beside random rows
    plan = api.fwd_chunked_plan(w.B, w.H, w.T, w.d_k, w.d_v, w.C, q.dtype, w.feature)
    assert plan["segments"] > 1, plan
    seg = plan["segment_tokens"]
    bounds = [g * seg + d for g in range(1, plan["segments"]) for d in (-1, 0, 1)]
    rows = sample_rows(w.T, w.C, 40, seed=4, extra=bounds)
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

def oracle_prior_states(kp, vp):
    """The oracle's state (S, z) of every sequence's own prior tokens, kp
    [B, H, n, d_k], vp [B, H, n, d_v] (device tensors, copied to the host one
    sequence at a time), computed on host threads."""
    from concurrent.futures import ThreadPoolExecutor
    B, H = kp.shape[:2]
    D = O.state_dim(kp.shape[3], O.PSD)
    S0 = np.empty((B, H, D, vp.shape[3]))
    z0 = np.empty((B, H, D))

    def one(b):
        kn, vn = f64(kp[b]), f64(vp[b])
        for h in range(H):
            S0[b, h], z0[b, h] = O.final_state(kn[h], vn[h], O.PSD)

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(one, range(B)))
    return S0, z0


def test_decode_batch256():
    B, H, d_k, d_v = W.DECODE_BATCH, W.DECODE_HEADS, W.DECODE_DK, W.DECODE_DV
    # A distinct prior state for every (sequence, head): the oracle's state of
    # that sequence's own 4096 seeded tokens (the tokens are drawn on the
    # device, as the benchmark draws them, and read back for the oracle).
    kp, vp = W.make_decode_prior_tokens(B, H, device="cuda")
    S0, z0 = oracle_prior_states(kp, vp)
    del kp, vp
    q, k, v = W.make_decode_inputs()
    y_ref, S_ref, z_ref = O.decode_step_batched(f64(q), f64(k), f64(v), S0, z0)
    S = torch.from_numpy(S0.astype(np.float32)).cuda()
    z = torch.from_numpy(z0.astype(np.float32)).cuda()
    qd, kd, vd = dev(q, k, v)
    y = api.decode_step(qd, kd, vd, S, z)
    assert rel_err(y.float().cpu().numpy(), y_ref) <= TOL["bf16"]
    # the step adds one fp32 term (exact bf16 products) to the fp32-rounded
    # prior: two roundings of the entry
    S_np, z_np = S.cpu().numpy(), z.cpu().numpy()
    assert np.all(np.abs(S_np - S_ref) <= 2 * 2.0 ** -24 * np.abs(S_ref) + 1e-30 +
                  2.0 ** -24 * np.abs(S0)), np.max(np.abs(S_np - S_ref))
    assert np.all(np.abs(z_np - z_ref) <= 2 * 2.0 ** -24 * np.abs(z_ref) + 1e-30 +
                  2.0 ** -24 * np.abs(z0)), np.max(np.abs(z_np - z_ref))
    # the batch is not one state broadcast: sequences differ
    assert not np.allclose(S_ref[0], S_ref[1])


# ---------------------------------------------------------------------------
# Which kernels run: the five workloads' forms on the families the plan names
# ---------------------------------------------------------------------------

FAMILY_PREFIX = {"tensor_core_psd": "tc_segment_", "tensor_core_first_order": "tc_fo_",
                 "cuda_core": "simt_"}


@pytest.mark.parametrize("name,path", [("tiny_f32", "cuda_core"), ("mid_bf16", "tensor_core_psd"),
                                       ("layer340m_bf16", "tensor_core_psd"),
                                       ("long131k_bf16", "tensor_core_psd"),
                                       ("first_order64k_bf16", "tensor_core_first_order")])
def test_workload_runs_on_its_kernel_family(name, path):
    """The plan query names the family, and the library's per-kernel profiler
    sees only that family's kernels run (the family is a function of the
    shape; the sequence is shortened to keep the test small)."""
    w = W.WORKLOADS[name]
    plan = api.fwd_chunked_plan(w.B, w.H, w.T, w.d_k, w.d_v, w.C, w.torch_dtype, w.feature)
    assert plan["path"] == path, plan
    ws = w.with_T(min(w.T, 4096))
    q, k, v = W.make_inputs(ws, device="cuda")
    assert api.fwd_chunked_plan(ws.B, ws.H, ws.T, ws.d_k, ws.d_v, ws.C, ws.torch_dtype,
                                ws.feature)["path"] == path
    api.profile_enable(True)
    try:
        api.fwd_chunked(q, k, v, ws.C, ws.feature)
        prof = api.profile_read()
    finally:
        api.profile_enable(False)
    assert prof and all(n.startswith(FAMILY_PREFIX[path]) for n in prof), prof


def test_decode_runs_on_its_kernel():
    q, k, v = W.make_decode_inputs(batch=4, device="cuda")
    D = api.state_dim(W.DECODE_DK)
    S = torch.zeros((4, W.DECODE_HEADS, D, W.DECODE_DV), device="cuda")
    z = torch.ones((4, W.DECODE_HEADS, D), device="cuda")
    api.profile_enable(True)
    try:
        api.decode_step(q, k, v, S, z)
        prof = api.profile_read()
    finally:
        api.profile_enable(False)
    assert set(prof) == {"simt_decode"}, prof


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
                                   (1, 2, 5000), (2, 80, 300), (1, 1, 150 * 128 + 5)])
def test_tc_chunked_c128_shapes_and_state(B, H, T):
    """Tensor-core PSD path against the oracle, outputs and state. The last
    shape has segments of two chunks whose increments are cut into pieces."""
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
        # element by element within the tensor-core path's arithmetic (bf16
        # key products, fp32 accumulation; tests/state_bounds.py)
        assert_state_close(S.cpu().numpy(), z.cpu().numpy(), kn, vn, "psd", True,
                           f"tc c128 seq={seq}")


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
        # the state's products of bf16 inputs are exact; only fp32 summation
        # rounds: element by element (tests/state_bounds.py)
        assert_state_close(S.cpu().numpy(), z.cpu().numpy(), kn, vn, "first_order", False,
                           f"tc first-order seq={seq}")


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
