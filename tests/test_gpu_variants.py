"""GPU parity of the two-factor KATA variants (KATA-Mg and KATA-Sigma-g with
g = 2; the explainer's section 2.3 names them, the library reads their
factors as the two halves of a head vector) through the C ABI, against the
fp64 oracle of oracle/variants.py on the same seeded inputs.

Tolerances are the forward's (per output row, max relative error): 1e-4 for
fp32, 2e-2 for bf16 inputs with fp32 accumulation. States are compared
element by element within the fp32 accumulation bound of the CUDA-core
kernels (tests/state_bounds.py).
"""

import numpy as np
import pytest
import torch

from oracle import variants as V
from kernelized_linear_attention_kata_b200 import api
from kernelized_linear_attention_kata_b200 import build as kbuild
from kernelized_linear_attention_kata_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
f64 = W.to_f64_numpy
# library feature name -> oracle reading (g = 2)
VARIANTS = {"mg2": V.MG, "sigma_g2": V.SIGMA_G}


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kbuild.build()
    api.lib()


def rel_err(y, ref):
    y = np.asarray(y, dtype=np.float64)
    return float(np.max(np.max(np.abs(y - ref), -1) / np.maximum(np.max(np.abs(ref), -1), 1e-6)))


def oracle(fn, q, k, v, *args):
    qn, kn, vn = f64(q), f64(k), f64(v)
    B, H = qn.shape[:2]
    return np.stack([np.stack([fn(qn[b, h], kn[b, h], vn[b, h], *args) for h in range(H)])
                     for b in range(B)])


def inputs(B, H, T, d_k, d_v, dtype, seed):
    w = W.Workload("variant", B=B, H=H, T=T, d_k=d_k, d_v=d_v, C=64, dtype=dtype, feature="psd",
                   seed=seed, recipe="unit")
    return W.make_inputs(w)


@pytest.mark.parametrize("feature", sorted(VARIANTS))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d_k,d_v", [(16, 16), (32, 64)])
def test_variant_forms_ragged(feature, dtype, d_k, d_v):
    """Chunked (scan and sequential carry), quadratic and decode replay
    against the definition, ragged lengths and every chunk size."""
    variant = VARIANTS[feature]
    for T, C, B, H in ((1, 64, 1, 2), (63, 16, 2, 1), (200, 32, 1, 3), (300, 128, 2, 2), (517, 64, 1, 1)):
        q, k, v = inputs(B, H, T, d_k, d_v, dtype, seed=T * 11 + C + d_k)
        ref = oracle(V.forward_variant_brute_force, q, k, v, variant, 2)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        for seq in (False, True):
            y = api.fwd_chunked(qd, kd, vd, C, feature, sequential=seq)
            assert rel_err(y.float().cpu().numpy(), ref) <= TOL[dtype], (T, C, seq)
        y = api.fwd_quadratic(qd, kd, vd, feature)
        assert rel_err(y.float().cpu().numpy(), ref) <= TOL[dtype], (T, "quadratic")
        if T <= 200:
            D = api.state_dim(d_k, feature)
            S = torch.zeros((B, H, D, d_v), device="cuda")
            z = torch.zeros((B, H, D), device="cuda")
            ys = [api.decode_step(qd[:, :, t].contiguous(), kd[:, :, t].contiguous(),
                                  vd[:, :, t].contiguous(), S, z, feature) for t in range(T)]
            yd = torch.stack(ys, dim=2).float().cpu().numpy()
            assert rel_err(yd, ref) <= TOL[dtype], (T, "decode")


@pytest.mark.parametrize("feature", sorted(VARIANTS))
def test_variant_state_layout(feature):
    """The returned state is the oracle's packed state, element by element
    (fp32 CUDA-core path: accumulation bound only)."""
    variant = VARIANTS[feature]
    B, H, T, d_k, d_v = 1, 2, 700, 32, 64
    q, k, v = inputs(B, H, T, d_k, d_v, "f32", seed=91)
    y, S, z = api.fwd_chunked(q.cuda(), k.cuda(), v.cuda(), 64, feature, return_state=True)
    qn, kn, vn = f64(q), f64(k), f64(v)
    for h in range(H):
        _, S_ref, z_ref = V.forward_variant_recurrent(qn[0, h], kn[0, h], vn[0, h], variant, 2,
                                                      return_state=True)
        _, S_abs, z_abs = V.forward_variant_recurrent(qn[0, h], np.abs(kn[0, h]), np.abs(vn[0, h]),
                                                      variant, 2, return_state=True)
        bound = (T + 8) * 2.0 ** -23
        assert np.all(np.abs(S[0, h].cpu().numpy() - S_ref) <= bound * S_abs + 1e-30), h
        assert np.all(np.abs(z[0, h].cpu().numpy() - z_ref) <= bound * z_abs + 1e-30), h
    assert S.shape[2] == V.variant_state_dim(d_k, variant, 2)


@pytest.mark.parametrize("feature", sorted(VARIANTS))
def test_variant_mid_bf16(feature):
    """The mid-size workload's shapes (B=4, H=8, T=4096, d_k=32, d_v=64,
    C=64, V ~ N(0, 0.5^2)): two heads in full, sampled rows of every head,
    and the chunked form against the quadratic form on the GPU."""
    variant = VARIANTS[feature]
    w = W.MID
    q, k, v = W.make_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    y = api.fwd_chunked(qd, kd, vd, w.C, feature).float().cpu().numpy()
    ref2 = oracle(V.forward_variant_brute_force, q[:1, :2], k[:1, :2], v[:1, :2], variant, 2)
    assert rel_err(y[:1, :2], ref2) <= TOL["bf16"]
    rows = np.array(sorted({0, 1, 63, 64, 2047, 4094, 4095} |
                           set(np.random.default_rng(7).integers(0, w.T, 24).tolist())))
    qn, kn, vn = f64(q), f64(k), f64(v)
    for b in range(w.B):
        for h in range(w.H):
            ref = V.forward_variant_rows(qn[b, h], kn[b, h], vn[b, h], rows, variant, 2)
            assert rel_err(y[b, h, rows], ref) <= TOL["bf16"], (b, h)
    yq = api.fwd_quadratic(qd, kd, vd, feature).float().cpu().numpy()
    assert rel_err(y, yq.astype(np.float64)) <= TOL["bf16"]


@pytest.mark.parametrize("feature", sorted(VARIANTS))
def test_variant_long131k_sampled_rows(feature):
    """The long workload's shapes (B=1, H=16, T=131072, C=128, MQAR-like
    inputs), sampled rows of every head against the definition."""
    variant = VARIANTS[feature]
    w = W.LONG
    q, k, v = W.make_inputs(w)
    y = api.fwd_chunked(q.cuda(), k.cuda(), v.cuda(), w.C, feature).float().cpu().numpy()
    plan = api.fwd_chunked_plan(w.B, w.H, w.T, w.d_k, w.d_v, w.C, q.dtype, feature)
    seg = plan["segment_tokens"]
    rows = {0, 1, 127, 128, w.T // 2, w.T - 1}
    rows |= {g * seg + d for g in range(1, plan["segments"]) for d in (-1, 0)}
    rows |= set(np.random.default_rng(8).integers(0, w.T, 12).tolist())
    rows = np.array(sorted(t for t in rows if 0 <= t < w.T))
    qn, kn, vn = f64(q), f64(k), f64(v)
    for h in range(w.H):
        ref = V.forward_variant_rows(qn[0, h], kn[0, h], vn[0, h], rows, variant, 2)
        assert rel_err(y[0, h, rows], ref) <= TOL["bf16"], h


def test_variant_backward_is_rejected():
    q = torch.zeros((1, 1, 8, 32), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Exception):
        api.bwd_chunked(q, q, v, v, 64, "mg2")


@pytest.mark.parametrize("feature", sorted(VARIANTS))
def test_variant_kernel_family(feature):
    """bf16 with d_k = 32, d_v = 64 and C in {64, 128} runs on the tensor
    cores; fp32, other chunk sizes and other shapes on the CUDA cores."""
    def path(dtype, d_k, d_v, C):
        return api.fwd_chunked_plan(1, 16, 131072, d_k, d_v, C, dtype, feature)["path"]
    assert path(torch.bfloat16, 32, 64, 128) == "tensor_core_multi_factor"
    assert path(torch.bfloat16, 32, 64, 64) == "tensor_core_multi_factor"
    assert path(torch.float32, 32, 64, 128) == "cuda_core"
    assert path(torch.bfloat16, 32, 64, 32) == "cuda_core"
    assert path(torch.bfloat16, 16, 16, 64) == "cuda_core"


@pytest.mark.parametrize("feature", sorted(VARIANTS))
def test_variant_tc_state_and_continuation(feature):
    """The tensor-core path's returned state, element by element, and a
    sequence processed in two calls (the second from the first's state)
    against the definition on the whole sequence.

    State bound per entry: fp32 accumulation of T terms, (T + 8) 2^-23
    sum_t |a_t|, plus one bf16 rounding (unit roundoff 2^-8) of each key
    feature entering the update MMA, at most 2^-8 sum_t |a_t|; z is formed
    from exact products (Z = K^T K) and gets the accumulation term only."""
    variant = VARIANTS[feature]
    B, H, T, T1, d_k, d_v = 1, 3, 700, 300, 32, 64
    q, k, v = inputs(B, H, T, d_k, d_v, "bf16", seed=131)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    y, S, z = api.fwd_chunked(qd, kd, vd, 128, feature, return_state=True)
    ref = oracle(V.forward_variant_brute_force, q, k, v, variant, 2)
    assert rel_err(y.float().cpu().numpy(), ref) <= TOL["bf16"]
    qn, kn, vn = f64(q), f64(k), f64(v)
    for h in range(H):
        _, S_ref, z_ref = V.forward_variant_recurrent(qn[0, h], kn[0, h], vn[0, h], variant, 2,
                                                      return_state=True)
        _, S_abs, z_abs = V.forward_variant_recurrent(qn[0, h], np.abs(kn[0, h]), np.abs(vn[0, h]),
                                                      variant, 2, return_state=True)
        acc = (T + 8) * 2.0 ** -23
        assert np.all(np.abs(S[0, h].cpu().numpy() - S_ref) <= (acc + 2.0 ** -8) * S_abs + 1e-30), h
        assert np.all(np.abs(z[0, h].cpu().numpy() - z_ref) <= acc * z_abs + 1e-30), h
    # two calls: tokens [0, T1), then [T1, T) from the first call's state
    y1, S1, z1 = api.fwd_chunked(qd[:, :, :T1].contiguous(), kd[:, :, :T1].contiguous(),
                                 vd[:, :, :T1].contiguous(), 128, feature, return_state=True)
    y2 = torch.empty_like(vd[:, :, T1:])
    S2 = torch.empty_like(S)
    z2 = torch.empty_like(z)
    api.kata_fwd_chunked(qd[:, :, T1:].contiguous(), kd[:, :, T1:].contiguous(),
                         vd[:, :, T1:].contiguous(), y2, 64, feature, S_out=S2, z_out=z2,
                         S0=S1, z0=z1)
    yy = torch.cat([y1, y2], dim=2).float().cpu().numpy()
    assert rel_err(yy, ref) <= TOL["bf16"]
    assert torch.allclose(S2, S, rtol=1e-3, atol=1e-3 * float(S.abs().max()))
    assert torch.allclose(z2, z, rtol=1e-5, atol=1e-5 * float(z.abs().max()))
