"""GPU parity of the state-only call (kata_chunked_state) and of the forward
from a given state (kata_fwd_chunked_from_state), the two entry points of the
sequence-sharded forward, through the C ABI, against the fp64 oracle.

A sequence cut into slices is processed slice by slice as the ranks of the
sequence-sharded forward would: each slice's state from kata_chunked_state,
the carry into slice r = the sum of the states of slices 0 .. r-1, each
slice's outputs from kata_fwd_chunked_from_state. The concatenated outputs
must match the definition on the whole sequence (per-row bound of the
forward: 1e-4 fp32, 2e-2 bf16), and the states the oracle's element by
element, within the bounds of each kernel family's arithmetic
(tests/state_bounds.py).
"""

import numpy as np
import pytest
import torch

import oracle as O
from kernelized_linear_attention_kata_b200 import api
from kernelized_linear_attention_kata_b200 import build as kbuild
from kernelized_linear_attention_kata_b200 import workloads as W
from state_bounds import assert_state_close, tc_psd_path

pytestmark = pytest.mark.gpu

f64 = W.to_f64_numpy


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kbuild.build()
    api.lib()


def rel_rows(y, ref):
    y = np.asarray(y, dtype=np.float64)
    return float(np.max(np.max(np.abs(y - ref), -1) / np.maximum(np.max(np.abs(ref), -1), 1e-6)))


# (feature, dtype, B, H, T, d_k, d_v, C, slice boundaries): the tensor-core
# PSD and first-order paths, the CUDA-core path in fp32 and bf16, ragged
# slices and chunk tails
CASES = [
    ("psd", "bf16", 1, 2, 700, 32, 64, 128, [0, 256, 300, 700]),
    ("psd", "bf16", 2, 3, 513, 32, 64, 64, [0, 129, 513]),
    ("first_order", "bf16", 1, 2, 600, 64, 64, 64, [0, 128, 257, 600]),
    ("psd", "f32", 1, 2, 400, 16, 16, 64, [0, 64, 65, 400]),
    ("psd", "bf16", 1, 1, 300, 16, 32, 32, [0, 100, 300]),
    ("first_order", "f32", 2, 2, 333, 32, 32, 128, [0, 200, 333]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c[:8])))
def test_state_only_matches_oracle(case):
    feature, dtype, B, H, T, d_k, d_v, C, _ = case
    w = W.Workload("state", B=B, H=H, T=T, d_k=d_k, d_v=d_v, C=C, dtype=dtype, feature=feature,
                   seed=500 + T, recipe="unit")
    q, k, v = W.make_inputs(w)
    S, z = api.chunked_state(k.cuda(), v.cuda(), C, feature)
    assert_state_close(S.cpu().numpy(), z.cpu().numpy(), f64(k), f64(v), feature,
                       tc_psd_path(dtype, feature, d_k, d_v, C), "state only")


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c[:8])))
def test_slices_from_carried_state_match_whole_sequence(case):
    feature, dtype, B, H, T, d_k, d_v, C, cuts = case
    w = W.Workload("slices", B=B, H=H, T=T, d_k=d_k, d_v=d_v, C=C, dtype=dtype, feature=feature,
                   seed=600 + T, recipe="unit")
    q, k, v = W.make_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    D = api.state_dim(d_k, feature)
    S0 = torch.zeros((B, H, D, d_v), dtype=torch.float32, device="cuda")
    z0 = torch.zeros((B, H, D), dtype=torch.float32, device="cuda")
    outs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sl = (slice(None), slice(None), slice(a, b))
        qs, ks, vs = (t[sl].contiguous() for t in (qd, kd, vd))
        o = torch.empty_like(vs)
        S_out, z_out = torch.empty_like(S0), torch.empty_like(z0)
        api.kata_fwd_chunked(qs, ks, vs, o, C, feature, S_out=S_out, z_out=z_out, S0=S0, z0=z0)
        outs.append(o)
        # the carry into the next slice, as the sequence-sharded forward forms
        # it: the previous carry plus this slice's own state
        Sl, zl = api.chunked_state(ks, vs, C, feature)
        S0, z0 = S0 + Sl, z0 + zl
        # the forward's own final state and that carry are both the state of
        # tokens 0 .. b - 1 (the carry is a sum of up to len(cuts) - 1
        # separately rounded slice states)
        kb, vb = f64(k[:, :, :b]), f64(v[:, :, :b])
        tc = tc_psd_path(dtype, feature, d_k, d_v, C)
        assert_state_close(S_out.cpu().numpy(), z_out.cpu().numpy(), kb, vb, feature, tc,
                           f"forward's state after token {b}", scale=float(len(cuts)))
        assert_state_close(S0.cpu().numpy(), z0.cpu().numpy(), kb, vb, feature, tc,
                           f"carry after token {b}", scale=float(len(cuts)))
    y = torch.cat(outs, dim=2).float().cpu().numpy()
    ref = O.per_head(O.forward_brute_force, f64(q), f64(k), f64(v), feature)
    tol = 1e-4 if dtype == "f32" else 2e-2
    assert rel_rows(y, ref) <= tol



def test_from_state_with_no_tokens_returns_the_state():
    D = api.state_dim(32, "psd")
    S0 = torch.randn((1, 2, D, 64), device="cuda")
    z0 = torch.rand((1, 2, D), device="cuda")
    q = torch.empty((1, 2, 0, 32), device="cuda", dtype=torch.bfloat16)
    v = torch.empty((1, 2, 0, 64), device="cuda", dtype=torch.bfloat16)
    S_out, z_out = torch.empty_like(S0), torch.empty_like(z0)
    api.kata_fwd_chunked(q, q, v, torch.empty_like(v), 64, "psd", S_out=S_out, z_out=z_out,
                         S0=S0, z0=z0)
    torch.cuda.synchronize()
    assert torch.equal(S_out, S0) and torch.equal(z_out, z0)


def test_sequence_parallel_on_one_rank_is_the_plain_forward():
    """Without a process group there is one slice and a zero carry. The state
    (one MMA issuer) is bitwise the plain forward's; the outputs agree to
    rounding: two issuers accumulate the readout into one accumulator, in an
    order that varies from run to run."""
    from kernelized_linear_attention_kata_b200 import sequence_parallel as SP
    w = W.Workload("sp1", B=1, H=2, T=300, d_k=32, d_v=64, C=128, dtype="bf16", feature="psd",
                   seed=71, recipe="unit")
    q, k, v = (t.cuda() for t in W.make_inputs(w))
    o_sp, S_sp, z_sp = SP.fwd_chunked_sequence_parallel(q, k, v, w.C, w.feature, return_state=True)
    o, S, z = api.fwd_chunked(q, k, v, w.C, w.feature, return_state=True)
    torch.cuda.synchronize()
    assert torch.equal(S_sp, S) and torch.equal(z_sp, z)
    a, b = o_sp.float(), o.float()
    row_err = (a - b).abs().amax(-1) / b.abs().amax(-1).clamp_min(1e-6)
    assert float(row_err.max()) <= 8e-3          # two bf16 rounding steps
