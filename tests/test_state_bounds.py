"""The element-wise state bounds of the GPU parity tests (tests/state_bounds.py),
checked on the CPU against a numpy emulation of the arithmetic they model:
they must accept that arithmetic and reject the mistakes they exist to catch
(a mis-scaled diagonal or off-diagonal feature, a dropped token)."""

import numpy as np
import torch

import oracle as O
from kernelized_linear_attention_kata_b200 import workloads as W
from state_bounds import assert_state_close


def bf16(x):
    """Round fp64/fp32 values to bf16 (round to nearest even), back as fp64."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def emulated_tc_state(k, v):
    """The bf16 tensor-core PSD path's state: key products k_i k_j rounded to
    bf16, products with v exact, accumulated in fp32 token by token."""
    iu, ju = np.triu_indices(k.shape[1])
    S = np.zeros((iu.size, v.shape[1]), dtype=np.float32)
    z = np.zeros(iu.size, dtype=np.float32)
    for t in range(k.shape[0]):
        p = bf16(k[t, iu] * k[t, ju]).astype(np.float32)
        S += p[:, None] * v[t][None, :].astype(np.float32)
        z += (k[t, iu] * k[t, ju]).astype(np.float32)
    return S, z


def inputs(T, seed):
    w = W.Workload("b", B=1, H=1, T=T, d_k=32, d_v=64, C=128, dtype="bf16", feature="psd",
                   seed=seed, recipe="unit")
    _, k, v = W.make_inputs(w)
    return W.to_f64_numpy(k), W.to_f64_numpy(v)


def check(S, z, kn, vn):
    assert_state_close(S[None, None], z[None, None], kn, vn, "psd", True)


def test_bound_accepts_emulated_tensor_core_arithmetic():
    for T, seed in ((1, 1), (300, 2), (2000, 3)):
        kn, vn = inputs(T, seed)
        S, z = emulated_tc_state(kn[0, 0], vn[0, 0])
        check(S, z, kn, vn)


def test_bound_rejects_planted_mistakes():
    kn, vn = inputs(2000, 4)
    S, z = emulated_tc_state(kn[0, 0], vn[0, 0])
    diag = [i * 32 - i * (i - 1) // 2 for i in range(32)]       # packed rows (i, i)
    for mistake in ("diag_x2", "offdiag_x2", "drop_token"):
        S2, z2 = S.copy(), z.copy()
        if mistake == "diag_x2":
            S2[diag[7]] *= 2
        elif mistake == "offdiag_x2":
            S2[diag[7] + 3] *= 2
        else:
            S2, _ = emulated_tc_state(kn[0, 0, 1:], vn[0, 0, 1:])
        try:
            check(S2, z2, kn, vn)
        except AssertionError:
            continue
        raise AssertionError(f"the state bound let {mistake} through")
