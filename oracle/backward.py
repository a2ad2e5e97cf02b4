"""Plain fp64 CPU oracle for the gradient of the KATA causal forward.

TEST INFRASTRUCTURE, like ``oracle.kata``: read only by the tests, the smoke
check and the benchmark's CPU legs; the CUDA library never imports it.

The forward is normalised causal linear attention [LA definition; ABS]:

    y_t = n_t / d_t,   n_t = sum_{s<=t} w_ts v_s,   d_t = sum_{s<=t} w_ts,

with w_ts = <q_t, k_s>^2 for the rank-one PSD feature [JA 2.2, IT 2.2] or
1 + <q_t, k_s> for the first-order reading of the abstract's scanned feature.
The pages pre-train 340M-parameter language models on these kernels [ABS;
JA 3 and 4, IT 3 and 4] but print no backward pass; the gradient here is the
chain rule of the definition above, written out. For an upstream gradient
dy (dL/dy_t), with

    g_t = dy_t / d_t               (d_v vector)
    c_t = -(dy_t . y_t) / d_t      (scalar: dL/dd_t)
    e_ts = g_t . v_s + c_t         (dL/dw_ts, for s <= t)

the gradients are

    dv_s = sum_{t>=s} w_ts g_t
    dq_t = sum_{s<=t} e_ts dw_ts/dq_t,   dk_s = sum_{t>=s} e_ts dw_ts/dk_s

where dw/dq = 2 <q, k> k and dw/dk = 2 <q, k> q (PSD), or k and q
(first-order). Pinned in tests/test_oracle_backward.py by central finite
differences of ``forward_brute_force`` and by closed forms.
"""

from __future__ import annotations

import numpy as np

from .kata import FIRST_ORDER, PSD, _check_den, key_feature, query_feature, weights


def _weight_grad_factor(g: np.ndarray, feature: str) -> np.ndarray:
    """dw/d<q,k> as a function of the dot product g = <q, k>."""
    if feature == PSD:
        return 2.0 * g
    if feature == FIRST_ORDER:
        return np.ones_like(g)
    raise ValueError(f"unknown feature {feature!r}")


def backward_brute_force(q, k, v, dy, feature=PSD):
    """(dq, dk, dv) of L = sum_t dy_t . y_t from the definition, O(T^2).

    One head: q, k [T, d_k], v, dy [T, d_v], float64.
    """
    T = q.shape[0]
    mask = np.tril(np.ones((T, T)))                # s <= t, diagonal included
    dots = q @ k.T                                  # <q_t, k_s>
    W = weights(q, k, feature) * mask
    den = W.sum(axis=1)
    _check_den(den)
    y = (W @ v) / den[:, None]
    g = dy / den[:, None]
    c = -np.sum(dy * y, axis=1) / den
    E = (g @ v.T + c[:, None]) * mask               # dL/dw_ts
    dv = W.T @ g
    F = E * _weight_grad_factor(dots, feature)      # dL/d<q_t, k_s>
    dq = F @ k
    dk = F.T @ q
    return dq, dk, dv


def backward_rows(q, k, v, dy, rows, feature=PSD):
    """dq, dk, dv of ``backward_brute_force`` at the given rows only.

    For sequences too long for the O(T^2) form: the normalisers d_t and the
    outputs y_t of every token come from the packed-state recurrence
    (prefix sums of phi(k_s) and phi(k_s) v_s^T, the RNN view of [LA]); each
    requested row is then one O(T) sum of the formulas in the module
    docstring.
    """
    rows = np.asarray(rows, dtype=np.int64)
    fk = key_feature(k, feature)
    fq = query_feature(q, feature)
    z = np.cumsum(fk, axis=0)                       # z_t = sum_{s<=t} phi(k_s)
    den = np.einsum("td,td->t", fq, z)
    _check_den(den)
    S = np.zeros((fk.shape[1], v.shape[1]))
    y = np.empty_like(v)
    for t in range(q.shape[0]):
        S += np.outer(fk[t], v[t])
        y[t] = (fq[t] @ S) / den[t]
    g = dy / den[:, None]
    c = -np.sum(dy * y, axis=1) / den
    dq = np.empty((len(rows), q.shape[1]))
    dk = np.empty((len(rows), k.shape[1]))
    dv = np.empty((len(rows), v.shape[1]))
    for n, r in enumerate(rows):
        # query row r: keys s <= r
        dots = k[:r + 1] @ q[r]
        e = v[:r + 1] @ g[r] + c[r]
        dq[n] = (e * _weight_grad_factor(dots, feature)) @ k[:r + 1]
        # key row r: queries t >= r
        dots = q[r:] @ k[r]
        w = weights(q[r:], k[r:r + 1], feature)[:, 0]
        e = g[r:] @ v[r] + c[r:]
        dk[n] = (e * _weight_grad_factor(dots, feature)) @ q[r:]
        dv[n] = w @ g[r:]
    return dq, dk, dv
