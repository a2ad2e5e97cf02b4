"""Pins for the fp64 gradient oracle (oracle/backward.py): central finite
differences of the forward definition, and identities that the definition
fixes, not the oracle's own formulas.

Pages cited by title and section:
  [LA]  "線形注意" wiki page, definition (normalised linear attention).
  [JA]  "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
        Cones", gist.science explainer, technical summary 2.1-2.2 (weights
        <q, k>^2, the normaliser as a convex gate).
"""

import numpy as np
import pytest

import oracle as O


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_head(T, d_k, d_v, seed):
    r = np.random.default_rng(seed)
    q = unit(r.standard_normal((T, d_k)))
    k = unit(r.standard_normal((T, d_k)))
    v = r.standard_normal((T, d_v))
    dy = r.standard_normal((T, d_v))
    return q, k, v, dy


def loss(q, k, v, dy, feature):
    return float(np.sum(dy * O.forward_brute_force(q, k, v, feature)))


@pytest.mark.parametrize("feature", O.FEATURES)
def test_central_finite_differences(feature):
    """Every entry of dq, dk, dv against (L(x + h) - L(x - h)) / 2h, where L is
    the forward definition contracted with dy: a dropped term, a wrong sign,
    a missing factor 2 or a transposed operand all fail here."""
    q, k, v, dy = rand_head(7, 3, 2, seed=11)
    dq, dk, dv = O.backward_brute_force(q, k, v, dy, feature)
    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (loss(args_p["q"], args_p["k"], args_p["v"], dy, feature)
                       - loss(args_m["q"], args_m["k"], args_m["v"], dy, feature)) / (2 * h)
        scale = max(np.max(np.abs(fd)), 1e-3)
        assert np.max(np.abs(fd - grad)) <= 1e-7 * scale, name


@pytest.mark.parametrize("feature", O.FEATURES)
def test_single_token(feature):
    """T = 1: y_1 = v_1 whatever q, k are (the only weight normalises to 1), so
    dq = dk = 0 and dv = dy."""
    q, k, v, dy = rand_head(1, 4, 3, seed=2)
    dq, dk, dv = O.backward_brute_force(q, k, v, dy, feature)
    assert np.allclose(dq, 0.0, atol=1e-14)
    assert np.allclose(dk, 0.0, atol=1e-14)
    assert np.allclose(dv, dy, rtol=0, atol=1e-14)


@pytest.mark.parametrize("feature", O.FEATURES)
def test_normalisation_and_linearity_in_v(feature):
    """The normalised weights of each row sum to one [LA; JA 2.1], so adding a
    common vector to every v_s adds it to every y_t: sum_s dv_s = sum_t dy_t.
    y is linear in v: sum_s v_s . dv_s = sum_t y_t . dy_t."""
    q, k, v, dy = rand_head(50, 6, 5, seed=3)
    dq, dk, dv = O.backward_brute_force(q, k, v, dy, feature)
    assert np.allclose(dv.sum(axis=0), dy.sum(axis=0), rtol=1e-12, atol=1e-12)
    y = O.forward_brute_force(q, k, v, feature)
    assert np.isclose(np.sum(v * dv), np.sum(y * dy), rtol=1e-12, atol=1e-12)


def test_psd_homogeneity():
    """w = <q, k>^2 [JA 2.2]: scaling one query by a leaves its row of weights
    scaled by a^2, which the normaliser cancels, so q_t . dq_t = 0 for every t;
    scaling every key by b scales every weight by b^2, so sum_s k_s . dk_s = 0."""
    q, k, v, dy = rand_head(40, 5, 4, seed=4)
    dq, dk, dv = O.backward_brute_force(q, k, v, dy, O.PSD)
    assert np.max(np.abs(np.sum(q * dq, axis=1))) <= 1e-12 * max(np.max(np.abs(dq)), 1.0)
    assert abs(np.sum(k * dk)) <= 1e-11 * max(np.max(np.abs(dk)), 1.0)


def test_psd_sign_flip_of_a_key():
    """psi(-u) = psi(u): flipping one key leaves y unchanged, so that key's
    gradient flips sign and every other gradient stays."""
    q, k, v, dy = rand_head(12, 4, 3, seed=5)
    dq, dk, dv = O.backward_brute_force(q, k, v, dy, O.PSD)
    k2 = k.copy()
    k2[5] = -k2[5]
    dq2, dk2, dv2 = O.backward_brute_force(q, k2, v, dy, O.PSD)
    assert np.allclose(dk2[5], -dk[5], atol=1e-13)
    assert np.allclose(np.delete(dk2, 5, 0), np.delete(dk, 5, 0), atol=1e-13)
    assert np.allclose(dq2, dq, atol=1e-13) and np.allclose(dv2, dv, atol=1e-13)


def prefix_mean_dv(dy):
    """y_t = mean(v_0 .. v_t) gives dv_s = sum_{t >= s} dy_t / (t + 1)."""
    T = dy.shape[0]
    coef = 1.0 / np.arange(1, T + 1)
    return np.cumsum((dy * coef[:, None])[::-1], axis=0)[::-1]


def test_psd_equal_keys():
    """All keys equal: every causal weight of row t is the same, y_t is the
    prefix mean of v, independent of q (dq = 0)."""
    q, k, v, dy = rand_head(30, 4, 3, seed=6)
    k[:] = k[0]
    dq, dk, dv = O.backward_brute_force(q, k, v, dy, O.PSD)
    assert np.allclose(dq, 0.0, atol=1e-12)
    assert np.allclose(dv, prefix_mean_dv(dy), rtol=1e-12, atol=1e-12)


def test_first_order_zero_queries():
    """First-order feature with q = 0: every weight is 1, y_t is the prefix
    mean of v, and dw/dk = q = 0 gives dk = 0."""
    q, k, v, dy = rand_head(30, 4, 3, seed=7)
    q[:] = 0.0
    dq, dk, dv = O.backward_brute_force(q, k, v, dy, O.FIRST_ORDER)
    assert np.allclose(dk, 0.0, atol=1e-14)
    assert np.allclose(dv, prefix_mean_dv(dy), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("feature", O.FEATURES)
def test_rows_form_matches_brute_force(feature):
    """The per-row form (prefix-sum normalisers, one O(T) sum per row) agrees
    with the O(T^2) form."""
    q, k, v, dy = rand_head(45, 6, 5, seed=8)
    ref = O.backward_brute_force(q, k, v, dy, feature)
    rows = [0, 1, 7, 22, 44]
    got = O.backward_rows(q, k, v, dy, rows, feature)
    for a, b in zip(got, ref):
        assert np.allclose(a, b[rows], rtol=1e-11, atol=1e-12)
