"""Pins for the fp64 oracle of the named KATA variants (oracle/variants.py):
KATA-Mg, KATA-Sigma-g and DeltaKATA. The pages name these variants without
constructing them, so the READINGS are unpinned; what is pinned here is that
each function computes its reading: reductions to the rank-one PSD oracle
(itself pinned in test_oracle_pins.py), closed forms, invariances that tell
the two factor constructions apart, and an independent unpacked
implementation of the delta rule.

Pages cited by title and section:
  [JA]  "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
        Cones", gist.science Japanese explainer: 2.3 (the Mg / Sigma-g
        variants), 4 (delta-rule overwrite), 5 (M1's capacity above M2's).
  [LA]  "線形注意" wiki page, definition.
"""

import numpy as np
import pytest

import oracle as O
from oracle import variants as V


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand(T, d_k, d_v, seed):
    r = np.random.default_rng(seed)
    return unit(r.standard_normal((T, d_k))), unit(r.standard_normal((T, d_k))), \
        r.standard_normal((T, d_v))


# ---------------------------------------------------------------------------
# KATA-Mg and KATA-Sigma-g
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("variant", V.VARIANTS)
def test_one_factor_is_the_rank_one_feature(variant):
    """g = 1: both variants are psi(x) = x x^T, so every form equals the PSD
    oracle."""
    q, k, v = rand(40, 6, 3, seed=1)
    ref = O.forward_brute_force(q, k, v, O.PSD)
    assert np.allclose(V.forward_variant_brute_force(q, k, v, variant, 1), ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(V.forward_variant_recurrent(q, k, v, variant, 1), ref, rtol=1e-11, atol=1e-12)
    assert np.allclose(V.variant_key_feature(k, variant, 1), O.psd_key_feature(k), atol=0)


@pytest.mark.parametrize("variant,g", [(V.MG, 2), (V.MG, 4), (V.SIGMA_G, 2), (V.SIGMA_G, 4)])
def test_feature_inner_product_is_the_frobenius_product(variant, g):
    """phi~(q) . phi(k) equals the Frobenius product of the unpacked factor
    matrices: sum_i <q_i q_i^T, k_i k_i^T> for Mg, <sum_i q_i q_i^T,
    sum_j k_j k_j^T> for Sigma-g, computed here from full outer products (a
    wrong multiplicity or a dropped block fails)."""
    q, k, _ = rand(9, 8, 1, seed=2)
    got = V.variant_query_feature(q, variant, g) @ V.variant_key_feature(k, variant, g).T
    fq, fk = V.factors(q, g), V.factors(k, g)
    want = np.empty((9, 9))
    for t in range(9):
        for s in range(9):
            Qm = [np.outer(fq[t, i], fq[t, i]) for i in range(g)]
            Km = [np.outer(fk[s, i], fk[s, i]) for i in range(g)]
            if variant == V.MG:
                want[t, s] = sum(np.sum(a * b) for a, b in zip(Qm, Km))
            else:
                want[t, s] = np.sum(sum(Qm) * sum(Km))
    assert np.allclose(got, want, rtol=1e-13, atol=1e-14)
    assert np.allclose(V.variant_weights(q, k, variant, g), want, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("variant,g", [(V.MG, 2), (V.MG, 8), (V.SIGMA_G, 2), (V.SIGMA_G, 4)])
def test_recurrent_equals_brute_force(variant, g):
    q, k, v = rand(60, 8, 5, seed=3)
    a = V.forward_variant_brute_force(q, k, v, variant, g)
    b = V.forward_variant_recurrent(q, k, v, variant, g)
    assert np.allclose(a, b, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("variant,g", [(V.MG, 2), (V.SIGMA_G, 2)])
def test_rows_form_equals_brute_force(variant, g):
    """The per-row form (used on long sequences) is the brute force's rows."""
    q, k, v = rand(70, 8, 5, seed=13)
    rows = np.array([0, 1, 2, 33, 68, 69])
    a = V.forward_variant_brute_force(q, k, v, variant, g)[rows]
    b = V.forward_variant_rows(q, k, v, rows, variant, g)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)


def test_state_dims_order_m1_above_m2():
    """Reading 1 gives M1 the largest state at a fixed d_k [JA 5]: 528 rows at
    d_k = 32, 272 for M2 (two 16-wide factors), 136 for Sigma-2."""
    assert V.variant_state_dim(32, V.MG, 1) == O.state_dim(32, O.PSD) == 528
    assert V.variant_state_dim(32, V.MG, 2) == 272
    assert V.variant_state_dim(32, V.SIGMA_G, 2) == 136
    q = unit(np.random.default_rng(4).standard_normal((3, 32)))
    assert V.variant_key_feature(q, V.MG, 2).shape == (3, 272)
    assert V.variant_key_feature(q, V.SIGMA_G, 2).shape == (3, 136)
    with pytest.raises(ValueError):
        V.factors(q, 3)


def test_mg_key_on_one_slice_reduces_to_that_slice():
    """Keys supported on slice j only: the Mg weight is <q_j, k_j>^2, so the
    output is the rank-one PSD oracle run on slice j of q and k."""
    r = np.random.default_rng(5)
    q = unit(r.standard_normal((30, 8)))
    k = np.zeros((30, 8))
    k[:, 4:6] = unit(r.standard_normal((30, 2)))
    v = r.standard_normal((30, 3))
    got = V.forward_variant_brute_force(q, k, v, V.MG, 4)
    ref = O.forward_brute_force(q[:, 4:6], k[:, 4:6], v, O.PSD)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_sigma_g_invariant_to_mixing_a_keys_factors():
    """Psi(k) = F^T F for the g x d' factor matrix F, unchanged by F -> U F
    with U orthogonal: Sigma-g's weights do not move. Mg's do (its factors
    are not summed), which tells the two constructions apart."""
    r = np.random.default_rng(6)
    q, k, _ = rand(12, 12, 1, seed=7)
    U, _ = np.linalg.qr(r.standard_normal((3, 3)))
    F = V.factors(k, 3)
    k_mixed = np.einsum("ij,sjd->sid", U, F).reshape(12, 12)
    assert np.allclose(V.variant_weights(q, k_mixed, V.SIGMA_G, 3),
                       V.variant_weights(q, k, V.SIGMA_G, 3), rtol=1e-12, atol=1e-13)
    assert not np.allclose(V.variant_weights(q, k_mixed, V.MG, 3), V.variant_weights(q, k, V.MG, 3),
                           rtol=1e-3)


def test_mg_invariant_to_permuting_factors_of_both():
    """Permuting the slices of q and k together leaves sum_i <q_i, k_i>^2
    alone; permuting only the keys' slices does not (Sigma-g's sum over all
    pairs does not notice either)."""
    q, k, _ = rand(10, 9, 1, seed=8)
    perm = [2, 0, 1]
    qp = V.factors(q, 3)[:, perm].reshape(10, 9)
    kp = V.factors(k, 3)[:, perm].reshape(10, 9)
    w = V.variant_weights(q, k, V.MG, 3)
    assert np.allclose(V.variant_weights(qp, kp, V.MG, 3), w, rtol=1e-13)
    assert not np.allclose(V.variant_weights(q, kp, V.MG, 3), w, rtol=1e-3)
    assert np.allclose(V.variant_weights(q, kp, V.SIGMA_G, 3), V.variant_weights(q, k, V.SIGMA_G, 3),
                       rtol=1e-13)


def test_sigma_g_with_scalar_factors_is_the_prefix_mean():
    """g = d_k: every factor is a scalar, Psi(x) = |x|^2, so unit q, k give
    equal weights and y_t is the mean of v_0 .. v_t."""
    q, k, v = rand(25, 4, 3, seed=9)
    got = V.forward_variant_brute_force(q, k, v, V.SIGMA_G, 4)
    want = np.cumsum(v, axis=0) / np.arange(1, 26)[:, None]
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    assert np.allclose(V.forward_variant_recurrent(q, k, v, V.SIGMA_G, 4), want, rtol=1e-11,
                       atol=1e-12)


@pytest.mark.parametrize("variant,g", [(V.MG, 2), (V.SIGMA_G, 2)])
def test_variant_outputs_stay_in_the_convex_hull(variant, g):
    """Nonnegative weights that sum to one: each coordinate of y_t lies
    between the smallest and largest v_s, s <= t [LA definition]."""
    q, k, v = rand(50, 8, 4, seed=10)
    y = V.forward_variant_brute_force(q, k, v, variant, g)
    assert np.all(V.variant_weights(q, k, variant, g) >= 0.0)
    lo = np.minimum.accumulate(v, axis=0)
    hi = np.maximum.accumulate(v, axis=0)
    assert np.all(y >= lo - 1e-12) and np.all(y <= hi + 1e-12)


# ---------------------------------------------------------------------------
# DeltaKATA
# ---------------------------------------------------------------------------

def test_delta_packed_equals_unpacked():
    """The packed, normaliser-augmented state and the full d_k x d_k x
    (d_v + 1) state give the same outputs (checks the packing of the
    correction term phi~(k)^T S')."""
    r = np.random.default_rng(11)
    q, k, v = rand(40, 5, 3, seed=12)
    beta = r.uniform(0.2, 1.0, size=40)
    a = V.forward_delta(q, k, v, beta)
    b = V.forward_delta_unpacked(q, k, v, beta)
    assert np.allclose(a, b, rtol=1e-10, atol=1e-11)


def test_delta_with_feature_orthogonal_keys_is_additive():
    """Orthonormal keys e_s (T <= d_k): (k_s . k_t)^2 = 0 for s != t, so the
    correction term is zero and the state is the additive one with weights
    scaled by beta: y_t = sum beta_s w_ts v_s / sum beta_s w_ts; with
    beta = 1 it is the KATA forward itself."""
    r = np.random.default_rng(13)
    T, d_k = 6, 6
    k = np.eye(d_k)[:T]
    q = unit(r.standard_normal((T, d_k)))
    v = r.standard_normal((T, 3))
    assert np.allclose(V.forward_delta(q, k, v, np.ones(T)), O.forward_brute_force(q, k, v, O.PSD),
                       rtol=1e-12, atol=1e-12)
    beta = r.uniform(0.1, 1.0, size=T)
    W = O.weights(q, k, O.PSD) * np.tril(np.ones((T, T))) * beta[None, :]
    want = (W @ v) / W.sum(axis=1)[:, None]
    assert np.allclose(V.forward_delta(q, k, v, beta), want, rtol=1e-12, atol=1e-12)


def test_delta_overwrites_a_repeated_key():
    """Bind v1 to a unit key a, then v2 to another key b, then v3 to a again
    (beta = 1). Right after the third write the binding read at a is exactly
    [v3, 1], so the query a returns v3 [JA 4: delta rules overwrite stale
    bindings]. The additive KATA state would still mix in v1."""
    r = np.random.default_rng(14)
    a, b = unit(r.standard_normal(4)), unit(r.standard_normal(4))
    k = np.stack([a, b, a])
    q = np.stack([a, b, a])
    v = r.standard_normal((3, 2))
    y, Sa = V.forward_delta(q, k, v, np.ones(3), return_state=True)
    assert np.allclose(y[2], v[2], rtol=1e-12, atol=1e-12)
    assert np.allclose(O.psd_query_feature(a) @ Sa, np.append(v[2], 1.0), rtol=1e-12, atol=1e-12)
    additive = O.forward_brute_force(q, k, v, O.PSD)[2]
    assert not np.allclose(additive, v[2], atol=1e-3)


def test_delta_single_repeated_key_returns_the_latest_value():
    """Every token writes to the same unit key with beta = 1: each write
    replaces the last, so y_t = v_t for any query with <q, k> != 0 (KATA
    would give the prefix mean)."""
    r = np.random.default_rng(15)
    key = unit(r.standard_normal(5))
    k = np.tile(key, (20, 1))
    q = unit(r.standard_normal((20, 5)))
    v = r.standard_normal((20, 3))
    assert np.allclose(V.forward_delta(q, k, v, np.ones(20)), v, rtol=1e-10, atol=1e-11)


def test_delta_first_output_is_first_value_and_beta_is_checked():
    q, k, v = rand(1, 4, 2, seed=16)
    assert np.allclose(V.forward_delta(q, k, v, [0.7]), v, rtol=1e-13)
    with pytest.raises(ValueError):
        V.forward_delta(q, k, v, [0.0])
    with pytest.raises(ValueError):
        V.forward_delta(q, k, v, [1.5])


def test_delta_with_a_variant_feature():
    """DeltaKATA on the Mg feature: g = 1 equals DeltaKATA-M1; g = 2 with
    keys on one slice equals DeltaKATA-M1 on that slice."""
    r = np.random.default_rng(17)
    q, k, v = rand(15, 4, 2, seed=18)
    beta = r.uniform(0.3, 1.0, size=15)
    kf = lambda x: V.variant_key_feature(x, V.MG, 1)  # noqa: E731
    qf = lambda x: V.variant_query_feature(x, V.MG, 1)  # noqa: E731
    assert np.allclose(V.forward_delta(q, k, v, beta, kf, qf), V.forward_delta(q, k, v, beta),
                       rtol=1e-12, atol=1e-12)
    k2 = np.zeros_like(k)
    k2[:, :2] = unit(k[:, :2])
    kf2 = lambda x: V.variant_key_feature(x, V.MG, 2)  # noqa: E731
    qf2 = lambda x: V.variant_query_feature(x, V.MG, 2)  # noqa: E731
    got = V.forward_delta(q, k2, v, beta, kf2, qf2)
    ref = V.forward_delta(q[:, :2], k2[:, :2], v, beta)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-11)


def test_planted_mistakes_are_caught(monkeypatch):
    """Each plausible mistake, planted in the variant oracle, makes a pin fail."""
    q, k, _ = rand(9, 8, 1, seed=2)

    # Sigma-g's query side without the off-diagonal multiplicity 2
    real_packed = V._packed
    monkeypatch.setattr(V, "_packed", lambda M, query_side: real_packed(M, False))
    got = V.variant_query_feature(q, V.SIGMA_G, 2) @ V.variant_key_feature(k, V.SIGMA_G, 2).T
    assert not np.allclose(got, V.variant_weights(q, k, V.SIGMA_G, 2), rtol=1e-6)
    monkeypatch.undo()

    # Mg computed with Sigma-g's all-pairs sum: a key on one slice no longer
    # reduces to that slice
    r = np.random.default_rng(5)
    qq = unit(r.standard_normal((30, 8)))
    kk = np.zeros((30, 8))
    kk[:, 4:6] = unit(r.standard_normal((30, 2)))
    vv = r.standard_normal((30, 3))
    real_w = V.variant_weights
    monkeypatch.setattr(V, "variant_weights", lambda a, b, variant, g: real_w(a, b, V.SIGMA_G, g))
    assert not np.allclose(V.forward_variant_brute_force(qq, kk, vv, V.MG, 4),
                           O.forward_brute_force(qq[:, 4:6], kk[:, 4:6], vv, O.PSD), atol=1e-6)
    monkeypatch.undo()

    # DeltaKATA reading the stored binding without the query-side
    # multiplicity: the overwrite at a repeated key is no longer exact
    a, b = unit(r.standard_normal(4)), unit(r.standard_normal(4))
    kd = np.stack([a, b, a])
    vd = r.standard_normal((3, 2))
    y = V.forward_delta(kd, kd, vd, np.ones(3), query_feature=O.psd_key_feature)
    assert not np.allclose(y[2], vd[2], atol=1e-6)


@pytest.mark.parametrize("C", [1, 5, 16, 64, 100])
def test_delta_chunked_equals_recurrent(C):
    """The chunked delta rule (a triangular solve per chunk for the tokens'
    corrections) gives the recurrent rule's outputs and final state, for
    chunk sizes that divide T, leave a ragged tail, or exceed T."""
    r = np.random.default_rng(40 + C)
    q, k, v = rand(70, 6, 3, seed=41)
    beta = r.uniform(0.2, 1.0, size=70)
    y, Sa = V.forward_delta(q, k, v, beta, return_state=True)
    yc, Sc = V.forward_delta_chunked(q, k, v, beta, C, return_state=True)
    assert np.allclose(yc, y, rtol=1e-11, atol=1e-12)
    assert np.allclose(Sc, Sa, rtol=1e-11, atol=1e-12)


def test_delta_chunked_with_other_features():
    """Mg and first-order features through the same chunked form."""
    r = np.random.default_rng(50)
    q, k, v = rand(45, 8, 2, seed=51)
    kf = lambda x: V.variant_key_feature(x, V.MG, 2)  # noqa: E731
    qf = lambda x: V.variant_query_feature(x, V.MG, 2)  # noqa: E731
    beta = r.uniform(0.2, 1.0, size=45)
    assert np.allclose(V.forward_delta_chunked(q, k, v, beta, 8, kf, qf),
                       V.forward_delta(q, k, v, beta, kf, qf), rtol=1e-11, atol=1e-12)
    kf1 = lambda x: O.key_feature(x, O.FIRST_ORDER)  # noqa: E731
    qf1 = lambda x: O.query_feature(x, O.FIRST_ORDER)  # noqa: E731
    beta = r.uniform(0.1, 0.5, size=45)
    assert np.allclose(V.forward_delta_chunked(q, k, v, beta, 8, kf1, qf1),
                       V.forward_delta(q, k, v, beta, kf1, qf1), rtol=1e-11, atol=1e-12)


def test_delta_chunked_planted_diagonal_is_caught(monkeypatch):
    """Counting the token's own key in its correction (tril with the
    diagonal) changes the result."""
    r = np.random.default_rng(60)
    q, k, v = rand(30, 5, 2, seed=61)
    beta = r.uniform(0.2, 1.0, size=30)
    real_tril = np.tril
    monkeypatch.setattr(V.np, "tril", lambda m, k=0: real_tril(m, 0))
    planted = V.forward_delta_chunked(q, k, v, beta, 8)
    monkeypatch.undo()
    assert not np.allclose(planted, V.forward_delta(q, k, v, beta), atol=1e-6)
