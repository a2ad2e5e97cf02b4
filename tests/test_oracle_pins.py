"""Pins for the fp64 oracle: checks against what the pages and mathematics fix,
not against the oracle's own formulas.

Pages cited by title and section:
  [LA]  "線形注意" wiki page, definition (normalised linear attention).
  [JA]  "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
        Cones", gist.science explainer, technical summary 2.1-2.3.
  [ABS] same title, arXiv 2607.17419v1 abstract.
"""

import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

FORMS_1E12 = 1e-12


def rng(seed=0):
    return np.random.default_rng(seed)


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_head(T, d_k, d_v, seed=0, unit_qk=True):
    r = rng(seed)
    q = r.standard_normal((T, d_k))
    k = r.standard_normal((T, d_k))
    if unit_qk:
        q, k = unit(q), unit(k)
    v = r.standard_normal((T, d_v))
    return q, k, v


def rel_err(y, ref):
    num = np.max(np.abs(y - ref), axis=-1)
    den = np.maximum(np.max(np.abs(ref), axis=-1), 1e-6)
    return float(np.max(num / den))


# ---------------------------------------------------------------------------
# Hand-worked fixtures (tests/golden/hand_worked.txt)
# ---------------------------------------------------------------------------

def _parse_rows(text):
    return [[Fraction(x) for x in row.split()] for row in text.split(";")]


def load_cases(path):
    cases, cur = [], None
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, _, rest = line.partition(" ")
            if key == "case":
                cur = {"name": rest}
            elif key == "end":
                cases.append(cur)
                cur = None
            elif key == "feature":
                cur["feature"] = rest
            elif key == "z":
                cur["z"] = [Fraction(x) for x in rest.split()]
            else:
                cur[key] = _parse_rows(rest)
    return cases


def _as_f64(rows):
    return np.array([[float(x) for x in r] for r in rows])


@pytest.fixture(scope="module")
def hand_cases(golden_dir):
    return load_cases(os.path.join(golden_dir, "hand_worked.txt"))


def test_hand_worked_forward(hand_cases):
    assert len(hand_cases) == 4
    for c in hand_cases:
        q, k, v = _as_f64(c["q"]), _as_f64(c["k"]), _as_f64(c["v"])
        y_ref = _as_f64(c["y"])
        for form in (
            lambda: O.forward_brute_force(q, k, v, c["feature"]),
            lambda: O.forward_recurrent(q, k, v, c["feature"]),
            lambda: O.forward_chunked(q, k, v, 2, c["feature"]),
            lambda: O.forward_chunked_scanned(q, k, v, 1, c["feature"]),
            lambda: O.forward_gated(q, k, v, c["feature"]),
        ):
            np.testing.assert_allclose(form(), y_ref, rtol=0, atol=1e-14, err_msg=c["name"])
        if c["feature"] == O.PSD:
            np.testing.assert_allclose(O.forward_recurrent_unpacked(q, k, v), y_ref, atol=1e-14)


def test_hand_worked_state(hand_cases):
    """Packed state layout, including the order of the (i, j) rows."""
    for c in hand_cases:
        if "S" not in c:
            continue
        q, k, v = _as_f64(c["q"]), _as_f64(c["k"]), _as_f64(c["v"])
        S, z = O.final_state(k, v, c["feature"])
        np.testing.assert_array_equal(S, _as_f64(c["S"]))
        np.testing.assert_array_equal(z, np.array([float(x) for x in c["z"]]))
        _, S2, z2 = O.forward_chunked(q, k, v, 3, c["feature"], return_state=True)
        np.testing.assert_array_equal(S2, S)
        np.testing.assert_array_equal(z2, z)


def test_hand_worked_decode(hand_cases):
    """Decode from the state of the first T-1 tokens reproduces the last row."""
    for c in hand_cases:
        q, k, v = _as_f64(c["q"]), _as_f64(c["k"]), _as_f64(c["v"])
        S, z = O.final_state(k[:-1], v[:-1], c["feature"])
        y, S2, z2 = O.decode_step(q[-1], k[-1], v[-1], S, z, c["feature"])
        np.testing.assert_allclose(y, _as_f64(c["y"])[-1], atol=1e-14)
        if "S" in c:
            np.testing.assert_array_equal(S2, _as_f64(c["S"]))


# ---------------------------------------------------------------------------
# Feature identities [JA 2.2]
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d_k", [1, 2, 3, 16, 32])
def test_trace_identity(d_k):
    """<vec(q q^T), vec(k k^T)> = tr(q q^T k k^T) = (q.k)^2, and the packed
    features reproduce it."""
    r = rng(d_k)
    for _ in range(20):
        q, k = r.standard_normal(d_k), r.standard_normal(d_k)
        frob = float(np.sum(np.outer(q, q) * np.outer(k, k)))
        trace = float(np.trace(np.outer(q, q) @ np.outer(k, k)))
        dot2 = float(np.dot(q, k)) ** 2
        packed = float(O.psd_query_feature(q) @ O.psd_key_feature(k))
        assert abs(frob - dot2) <= 1e-12 * max(1.0, dot2)
        assert abs(trace - dot2) <= 1e-12 * max(1.0, dot2)
        assert abs(packed - dot2) <= 1e-12 * max(1.0, dot2)
        assert abs(O.weights(q[None], k[None], O.PSD)[0, 0] - dot2) <= 1e-12 * max(1.0, dot2)


def test_packed_layout_matches_pairs():
    """Row r of the packed feature is u_i u_j for the r-th (i <= j) pair in
    row-major order -- checked with a plain Python loop."""
    d_k = 5
    u = rng(3).standard_normal(d_k)
    f = O.psd_key_feature(u)
    r = 0
    for i in range(d_k):
        for j in range(i, d_k):
            assert f[r] == u[i] * u[j]
            r += 1
    assert r == O.state_dim(d_k, O.PSD) == len(f)
    assert O.psd_pairs(d_k)[7] == (1, 3)


def test_first_order_feature_identity():
    r = rng(4)
    for _ in range(10):
        q, k = r.standard_normal(7), r.standard_normal(7)
        assert abs(O.first_order_feature(q) @ O.first_order_feature(k) - (1 + q @ k)) < 1e-12
    assert O.state_dim(64, O.FIRST_ORDER) == 65


def test_state_dims():
    assert O.state_dim(32, O.PSD) == 528
    assert O.state_dim(16, O.PSD) == 136


def test_weights_nonnegative():
    """Self-dual cone => nonnegative weights [JA 2.1], including for keys and
    queries with negative inner products."""
    r = rng(5)
    q, k = r.standard_normal((64, 8)), r.standard_normal((64, 8))
    W = O.weights(q, k, O.PSD)
    assert np.all(W >= 0)
    assert np.any((q @ k.T) < 0)        # the inputs did have negative dots
    # first-order: nonnegative for unit vectors (1 + cos >= 0)
    Wf = O.weights(unit(q), unit(k), O.FIRST_ORDER)
    assert np.all(Wf >= -1e-15)


def test_sign_flip_invariance():
    """psi(-u) = psi(u): flipping the sign of any query or key changes nothing."""
    q, k, v = rand_head(40, 6, 3, seed=6)
    y = O.forward_brute_force(q, k, v)
    s = np.where(rng(7).random(40) < 0.5, -1.0, 1.0)[:, None]
    np.testing.assert_allclose(O.forward_brute_force(q * s, k * s[::-1], v), y, rtol=1e-12, atol=1e-13)


def test_rotation_invariance():
    """Isometric invariance [JA 2.1]: a joint orthogonal rotation of q and k
    leaves the output unchanged (both features)."""
    q, k, v = rand_head(50, 8, 4, seed=8)
    R, _ = np.linalg.qr(rng(9).standard_normal((8, 8)))
    for feat in O.FEATURES:
        y = O.forward_chunked(q, k, v, 7, feat)
        y_rot = O.forward_chunked(q @ R.T, k @ R.T, v, 7, feat)
        np.testing.assert_allclose(y_rot, y, rtol=1e-10, atol=1e-12)


def test_query_scale_invariance():
    """Homogeneity: scaling a query by any nonzero factor leaves its PSD output
    unchanged (the weights of row t all scale by the same alpha^2)."""
    q, k, v = rand_head(30, 5, 3, seed=10)
    alpha = rng(11).uniform(0.1, 10.0, size=(30, 1)) * np.where(rng(12).random((30, 1)) < 0.5, -1, 1)
    np.testing.assert_allclose(O.forward_chunked(q * alpha, k, v, 4), O.forward_chunked(q, k, v, 4),
                               rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# Normaliser and gate [JA 2.1, LA]
# ---------------------------------------------------------------------------

def test_convex_hull():
    """Each output coordinate lies between the min and max of the prefix values."""
    for feat in O.FEATURES:
        q, k, v = rand_head(120, 6, 5, seed=13)
        y = O.forward_chunked(q, k, v, 16, feat)
        lo = np.minimum.accumulate(v, axis=0)
        hi = np.maximum.accumulate(v, axis=0)
        assert np.all(y >= lo - 1e-12) and np.all(y <= hi + 1e-12)


def test_weights_sum_to_one():
    """Normalised weights w_ts / den_t sum to 1 over s <= t: with V = the
    identity basis, the outputs are exactly those normalised weights."""
    T = 12
    q, k, _ = rand_head(T, 4, 1, seed=14)
    v = np.eye(T)
    Y = O.forward_chunked(q, k, v, 5)
    np.testing.assert_allclose(Y.sum(axis=1), 1.0, atol=1e-13)
    assert np.all(np.triu(Y, 1) == 0)          # no weight on future tokens
    assert np.all(Y >= 0)


def test_gated_equals_normalised():
    for feat in O.FEATURES:
        q, k, v = rand_head(64, 6, 4, seed=15)
        np.testing.assert_allclose(O.forward_gated(q, k, v, feat),
                                   O.forward_brute_force(q, k, v, feat), rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# Closed forms
# ---------------------------------------------------------------------------

def test_first_output_is_first_value():
    for feat in O.FEATURES:
        q, k, v = rand_head(10, 4, 3, seed=16)
        for fn in (O.forward_brute_force, O.forward_recurrent, O.forward_gated):
            np.testing.assert_allclose(fn(q, k, v, feat)[0], v[0], rtol=1e-14)


def test_equal_keys_give_prefix_mean():
    """All keys equal => every weight in row t equals (q_t.k)^2 => prefix mean."""
    T = 33
    q, _, v = rand_head(T, 5, 4, seed=17)
    k = np.tile(unit(rng(18).standard_normal(5)), (T, 1))
    mean = np.cumsum(v, axis=0) / np.arange(1, T + 1)[:, None]
    for C in (1, 4, 33):
        np.testing.assert_allclose(O.forward_chunked(q, k, v, C), mean, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.forward_brute_force(q, k, v), mean, rtol=1e-12, atol=1e-13)


def test_d1_unit_keys_give_prefix_mean():
    T = 20
    r = rng(19)
    q = r.standard_normal((T, 1))
    k = np.where(r.random((T, 1)) < 0.5, -1.0, 1.0)
    v = r.standard_normal((T, 2))
    mean = np.cumsum(v, axis=0) / np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(O.forward_brute_force(q, k, v), mean, rtol=1e-12)
    np.testing.assert_allclose(O.forward_recurrent(q, k, v), mean, rtol=1e-12)


def test_orthonormal_keys_exact_retrieval():
    """k_s = e_s, q_t = e_j with j <= t => only s = j has weight: y_t = v_j."""
    d = 8
    k = np.eye(d)
    v = rng(20).standard_normal((d, 3))
    r = rng(21)
    js = [int(r.integers(0, t + 1)) for t in range(d)]
    q = np.stack([np.eye(d)[j] for j in js])
    expect = np.stack([v[j] for j in js])
    for fn in (lambda: O.forward_brute_force(q, k, v), lambda: O.forward_recurrent(q, k, v),
               lambda: O.forward_recurrent_unpacked(q, k, v), lambda: O.forward_chunked(q, k, v, 3),
               lambda: O.forward_chunked_scanned(q, k, v, 2)):
        np.testing.assert_allclose(fn(), expect, atol=1e-15)


def test_query_orthogonal_to_history_returns_current_value():
    """q_t orthogonal to every earlier key => y_t = v_t (gate fully open)."""
    d = 6
    T = 5
    r = rng(22)
    k = r.standard_normal((T, d))
    q = r.standard_normal((T, d))
    t = T - 1
    basis, _ = np.linalg.qr(k[:t].T, mode="complete")
    q[t] = basis[:, t]                      # orthogonal to k_0..k_{t-1}
    assert abs(q[t] @ k[t]) > 1e-3
    v = r.standard_normal((T, 2))
    for feat_fn in (O.forward_brute_force, O.forward_gated, lambda a, b, c: O.forward_chunked(a, b, c, 2)):
        np.testing.assert_allclose(feat_fn(q, k, v)[t], v[t], atol=1e-12)


def test_first_order_antipodal_key_has_zero_weight():
    q = unit(rng(23).standard_normal((1, 4)))
    assert abs(O.weights(q, -q, O.FIRST_ORDER)[0, 0]) < 1e-15


def test_nonpositive_denominator_is_an_error():
    q = np.array([[1.0, 0.0]])
    k = np.array([[0.0, 1.0]])
    with pytest.raises(FloatingPointError):
        O.forward_brute_force(q, k, np.ones((1, 1)))


# ---------------------------------------------------------------------------
# Forms agree: brute force = recurrent (unpacked, packed) = chunked (any C,
# ragged) = scanned = gated  ("exact" chunked-state form [ABS])
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 2, 7, 64, 100])
def test_forms_agree_psd(T):
    q, k, v = rand_head(T, 5, 3, seed=30 + T)
    ref = O.forward_brute_force(q, k, v)
    assert rel_err(O.forward_recurrent_unpacked(q, k, v), ref) < FORMS_1E12
    assert rel_err(O.forward_recurrent(q, k, v), ref) < FORMS_1E12
    for C in sorted({1, 2, 3, 5, 8, 16, max(T, 1), T + 3}):
        assert rel_err(O.forward_chunked(q, k, v, C), ref) < FORMS_1E12, C
        assert rel_err(O.forward_chunked_scanned(q, k, v, C), ref) < FORMS_1E12, C


@pytest.mark.parametrize("T", [1, 9, 65])
def test_forms_agree_first_order(T):
    q, k, v = rand_head(T, 6, 4, seed=40 + T)
    ref = O.forward_brute_force(q, k, v, O.FIRST_ORDER)
    assert rel_err(O.forward_recurrent(q, k, v, O.FIRST_ORDER), ref) < FORMS_1E12
    for C in (1, 4, 8, 64):
        assert rel_err(O.forward_chunked(q, k, v, C, O.FIRST_ORDER), ref) < FORMS_1E12
        assert rel_err(O.forward_chunked_scanned(q, k, v, C, O.FIRST_ORDER), ref) < FORMS_1E12


def test_forward_rows_matches_brute_force():
    q, k, v = rand_head(90, 4, 3, seed=50)
    rows = [0, 1, 17, 63, 89]
    np.testing.assert_allclose(O.forward_rows(q, k, v, rows), O.forward_brute_force(q, k, v)[rows],
                               rtol=1e-13)


def test_chunked_state_continuation():
    """Prefill in one call, continue from its returned state in another."""
    q, k, v = rand_head(50, 4, 3, seed=51)
    y_all = O.forward_chunked(q, k, v, 8)
    y1, S, z = O.forward_chunked(q[:21], k[:21], v[:21], 8, return_state=True)
    y2 = O.forward_chunked(q[21:], k[21:], v[21:], 8, S0=S, z0=z)
    np.testing.assert_allclose(np.concatenate([y1, y2]), y_all, rtol=1e-12)


def test_decode_replays_forward():
    for feat in O.FEATURES:
        q, k, v = rand_head(30, 4, 3, seed=52)
        D = O.state_dim(4, feat)
        S, z = np.zeros((D, 3)), np.zeros(D)
        ys = []
        for t in range(30):
            y, S, z = O.decode_step(q[t], k[t], v[t], S, z, feat)
            ys.append(y)
        np.testing.assert_allclose(np.array(ys), O.forward_brute_force(q, k, v, feat), rtol=1e-11)


def test_decode_batched_matches_single():
    r = rng(53)
    B, H, d_k, d_v = 3, 2, 4, 5
    D = O.state_dim(d_k, O.PSD)
    kp = unit(r.standard_normal((B, H, 20, d_k)))
    vp = r.standard_normal((B, H, 20, d_v))
    S = np.einsum("bhtd,bhtv->bhdv", O.psd_key_feature(kp), vp)
    z = O.psd_key_feature(kp).sum(axis=2)
    q, k, v = unit(r.standard_normal((B, H, d_k))), unit(r.standard_normal((B, H, d_k))), r.standard_normal((B, H, d_v))
    y, S2, z2 = O.decode_step_batched(q, k, v, S, z)
    for b in range(B):
        for h in range(H):
            yy, SS, zz = O.decode_step(q[b, h], k[b, h], v[b, h], S[b, h], z[b, h])
            np.testing.assert_allclose(y[b, h], yy, rtol=1e-13)
            np.testing.assert_allclose(S2[b, h], SS, rtol=1e-14)


# ---------------------------------------------------------------------------
# Scan
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 13])
def test_tree_scan_is_exclusive_running_sum(n):
    r = rng(60 + n)
    items = [(r.standard_normal((3, 2)), r.standard_normal(3)) for _ in range(n)]
    out = O.exclusive_tree_scan(items)
    run_S = np.cumsum(np.stack([a for a, _ in items]), axis=0)
    run_z = np.cumsum(np.stack([b for _, b in items]), axis=0)
    assert len(out) == n
    np.testing.assert_array_equal(out[0][0], 0.0)
    for i in range(1, n):
        np.testing.assert_allclose(out[i][0], run_S[i - 1], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(out[i][1], run_z[i - 1], rtol=1e-13, atol=1e-14)


def test_tree_scan_order_insensitive():
    """The combine is +, associative and commutative: permuting the chunks
    permutes the increments but the total is unchanged."""
    r = rng(70)
    items = [(r.standard_normal((4, 3)), r.standard_normal(4)) for _ in range(9)]
    perm = r.permutation(9)
    a = O.exclusive_tree_scan(items)
    b = O.exclusive_tree_scan([items[i] for i in perm])
    tot_a = a[-1][0] + items[-1][0]
    tot_b = b[-1][0] + items[perm[-1]][0]
    np.testing.assert_allclose(tot_a, tot_b, rtol=1e-13)


# ---------------------------------------------------------------------------
# Mistakes planted in the oracle (on the CPU) are caught by the pins above
# ---------------------------------------------------------------------------

def test_planted_mistakes_are_caught(hand_cases, monkeypatch):
    """Each plausible mistake, planted in a copy of a feature map, makes a pin fail."""
    import oracle.kata as K

    case = [c for c in hand_cases if c["name"] == "psd_d3_t4"][0]
    q, k, v = _as_f64(case["q"]), _as_f64(case["k"]), _as_f64(case["v"])
    y_ref = _as_f64(case["y"])

    def no_multiplicity(x):
        iu, ju = np.triu_indices(x.shape[-1])
        return x[..., iu] * x[..., ju]

    monkeypatch.setattr(K, "psd_query_feature", no_multiplicity)
    assert not np.allclose(K.forward_recurrent(q, k, v), y_ref)
    monkeypatch.undo()

    # strict causal mask (diagonal dropped) breaks y_1 = v_1
    def strict_chunked(qq, kk, vv, C, feature=O.PSD):
        T = qq.shape[0]
        W = K.weights(qq, kk, feature) * np.tril(np.ones((T, T)), -1)
        with np.errstate(invalid="ignore", divide="ignore"):
            return (W @ vv) / W.sum(1)[:, None]
    assert not np.allclose(strict_chunked(q, k, v, 4), y_ref, equal_nan=False)

    # swapping the roles of q and k changes the hand-worked values
    assert not np.allclose(K.forward_brute_force(k, q, v), y_ref)
