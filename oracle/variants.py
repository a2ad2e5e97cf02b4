"""fp64 oracle for the KATA variants the pages name without constructing:
KATA-Mg (multiple PSD factors), KATA-Sigma-g (summed PSD factors) and
DeltaKATA (a delta-rule state update).

TEST INFRASTRUCTURE, under the same rules as oracle/kata.py: read by the tests
only; the CUDA library never imports it. Every function works on one head:
q, k [T, d_k], v [T, d_v], float64.

What the pages fix, restated:

* The framework has two variants that trade state size against packing
  efficiency: one with several PSD factors (Mg) and one whose PSD factors are
  added (Sigma-g) [JA 2.3, IT 2.3].
* KATA-M1 has the larger theoretical capacity, yet KATA-M2 can do better in
  training [JA 5, IT 5]; the linear-state M2 kernel is the fast one at 131k
  tokens [JA 4, IT 4].
* Variants with a delta rule (DeltaKATA) correct stale bindings at repeated
  keys and overwrite almost perfectly [JA 4, IT 4].

Readings (the pages give no construction; the PARITY OF EACH READING IS
UNPINNED, while the arithmetic of each is pinned by
tests/test_oracle_variants.py):

1. The g factors of a head vector x in R^{d_k} are its g contiguous equal
   slices x_1 .. x_g in R^{d'}, d' = d_k / g. With g = 1 both variants are
   the rank-one PSD feature psi(x) = x x^T. Of the plain constructions, only
   slices give M1 the larger state at a given d_k (d_k(d_k+1)/2 rows against
   g d'(d'+1)/2) and so the larger capacity; separate full-width factors
   would give M2 twice M1's state.
2. KATA-Mg keeps one PSD factor per slice, phi(x) = [psi(x_1), .., psi(x_g)],
   so the weight is sum_i <q_i, k_i>^2 and the state has g d'(d'+1)/2 rows
   (each block packed like the rank-one feature, blocks in slice order).
3. KATA-Sigma-g adds the factors, Psi(x) = sum_i x_i x_i^T, so the weight is
   <Psi(q), Psi(k)>_F = sum_{i,j} <q_i, k_j>^2 and the state has d'(d'+1)/2
   rows.
4. DeltaKATA applies the delta rule to the state augmented with its
   normaliser, S' = [S | z] (D x (d_v + 1)):
       S'_t = S'_{t-1} + beta_t phi(k_t) ([v_t, 1] - phi~(k_t)^T S'_{t-1}),
       y_t  = (phi~(q_t)^T S'_t)[:d_v] / (phi~(q_t)^T S'_t)[d_v],
   with phi the key-side and phi~ the query-side packed feature (so that
   phi~(a) . phi(b) is the weight between a and b), beta_t in (0, 1] a given
   per-token write strength, and the read after the update (as in the
   additive forward). For a unit key phi~(k) . phi(k) = |k|^4 = 1, so
   beta = 1 makes phi~(k)^T S' equal [v, 1] right after the write: the
   binding at a repeated key is overwritten exactly. When the keys are
   orthogonal in feature space the correction term vanishes and the rule is
   the additive KATA state with weights scaled by beta.
"""

from __future__ import annotations

import numpy as np

from .kata import _check_den, psd_key_feature, psd_pairs, psd_query_feature

MG = "mg"
SIGMA_G = "sigma_g"
VARIANTS = (MG, SIGMA_G)


def factors(x: np.ndarray, g: int) -> np.ndarray:
    """The g contiguous equal slices of the last axis: [..., d_k] -> [..., g, d_k / g]
    (reading 1)."""
    d_k = x.shape[-1]
    if g < 1 or d_k % g:
        raise ValueError(f"g = {g} does not divide d_k = {d_k}")
    return x.reshape(x.shape[:-1] + (g, d_k // g))


def variant_state_dim(d_k: int, variant: str, g: int) -> int:
    """State rows: g d'(d'+1)/2 for Mg, d'(d'+1)/2 for Sigma-g, d' = d_k / g."""
    if g < 1 or d_k % g:
        raise ValueError(f"g = {g} does not divide d_k = {d_k}")
    dp = d_k // g
    if variant == MG:
        return g * dp * (dp + 1) // 2
    if variant == SIGMA_G:
        return dp * (dp + 1) // 2
    raise ValueError(f"unknown variant {variant!r}")


def _packed(M: np.ndarray, query_side: bool) -> np.ndarray:
    """Upper triangle (i <= j, row-major) of symmetric [..., d, d] matrices;
    the query side doubles the off-diagonal entries."""
    d = M.shape[-1]
    out = np.stack([M[..., i, j] * (2.0 if (query_side and i < j) else 1.0)
                    for i, j in psd_pairs(d)], axis=-1)
    return out


def variant_key_feature(x: np.ndarray, variant: str, g: int) -> np.ndarray:
    """Key-side packed feature of Mg (reading 2) or Sigma-g (reading 3)."""
    f = factors(x, g)
    if variant == MG:
        return np.concatenate([psd_key_feature(f[..., i, :]) for i in range(g)], axis=-1)
    if variant == SIGMA_G:
        return _packed(np.einsum("...ia,...ib->...ab", f, f), query_side=False)
    raise ValueError(f"unknown variant {variant!r}")


def variant_query_feature(x: np.ndarray, variant: str, g: int) -> np.ndarray:
    """Query-side packed feature (off-diagonal multiplicity 2 folded in)."""
    f = factors(x, g)
    if variant == MG:
        return np.concatenate([psd_query_feature(f[..., i, :]) for i in range(g)], axis=-1)
    if variant == SIGMA_G:
        return _packed(np.einsum("...ia,...ib->...ab", f, f), query_side=True)
    raise ValueError(f"unknown variant {variant!r}")


def variant_weights(q: np.ndarray, k: np.ndarray, variant: str, g: int) -> np.ndarray:
    """W[t, s] in closed form: sum_i <q_i, k_i>^2 (Mg), sum_{i,j} <q_i, k_j>^2
    (Sigma-g)."""
    fq, fk = factors(q, g), factors(k, g)
    if variant == MG:
        G = np.einsum("tia,sia->tsi", fq, fk)           # <q_t,i , k_s,i>
        return np.sum(G * G, axis=-1)
    if variant == SIGMA_G:
        G = np.einsum("tia,sja->tsij", fq, fk)          # <q_t,i , k_s,j>
        return np.sum(G * G, axis=(-2, -1))
    raise ValueError(f"unknown variant {variant!r}")


def forward_variant_brute_force(q, k, v, variant, g):
    """y_t = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts with the variant's weight,
    O(T^2) [LA definition]."""
    T = q.shape[0]
    W = variant_weights(q, k, variant, g) * np.tril(np.ones((T, T)))
    den = W.sum(axis=1)
    _check_den(den)
    return (W @ v) / den[:, None]


def forward_variant_rows(q, k, v, rows, variant, g):
    """Rows `rows` of the causal output from the definition, each in O(t):
    the closed-form weights of keys 0..t for query t [LA definition]."""
    out = np.empty((len(rows), v.shape[1]))
    for n, t in enumerate(rows):
        w = variant_weights(q[t:t + 1], k[:t + 1], variant, g)[0]
        den = w.sum()
        _check_den(np.array([den]))
        out[n] = (w @ v[:t + 1]) / den
    return out


def forward_variant_recurrent(q, k, v, variant, g, return_state=False):
    """The same output from the packed state: S_t = S_{t-1} + phi(k_t) v_t^T,
    z_t = z_{t-1} + phi(k_t), y_t = phi~(q_t)^T S_t / phi~(q_t)^T z_t."""
    fk = variant_key_feature(k, variant, g)
    fq = variant_query_feature(q, variant, g)
    S = np.zeros((fk.shape[1], v.shape[1]))
    z = np.zeros(fk.shape[1])
    y = np.empty((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        S += np.outer(fk[t], v[t])
        z += fk[t]
        den = float(fq[t] @ z)
        _check_den(np.array([den]))
        y[t] = (fq[t] @ S) / den
    if return_state:
        return y, S, z
    return y


def forward_delta(q, k, v, beta, key_feature=psd_key_feature, query_feature=psd_query_feature,
                  return_state=False):
    """DeltaKATA on the packed, normaliser-augmented state (reading 4).
    beta [T] in (0, 1]; the features default to the rank-one PSD feature
    (DeltaKATA-M1); pass a variant's feature functions for the others."""
    beta = np.asarray(beta, dtype=np.float64)
    if beta.shape != (q.shape[0],) or np.any(beta <= 0.0) or np.any(beta > 1.0):
        raise ValueError("beta must be [T] with entries in (0, 1]")
    fk = key_feature(k)
    fqk = query_feature(k)          # the key read as a query: its stored binding
    fq = query_feature(q)
    d_v = v.shape[1]
    Sa = np.zeros((fk.shape[1], d_v + 1))
    y = np.empty((q.shape[0], d_v))
    for t in range(q.shape[0]):
        target = np.append(v[t], 1.0)
        Sa += beta[t] * np.outer(fk[t], target - fqk[t] @ Sa)
        r = fq[t] @ Sa
        _check_den(np.array([r[d_v]]))
        y[t] = r[:d_v] / r[d_v]
    if return_state:
        return y, Sa
    return y


def forward_delta_chunked(q, k, v, beta, C, key_feature=psd_key_feature,
                          query_feature=psd_query_feature, return_state=False):
    """DeltaKATA (reading 4) in chunks of C tokens. Inside a chunk starting
    from S'_0, every state is S'_t = S'_0 + sum_{s<=t} phi(k_s) e_s^T, where
    e_t = beta_t ([v_t, 1] - phi~(k_t)^T S'_{t-1}) is the token's correction.
    Substituting gives a lower-triangular system for the chunk's corrections
    E (C x (d_v + 1)):
        e_t + beta_t sum_{s<t} A_ts e_s = beta_t ([v_t, 1] - phi~(k_t)^T S'_0),
    with A_ts = phi~(k_t) . phi(k_s), the weight between keys t and s. Then
        phi~(q_t)^T S'_t = phi~(q_t)^T S'_0 + sum_{s<=t} (phi~(q_t) . phi(k_s)) e_s,
        S'_C = S'_0 + Phi(K)^T E.
    A library triangular solve is the step for E."""
    beta = np.asarray(beta, dtype=np.float64)
    if beta.shape != (q.shape[0],) or np.any(beta <= 0.0) or np.any(beta > 1.0):
        raise ValueError("beta must be [T] with entries in (0, 1]")
    if C < 1:
        raise ValueError("C must be >= 1")
    fk, fqk, fq = key_feature(k), query_feature(k), query_feature(q)
    T, d_v = q.shape[0], v.shape[1]
    Sa = np.zeros((fk.shape[1], d_v + 1))
    y = np.empty((T, d_v))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        n = sl.stop - sl.start
        Phi, Psi, Fq, b = fk[sl], fqk[sl], fq[sl], beta[sl]
        U = np.concatenate([v[sl], np.ones((n, 1))], axis=1)
        A = np.tril(Psi @ Phi.T, -1)                       # A_ts, s < t
        M = np.eye(n) + b[:, None] * A
        E = np.linalg.solve(M, b[:, None] * (U - Psi @ Sa))
        R = Fq @ Sa + np.tril(Fq @ Phi.T) @ E               # phi~(q_t)^T S'_t
        _check_den(R[:, d_v])
        y[sl] = R[:, :d_v] / R[:, d_v:]
        Sa = Sa + Phi.T @ E
    if return_state:
        return y, Sa
    return y


def forward_delta_unpacked(q, k, v, beta):
    """DeltaKATA-M1 with the full d_k x d_k x (d_v + 1) state (no packing):
    M_t = M_{t-1} + beta_t (k_t k_t^T) (x) ([v_t, 1] - <k_t k_t^T, M_{t-1}>),
    y_t from <q_t q_t^T, M_t> -- reading 4 written with psi(x) = x x^T."""
    T, d_k = q.shape
    d_v = v.shape[1]
    M = np.zeros((d_k, d_k, d_v + 1))
    y = np.empty((T, d_v))
    for t in range(T):
        kk = np.outer(k[t], k[t])
        stored = np.tensordot(kk, M, axes=([0, 1], [0, 1]))
        M += beta[t] * kk[:, :, None] * (np.append(v[t], 1.0) - stored)[None, None, :]
        r = np.tensordot(np.outer(q[t], q[t]), M, axes=([0, 1], [0, 1]))
        _check_den(np.array([r[d_v]]))
        y[t] = r[:d_v] / r[d_v]
    return y
