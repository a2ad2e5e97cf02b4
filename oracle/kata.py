"""Plain fp64 CPU oracle for the KATA causal forward, its chunked and scanned
forms, and the one-token recurrent decode step.

TEST INFRASTRUCTURE. This module is read by the tests, by the smoke check and
by the benchmark's CPU-baseline leg only. The CUDA library and its Python
binding never import it; there is no CPU fallback anywhere in the product.

Every function works on ONE head: q, k are [T, d_k], v is [T, d_v], all
float64 numpy arrays. ``per_head`` lifts a function to [B, H, T, d] arrays.
Nothing here is blocked, fused or reordered beyond what the stated definition
or algorithm says; a library matmul is used as a step where the definition is
a matrix product.

Sources, cited by page title and section:

[ABS]  "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
       Cones", arXiv 2607.17419v1, abstract (fugumt.com listing).
[JA]   Same title, gist.science Japanese explainer, technical summary
       (sections 1-4).
[IT]   Same title, gist.science Italian explainer, section 2.
[LA]   "線形注意" (linear attention), notes wiki page, section "定義"
       (definition).

What the pages fix, restated:

* Linear attention replaces the exponential kernel by an inner product of
  finite-dimensional features, <phi(c), phi(q)>, so that the output can be
  produced by an RNN carrying a fixed-size state [LA, definition].
* KATA's rank-one PSD feature is psi(u) = u u^T; the weight between a query
  and a key is <psi(q), psi(k)> = <q, k>^2, never negative [JA 2.2, IT 2.2,
  ABS].
* The normaliser of normalised linear attention acts as a parameter-free,
  token-conditioned convex output gate interpolating between the previous
  readout and the current value [JA 2.1, IT 2.1, ABS].
* The exact O(T) chunked-state form splits the sequence into chunks; inside a
  chunk the attention block is dense, across chunks a state is carried, and
  the carry can be done by an associative scan (parallel prefix sum) whose
  depth is O(log(T/C)) [JA 2.3, IT 2.3, ABS].
* The abstract's scan is "of the first-order feature"; this oracle reads that
  as the Lorentz-cone (first-order Taylor) feature phi_1(u) = [1, u], weight
  1 + <q, k> [ABS; JA 2.2 names the Lorentz cone]. This reading is not fixed
  by the pages; parity for that feature is pinned only by the generic
  properties below (weights, hull, forms agreement), not by any printed value.

Readings where the pages are silent (each one is restated beside the code that
uses it):

* Causal mask includes the diagonal (s <= t), so y_1 = v_1.
* No temperature / 1/sqrt(d) scale; q and k are used as given.
* Packed PSD state: row (i, j) for i <= j, rows ordered row-major over i then
  j. The key side uses the raw product k_i k_j; the query side carries the
  multiplicity 2 for i < j, so that  phi_q(q) . phi_k(k) = <q q^T, k k^T>_F.
* A non-positive denominator is an error (no epsilon is added).
"""

from __future__ import annotations

import numpy as np

PSD = "psd"
FIRST_ORDER = "first_order"
FEATURES = (PSD, FIRST_ORDER)


# ---------------------------------------------------------------------------
# Feature maps
# ---------------------------------------------------------------------------

def psd_pairs(d_k: int) -> list[tuple[int, int]]:
    """Index pairs (i, j), i <= j, in packed-row order (row-major over i, then j).

    The rank-one PSD feature psi(u) = u u^T is symmetric [JA 2.2], so only the
    upper triangle carries information; its d_k (d_k + 1) / 2 entries are the
    packed state rows.
    """
    return [(i, j) for i in range(d_k) for j in range(i, d_k)]


def state_dim(d_k: int, feature: str) -> int:
    """D, the number of state rows: d_k(d_k+1)/2 for PSD, d_k+1 for first-order."""
    if feature == PSD:
        return d_k * (d_k + 1) // 2
    if feature == FIRST_ORDER:
        return d_k + 1
    raise ValueError(f"unknown feature {feature!r}")


def psd_key_feature(x: np.ndarray) -> np.ndarray:
    """Packed psi(x) = x x^T, upper triangle: [..., d_k] -> [..., D]."""
    d_k = x.shape[-1]
    iu, ju = np.triu_indices(d_k)          # same order as psd_pairs
    return np.take(x, iu, axis=-1) * np.take(x, ju, axis=-1)


def psd_query_feature(x: np.ndarray) -> np.ndarray:
    """Packed psi(x) with the off-diagonal multiplicity 2 folded in.

    <psi(q), psi(k)>_F sums every (i, j) and (j, i) entry; packing keeps one of
    each off-diagonal pair, so the query side counts it twice.
    """
    d_k = x.shape[-1]
    iu, ju = np.triu_indices(d_k)
    mult = np.where(iu == ju, 1.0, 2.0)
    return np.take(x, iu, axis=-1) * np.take(x, ju, axis=-1) * mult


def first_order_feature(x: np.ndarray) -> np.ndarray:
    """phi_1(u) = [1, u] (Lorentz / first-order reading of [ABS])."""
    ones = np.ones(x.shape[:-1] + (1,), dtype=x.dtype)
    return np.concatenate([ones, x], axis=-1)


def key_feature(x: np.ndarray, feature: str) -> np.ndarray:
    if feature == PSD:
        return psd_key_feature(x)
    if feature == FIRST_ORDER:
        return first_order_feature(x)
    raise ValueError(f"unknown feature {feature!r}")


def query_feature(x: np.ndarray, feature: str) -> np.ndarray:
    if feature == PSD:
        return psd_query_feature(x)
    if feature == FIRST_ORDER:
        return first_order_feature(x)
    raise ValueError(f"unknown feature {feature!r}")


def weights(q: np.ndarray, k: np.ndarray, feature: str) -> np.ndarray:
    """W[t, s] = <phi(q_t), phi(k_s)> written in closed form.

    PSD: <q_t, k_s>^2 [JA 2.2, IT 2.2]. First-order: 1 + <q_t, k_s>.
    """
    g = q @ k.T
    if feature == PSD:
        return g * g
    if feature == FIRST_ORDER:
        return 1.0 + g
    raise ValueError(f"unknown feature {feature!r}")


def _check_den(den: np.ndarray) -> None:
    if np.any(~(den > 0.0)):
        bad = int(np.argmax(~(den > 0.0)))
        raise FloatingPointError(f"non-positive normaliser at row {bad}: {den.flat[bad]!r}")


# ---------------------------------------------------------------------------
# Forms of the causal forward (single head)
# ---------------------------------------------------------------------------

def forward_brute_force(q, k, v, feature=PSD):
    """Normalised causal linear attention from its definition, O(T^2).

    y_t = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts   [LA definition; ABS].
    """
    T = q.shape[0]
    W = weights(q, k, feature)
    W = W * np.tril(np.ones((T, T)))       # causal, diagonal included
    num = W @ v
    den = W.sum(axis=1)
    _check_den(den)
    return num / den[:, None]


def forward_rows(q, k, v, rows, feature=PSD):
    """The definition evaluated only at the given rows (for long sequences)."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), v.shape[1]))
    for n, t in enumerate(rows):
        w = weights(q[t:t + 1], k[:t + 1], feature)[0]
        den = w.sum()
        _check_den(np.array([den]))
        out[n] = (w @ v[:t + 1]) / den
    return out


def forward_recurrent_unpacked(q, k, v):
    """PSD recurrence with the full d_k x d_k x d_v state (no packing).

    S_t = S_{t-1} + (k_t k_t^T) (x) v_t,  Z_t = Z_{t-1} + k_t k_t^T,
    y_t = <q_t q_t^T, S_t> / <q_t q_t^T, Z_t>   -- the RNN view of [LA] with
    the rank-one PSD feature of [JA 2.2].
    """
    T, d_k = q.shape
    d_v = v.shape[1]
    S = np.zeros((d_k, d_k, d_v))
    Z = np.zeros((d_k, d_k))
    y = np.empty((T, d_v))
    for t in range(T):
        kk = np.outer(k[t], k[t])
        S += kk[:, :, None] * v[t][None, None, :]
        Z += kk
        qq = np.outer(q[t], q[t])
        den = float(np.sum(qq * Z))
        _check_den(np.array([den]))
        y[t] = np.tensordot(qq, S, axes=([0, 1], [0, 1])) / den
    return y


def forward_recurrent(q, k, v, feature=PSD, S0=None, z0=None, return_state=False):
    """Recurrence on the packed state (the library's state layout).

    S_t = S_{t-1} + phi(k_t) v_t^T, z_t = z_{t-1} + phi(k_t),
    y_t = phi_q(q_t)^T S_t / phi_q(q_t)^T z_t.
    """
    T = q.shape[0]
    fk = key_feature(k, feature)
    fq = query_feature(q, feature)
    D = fk.shape[1]
    S = np.zeros((D, v.shape[1])) if S0 is None else np.array(S0, dtype=np.float64)
    z = np.zeros(D) if z0 is None else np.array(z0, dtype=np.float64)
    y = np.empty((T, v.shape[1]))
    for t in range(T):
        S += np.outer(fk[t], v[t])
        z += fk[t]
        den = float(fq[t] @ z)
        _check_den(np.array([den]))
        y[t] = (fq[t] @ S) / den
    if return_state:
        return y, S, z
    return y


def forward_gated(q, k, v, feature=PSD):
    """The normaliser read as a convex output gate [JA 2.1, IT 2.1, ABS].

    With the state before token t (S_{t-1}, z_{t-1}):
      prev readout  r_t     = phi_q(q_t)^T S_{t-1} / phi_q(q_t)^T z_{t-1}
      gate          gamma_t = w_tt / (phi_q(q_t)^T z_{t-1} + w_tt)
      output        y_t     = (1 - gamma_t) r_t + gamma_t v_t.
    Reading: the "previous readout" is the previous state read with the
    current query (not y_{t-1}); only this makes the gate equal the
    normaliser. When phi_q(q_t)^T z_{t-1} = 0 the previous readout carries no
    weight (gamma_t = 1) and y_t = v_t.
    """
    T = q.shape[0]
    fk = key_feature(k, feature)
    fq = query_feature(q, feature)
    D = fk.shape[1]
    S = np.zeros((D, v.shape[1]))
    z = np.zeros(D)
    y = np.empty((T, v.shape[1]))
    for t in range(T):
        prev_den = float(fq[t] @ z)
        w_tt = float(fq[t] @ fk[t])
        total = prev_den + w_tt
        _check_den(np.array([total]))
        gamma = w_tt / total
        if prev_den > 0.0:
            readout = (fq[t] @ S) / prev_den
            y[t] = (1.0 - gamma) * readout + gamma * v[t]
        else:
            y[t] = v[t]
        S += np.outer(fk[t], v[t])
        z += fk[t]
    return y


def forward_chunked(q, k, v, C, feature=PSD, S0=None, z0=None, return_state=False):
    """Exact chunked-state form [JA 2.3, IT 2.3, ABS], any chunk size C >= 1.

    For each chunk c (rows r0..r1-1; the last chunk may be shorter):
      A      = W(Q_c, K_c) masked to s <= t (intra-chunk block, diagonal kept)
      num    = A V_c + phi_q(Q_c) S_c
      den    = A 1   + phi_q(Q_c) z_c
      Y_c    = num / den
      S_{c+1} = S_c + phi(K_c)^T V_c,   z_{c+1} = z_c + phi(K_c)^T 1.
    """
    T = q.shape[0]
    D = state_dim(q.shape[1], feature)
    S = np.zeros((D, v.shape[1])) if S0 is None else np.array(S0, dtype=np.float64)
    z = np.zeros(D) if z0 is None else np.array(z0, dtype=np.float64)
    y = np.empty((T, v.shape[1]))
    for r0 in range(0, T, C):
        r1 = min(r0 + C, T)
        Qc, Kc, Vc = q[r0:r1], k[r0:r1], v[r0:r1]
        n = r1 - r0
        A = weights(Qc, Kc, feature) * np.tril(np.ones((n, n)))
        fq = query_feature(Qc, feature)
        num = A @ Vc + fq @ S
        den = A.sum(axis=1) + fq @ z
        _check_den(den)
        y[r0:r1] = num / den[:, None]
        fk = key_feature(Kc, feature)
        S = S + fk.T @ Vc
        z = z + fk.sum(axis=0)
    if return_state:
        return y, S, z
    return y


def chunk_deltas(k, v, C, feature=PSD):
    """Per-chunk state increments (Delta S_c, Delta z_c) = (phi(K_c)^T V_c, phi(K_c)^T 1)."""
    T = k.shape[0]
    out = []
    for r0 in range(0, T, C):
        r1 = min(r0 + C, T)
        fk = key_feature(k[r0:r1], feature)
        out.append((fk.T @ v[r0:r1], fk.sum(axis=0)))
    return out


def exclusive_tree_scan(items):
    """Exclusive prefix sums of a list of (S, z) pairs by a balanced tree.

    The associative scan (parallel prefix sum) across chunk states of [JA 2.3,
    IT 2.3, ABS]: an up-sweep builds partial sums over a binary tree, a
    down-sweep hands every node the sum of everything to its left. Depth is
    2 * ceil(log2 n) combine levels; the combine operator is elementwise +.
    """
    n = len(items)
    if n == 0:
        return []
    size = 1
    while size < n:
        size *= 2
    zero = (np.zeros_like(items[0][0]), np.zeros_like(items[0][1]))
    tree = [(a.copy(), b.copy()) for a, b in items] + [zero] * (size - n)
    # up-sweep: tree[i] becomes the sum of the block of 2*step ending at i
    step = 1
    while step < size:
        for i in range(2 * step - 1, size, 2 * step):
            left = tree[i - step]
            tree[i] = (tree[i][0] + left[0], tree[i][1] + left[1])
        step *= 2
    # down-sweep: the root receives the identity; each node passes its value
    # to the left child and (value + left-child sum) to the right child
    tree[size - 1] = (np.zeros_like(zero[0]), np.zeros_like(zero[1]))
    step = size // 2
    while step >= 1:
        for i in range(2 * step - 1, size, 2 * step):
            left = tree[i - step]
            tree[i - step] = tree[i]
            tree[i] = (tree[i][0] + left[0], tree[i][1] + left[1])
        step //= 2
    return tree[:n]


def forward_chunked_scanned(q, k, v, C, feature=PSD):
    """Chunked form whose inter-chunk carry is the tree scan above.

    Every chunk's carry-in state is the exclusive prefix of the chunk
    increments, so after the scan all chunks are independent.
    """
    T = q.shape[0]
    prefixes = exclusive_tree_scan(chunk_deltas(k, v, C, feature))
    y = np.empty((T, v.shape[1]))
    for c, r0 in enumerate(range(0, T, C)):
        r1 = min(r0 + C, T)
        S, z = prefixes[c]
        y[r0:r1] = forward_chunked(q[r0:r1], k[r0:r1], v[r0:r1], C, feature, S0=S, z0=z)
    return y


def final_state(k, v, feature=PSD):
    """(S_T, z_T) = (sum_t phi(k_t) v_t^T, sum_t phi(k_t))."""
    fk = key_feature(k, feature)
    return fk.T @ v, fk.sum(axis=0)


def decode_step(q, k, v, S, z, feature=PSD):
    """One recurrent step from a given state: update with (k, v), then read with q.

    q, k: [d_k]; v: [d_v]; S: [D, d_v]; z: [D]. Returns (y, S', z'). The
    current token is included in its own readout, as in the forward.
    """
    fk = key_feature(k, feature)
    S2 = S + np.outer(fk, v)
    z2 = z + fk
    fq = query_feature(q, feature)
    den = float(fq @ z2)
    _check_den(np.array([den]))
    return (fq @ S2) / den, S2, z2


def decode_step_batched(q, k, v, S, z, feature=PSD):
    """decode_step over leading batch axes: q,k [..., d_k], v [..., d_v], S [..., D, d_v], z [..., D]."""
    fk = key_feature(k, feature)
    S2 = S + fk[..., :, None] * v[..., None, :]
    z2 = z + fk
    fq = query_feature(q, feature)
    den = np.einsum("...d,...d->...", fq, z2)
    _check_den(den)
    num = np.einsum("...d,...dv->...v", fq, S2)
    return num / den[..., None], S2, z2


# ---------------------------------------------------------------------------
# Batch lifting
# ---------------------------------------------------------------------------

def per_head(fn, q, k, v, *args, **kwargs):
    """Apply a single-head form to [B, H, T, d] arrays; returns [B, H, T, d_v]."""
    B, H = q.shape[:2]
    out = np.empty(q.shape[:3] + (v.shape[-1],))
    for b in range(B):
        for h in range(H):
            out[b, h] = fn(q[b, h], k[b, h], v[b, h], *args, **kwargs)
    return out
