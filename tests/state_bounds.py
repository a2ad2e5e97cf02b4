"""Element-wise error bounds for the states (S, z) the library returns, from
the arithmetic each kernel family does, with the fp64 oracle's state as the
reference.

Every state entry is a sum over tokens, S_f,c = sum_t a_t with
a_t = phi_f(k_t) v_t,c (and z_f = sum_t phi_f(k_t)). Two error sources:

* fp32 accumulation of T terms. The recursive-summation bound is
  |error| <= (n - 1) u32 sum_t |a_t| with u32 = 2^-24; the tensor core's
  accumulator is held to twice that (n = T + 8 leaves room for the segment
  carry-in and the state reduction): (T + 8) 2^-23 S_abs, with
  S_abs = sum_t |a_t| the oracle's state of |k|, |v|.
* In the bf16 tensor-core PSD path only: the key feature k_i k_j enters the
  update MMA rounded to bf16, one rounding of unit roundoff u = 2^-8 per
  product (the factor 2 the kernel moves onto the key side is exact). The
  error sum_t e_t a_t, |e_t| <= u, of roughly independent roundings has a
  standard deviation of at most u R / sqrt(3), with R^2 = sum_t a_t^2 the
  oracle's state of k*k, v*v. The bound takes 4 u R (6.9 standard
  deviations). A mistake in the state is of the size of the entry itself,
  about R for keys and values of random sign, far above 4 u R. z is formed
  as K^T K from exact products, so only the accumulation term applies.

Inputs with many repeated keys (the long MQAR-like workload) correlate the
roundings; the states are compared on unit-recipe inputs only.
"""

import numpy as np

import oracle as O

U_BF16 = 2.0 ** -8
U_ACC = 2.0 ** -23


def reference_and_bounds(kn, vn, feature, tc_psd):
    """(S_ref, z_ref, S_bound, z_bound) for one head's fp64 k [T, d_k], v [T, d_v]."""
    T = kn.shape[0]
    S_ref, z_ref = O.final_state(kn, vn, feature)
    S_abs, z_abs = O.final_state(np.abs(kn), np.abs(vn), feature)
    S_bound = (T + 8) * U_ACC * S_abs
    z_bound = (T + 8) * U_ACC * z_abs
    if tc_psd:
        R2, _ = O.final_state(kn * kn, vn * vn, feature)
        S_bound = S_bound + 4.0 * U_BF16 * np.sqrt(R2)
    return S_ref, z_ref, S_bound, z_bound


def tc_psd_path(dtype, feature, d_k, d_v, C):
    """Whether the bf16 tensor-core PSD kernels (bf16 key products) run this shape."""
    return dtype == "bf16" and feature == "psd" and (d_k, d_v) == (32, 64) and C in (64, 128)


def assert_state_close(S, z, kn, vn, feature, tc_psd, label="", scale=1.0):
    """Compare device states S [B, H, D, d_v], z [B, H, D] with the oracle's
    for the fp64 inputs kn [B, H, T, d_k], vn [B, H, T, d_v], element by
    element. `scale` widens the bounds for a state summed from `scale`
    independently rounded parts."""
    S = np.asarray(S, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    B, H = kn.shape[:2]
    for b in range(B):
        for h in range(H):
            S_ref, z_ref, S_bd, z_bd = reference_and_bounds(kn[b, h], vn[b, h], feature, tc_psd)
            # a floor for entries whose terms all vanish (exact zeros)
            eS = np.abs(S[b, h] - S_ref) - (scale * S_bd + 1e-30)
            ez = np.abs(z[b, h] - z_ref) - (scale * z_bd + 1e-30)
            if np.any(eS > 0):
                f, c = np.unravel_index(int(np.argmax(eS)), eS.shape)
                raise AssertionError(
                    f"{label} S[{b},{h},{f},{c}] = {S[b, h, f, c]!r}, oracle {S_ref[f, c]!r}, "
                    f"bound {scale * S_bd[f, c]:.3e}")
            if np.any(ez > 0):
                f = int(np.argmax(ez))
                raise AssertionError(f"{label} z[{b},{h},{f}] = {z[b, h, f]!r}, oracle {z_ref[f]!r}, "
                                     f"bound {scale * z_bd[f]:.3e}")
