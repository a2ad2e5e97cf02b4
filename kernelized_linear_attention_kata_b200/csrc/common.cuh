// Shared device helpers for the KATA kernels: element conversion, feature
// indexing of the packed state, and the status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kata {

// Feature maps. kMg2 and kSg2 are the two-factor variants KATA-Mg and
// KATA-Sigma-g (g = 2) named by the KATA explainer (section 2.3), read with
// the factors of x in R^d_k as its two halves x_1, x_2 in R^(d_k / 2):
//   Mg2: phi(x) = [psi(x_1), psi(x_2)], weight <q_1,k_1>^2 + <q_2,k_2>^2,
//        state rows: the packed pairs of slice 1, then those of slice 2;
//   Sg2: Psi(x) = x_1 x_1^T + x_2 x_2^T, weight sum_{a,b} <q_a, k_b>^2,
//        state rows: the packed pairs (i <= j) of one slice.
enum Feature : int { kPSD = 0, kFirstOrder = 1, kMg2 = 2, kSg2 = 3 };

// Status bits written by kernels into the first word of the workspace.
enum : unsigned { kStatusNonPositiveNormaliser = 1u, kStatusDeviceTimeout = 2u };

__host__ __device__ constexpr int state_dim(int d_k, int feat) {
  return feat == kPSD          ? d_k * (d_k + 1) / 2
         : feat == kFirstOrder ? d_k + 1
         : feat == kMg2        ? 2 * ((d_k / 2) * (d_k / 2 + 1) / 2)
                               : (d_k / 2) * (d_k / 2 + 1) / 2;
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Packed PSD row r <-> (i, j), i <= j, row-major over i then j.
__host__ __device__ __forceinline__ void psd_pair(int r, int d_k, int &i, int &j) {
  int row_start = 0, ii = 0;
  while (r >= row_start + (d_k - ii)) {
    row_start += d_k - ii;
    ++ii;
  }
  i = ii;
  j = ii + (r - row_start);
}

// Key-side feature of state row r (no multiplicity), from a token's key in
// shared memory. PSD and Mg2: k_i k_j. Sg2: k_i k_j + k_(h+i) k_(h+j)
// (h = d_k / 2). First-order: row 0 -> 1, row 1+i -> k_i.
template <int DK, int FEAT>
__device__ __forceinline__ float key_feature_row(const float *kt, int i, int j) {
  if constexpr (FEAT == kPSD || FEAT == kMg2) {
    return kt[i] * kt[j];
  } else if constexpr (FEAT == kSg2) {
    return fmaf(kt[i], kt[j], kt[DK / 2 + i] * kt[DK / 2 + j]);
  } else {
    return i < 0 ? 1.f : kt[i];
  }
}

// Row r's feature indices: PSD (i, j); Mg2 (i, j) in slice (r < D/2 ? 1 :
// 2), as indices of the whole key; Sg2 (i, j) within a slice; first-order
// (r - 1, -) with -1 for the constant row.
template <int DK, int FEAT>
__device__ __forceinline__ void row_indices(int r, int &i, int &j) {
  if constexpr (FEAT == kPSD) {
    psd_pair(r, DK, i, j);
  } else if constexpr (FEAT == kMg2) {
    constexpr int H = DK / 2, D1 = H * (H + 1) / 2;
    const int b = r >= D1 ? 1 : 0;
    psd_pair(r - b * D1, H, i, j);
    i += b * H;
    j += b * H;
  } else if constexpr (FEAT == kSg2) {
    psd_pair(r, DK / 2, i, j);
  } else {
    i = r - 1;
    j = 0;
  }
}

// Query-side multiplicity of row (i, j): 2 off the diagonal for the PSD
// features (the packed state keeps one of the pairs (i, j), (j, i)).
template <int FEAT>
__device__ __forceinline__ float query_mult(int i, int j) {
  if constexpr (FEAT == kFirstOrder) {
    return 1.f;
  } else {
    return i == j ? 1.f : 2.f;
  }
}

// The weight <phi(q), phi(k)> of a query (registers) and a key (shared
// memory), in closed form: (q.k)^2, 1 + q.k, <q_1,k_1>^2 + <q_2,k_2>^2 or
// sum_{a,b} <q_a,k_b>^2.
template <int DK, int FEAT>
__device__ __forceinline__ float pair_weight(const float (&qv)[DK], const float *kr) {
  if constexpr (FEAT == kPSD || FEAT == kFirstOrder) {
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < DK; ++i) dot = fmaf(qv[i], kr[i], dot);
    return FEAT == kPSD ? dot * dot : 1.f + dot;
  } else {
    constexpr int H = DK / 2;
    float d11 = 0.f, d22 = 0.f, d12 = 0.f, d21 = 0.f;
#pragma unroll
    for (int i = 0; i < H; ++i) {
      d11 = fmaf(qv[i], kr[i], d11);
      d22 = fmaf(qv[H + i], kr[H + i], d22);
      if constexpr (FEAT == kSg2) {
        d12 = fmaf(qv[i], kr[H + i], d12);
        d21 = fmaf(qv[H + i], kr[i], d21);
      }
    }
    return FEAT == kMg2 ? fmaf(d11, d11, d22 * d22)
                        : fmaf(d11, d11, fmaf(d22, d22, fmaf(d12, d12, d21 * d21)));
  }
}

__device__ __forceinline__ void flag_status(unsigned *status, unsigned bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace kata
