// Shared device helpers for the KATA kernels: element conversion, feature
// indexing of the packed state, and the status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kata {

enum Feature : int { kPSD = 0, kFirstOrder = 1 };

// Status bits written by kernels into the first word of the workspace.
enum : unsigned { kStatusNonPositiveNormaliser = 1u, kStatusDeviceTimeout = 2u };

__host__ __device__ constexpr int state_dim(int d_k, int feat) {
  return feat == kPSD ? d_k * (d_k + 1) / 2 : d_k + 1;
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
// shared memory. PSD: k_i k_j. First-order: row 0 -> 1, row 1+i -> k_i.
template <int DK, int FEAT>
__device__ __forceinline__ float key_feature_row(const float *kt, int i, int j) {
  if constexpr (FEAT == kPSD) {
    return kt[i] * kt[j];
  } else {
    return i < 0 ? 1.f : kt[i];
  }
}

// Row r's feature indices: PSD (i, j); first-order (r - 1, -) with -1 for
// the constant row.
template <int DK, int FEAT>
__device__ __forceinline__ void row_indices(int r, int &i, int &j) {
  if constexpr (FEAT == kPSD) {
    psd_pair(r, DK, i, j);
  } else {
    i = r - 1;
    j = 0;
  }
}

// Query-side multiplicity of row (i, j): 2 off the diagonal for PSD.
template <int FEAT>
__device__ __forceinline__ float query_mult(int i, int j) {
  if constexpr (FEAT == kPSD) {
    return i == j ? 1.f : 2.f;
  } else {
    return 1.f;
  }
}

__device__ __forceinline__ void flag_status(unsigned *status, unsigned bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace kata
