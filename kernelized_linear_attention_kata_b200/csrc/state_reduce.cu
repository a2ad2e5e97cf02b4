// The state after a sequence, from the per-segment increments of the
// chunked form: S = sum over segments of sum phi(k_t) v_t^T, z = sum phi(k_t)
// (the state is additive over tokens, the property the scan across chunks
// rests on: KATA explainer 2.3). Converts each kernel family's increment
// layout to the library's packed layout (i <= j row-major for PSD; row 0 =
// the constant feature for first-order).
#include "common.cuh"
#include "launch.h"
#include "profile.h"

namespace kata {
namespace {

constexpr int kReduceThreads = 256;

// Index of the PSD tensor-core kernel's internal feature for the library row
// (i, j), i <= j, d_k = 32: f = 32 d + l is the pair (l, (l + d) mod 32) for
// d < 16, f = 512 + l is (l, l + 16). The kernel keeps m_f S_f (m_f = 2 off
// the diagonal).
__device__ __forceinline__ int psd_tc_feature(int i, int j) {
  const int d = j - i;
  if (d < 16) return 32 * d + i;
  if (d == 16) return 512 + i;
  return 32 * (32 - d) + j;
}

__global__ void __launch_bounds__(kReduceThreads)
state_reduce_kernel(int layout, const float *__restrict__ agg, int G, int D, int d_k, int d_v,
                    float *__restrict__ S_out, float *__restrict__ z_out, float count_pad) {
  const int nb = (D * (d_v + 1) + kReduceThreads - 1) / kReduceThreads;   // blocks per head
  const long long bh = blockIdx.x / nb;
  const size_t inc = layout == kAggLibrary ? (size_t)D * (d_v + 1)
                   : layout == kAggPsdTc   ? (size_t)D * d_v + (size_t)d_k * d_k
                                           : (size_t)(d_k + 1) * (d_k + 1);
  const float *base = agg + (size_t)bh * G * inc;
  const int e = (int)(blockIdx.x % nb) * kReduceThreads + threadIdx.x;   // one state entry per thread
  if (e < D * (d_v + 1)) {
    const int r = e / (d_v + 1), c = e % (d_v + 1);     // library row r, column c (c = d_v: z)
    size_t off;
    float scale = 1.f, pad = 0.f;
    if (layout == kAggLibrary) {
      off = (size_t)r * (d_v + 1) + c;
    } else if (layout == kAggPsdTc) {
      int i, j;
      psd_pair(r, d_k, i, j);
      if (c < d_v) {
        const int f = psd_tc_feature(i, j);
        off = (size_t)f * d_v + c;
        scale = f < d_k ? 1.f : 0.5f;
      } else {
        off = (size_t)D * d_v + (size_t)i * d_k + j;     // z_(i,j) = sum k_i k_j
      }
    } else {
      // first-order: internal row d_k is the constant feature, column d_v the count
      const int ri = r == 0 ? d_k : r - 1;
      off = (size_t)ri * (d_k + 1) + c;
      if (r == 0 && c == d_v) pad = count_pad;
    }
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += base[(size_t)g * inc + off];
    s = s * scale - pad;
    if (c < d_v) {
      if (S_out) S_out[((size_t)bh * D + r) * d_v + c] = s;
    } else if (z_out) {
      z_out[(size_t)bh * D + r] = s;
    }
  }
}

}  // namespace

cudaError_t state_reduce(AggLayout layout, const float *agg, long long BH, int G, int D, int d_k,
                         int d_v, float *S_out, float *z_out, float count_pad, cudaStream_t stream) {
  ProfileScope prof("state_reduce", stream);
  const long long nb = (D * (d_v + 1) + kReduceThreads - 1) / kReduceThreads;
  state_reduce_kernel<<<(unsigned)(BH * nb), kReduceThreads, 0, stream>>>((int)layout, agg, G, D, d_k,
                                                                          d_v, S_out, z_out,
                                                                          count_pad);
  return cudaGetLastError();
}

}  // namespace kata
