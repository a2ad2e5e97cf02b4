// DeltaKATA: the delta-rule state update the KATA explainer (section 4)
// credits with correcting stale bindings at repeated keys, on the CUDA cores
// (fp32 arithmetic for both element types).
//
// The pages name the variant without its rule; the library reads it as the
// delta rule on the state augmented with its normaliser, S' = [S | z]
// (D x (d_v + 1)), with a per-token write strength beta_t in (0, 1]:
//   S'_t = S'_(t-1) + beta_t phi(k_t) ([v_t, 1] - phi~(k_t)^T S'_(t-1)),
//   y_t  = (phi~(q_t)^T S'_t)[:d_v] / (phi~(q_t)^T S'_t)[d_v],
// phi the key-side and phi~ the query-side packed PSD feature, read after
// the write as in the additive forward.
//
// Computed in chunks of kDC tokens from the chunk's starting state S'_0
// (exact for any chunk length): with A_ts = <phi~(k_t), phi(k_s)>, s < t,
// the chunk's corrections E (kDC x (d_v + 1)) solve the lower-triangular
// system
//   E_t + beta_t sum_(s<t) A_ts E_s = beta_t ([v_t, 1] - phi~(k_t)^T S'_0),
// then
//   phi~(q_t)^T S'_t = phi~(q_t)^T S'_0 + sum_(s<=t) <phi~(q_t), phi(k_s)> E_s,
//   S'_kDC = S'_0 + Phi(K)^T E.
// The weights between tokens come in closed form ((a . b)^2 for PSD). One
// thread block per (b, h) walks its chunks in order: the delta rule does
// not add increments, so the sequence is not cut into segments.
//
// Shared memory (fp32): S' [D][d_v + 4] (column d_v holds z) | the chunk's
// q, k [kDC][d_k] and v [kDC][d_v] | phi~(K) S'_0 then the corrections E
// [kDC][d_v + 4] | phi~(Q) S'_0 then the readout [kDC][d_v + 4] | A and the
// query-key weights [kDC][kDC] | beta [kDC] | the packed row table [D].
#include "launch.h"
#include "profile.h"
#include "simt_kernels.cuh"

namespace kata {
namespace {

constexpr int kDC = 32;                 // tokens per chunk
constexpr int kDeltaThreads = 512;

template <int DK, int DV>
struct DeltaSmem {
  static constexpr int D = state_dim(DK, kPSD);
  static constexpr int P = DV + 4;      // augmented row stride (z at column DV)
  static constexpr int S = 0;
  static constexpr int Q = S + D * P;
  static constexpr int K = Q + kDC * DK;
  static constexpr int V = K + kDC * DK;
  static constexpr int E = V + kDC * DV;
  static constexpr int R = E + kDC * P;
  static constexpr int A = R + kDC * P;
  static constexpr int B = A + kDC * kDC;
  static constexpr int BETA = B + kDC * kDC;
  static constexpr int TAB = BETA + kDC;          // int4 entries, 16-byte aligned below
  static constexpr size_t bytes() { return sizeof(float) * (size_t)(TAB + 4 * D); }
  static_assert(Q % 4 == 0 && E % 4 == 0 && R % 4 == 0 && TAB % 4 == 0, "float4 alignment");
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kDeltaThreads, 1)
delta_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
             const float *__restrict__ beta, Tin *__restrict__ o, const float *__restrict__ S0,
             float *__restrict__ S_out, unsigned *__restrict__ status, int T) {
  using L = DeltaSmem<DK, DV>;
  constexpr int D = L::D, P = L::P, NC = DV + 1;
  extern __shared__ __align__(16) float sm[];
  float *Sa = sm + L::S, *qs = sm + L::Q, *ks = sm + L::K, *vs = sm + L::V;
  float *E = sm + L::E, *R = sm + L::R, *A = sm + L::A, *Bq = sm + L::B, *bs = sm + L::BETA;
  int4 *tab = reinterpret_cast<int4 *>(sm + L::TAB);
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;

  fill_row_table<DK, kPSD>(tab, tid, kDeltaThreads);
  for (int e = tid; e < D * P; e += kDeltaThreads) {
    const int r = e / P, c = e % P;
    Sa[e] = (S0 && c < NC) ? S0[((size_t)bh * D + r) * NC + c] : 0.f;
  }
  const size_t qoff = (size_t)bh * T * DK, voff = (size_t)bh * T * DV;

  for (int c0 = 0; c0 < T; c0 += kDC) {
    const int n = min(kDC, T - c0);
    __syncthreads();
    load_rows_f32<Tin, DK>(qs, q + qoff + (size_t)c0 * DK, n, kDC, tid, kDeltaThreads);
    load_rows_f32<Tin, DK>(ks, k + qoff + (size_t)c0 * DK, n, kDC, tid, kDeltaThreads);
    load_rows_f32<Tin, DV>(vs, v + voff + (size_t)c0 * DV, n, kDC, tid, kDeltaThreads);
    if (tid < kDC) bs[tid] = tid < n ? beta[(size_t)bh * T + c0 + tid] : 0.f;
    __syncthreads();

    // ---- phi~(k_t)^T S'_0 and phi~(q_t)^T S'_0: one (token, 4 columns) per item ----
    constexpr int NG = P / 4;
    for (int item = tid; item < kDC * NG; item += kDeltaThreads) {
      const int t = item / NG, g = item % NG;
      const float *kt = ks + t * DK, *qt = qs + t * DK;
      float4 ak = make_float4(0.f, 0.f, 0.f, 0.f), aq = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int r = 0; r < D; ++r) {
        const int4 e = tab[r];
        const float m = __int_as_float(e.z);
        const float fk = m * kt[e.x] * kt[e.y], fq = m * qt[e.x] * qt[e.y];
        const float4 s = reinterpret_cast<const float4 *>(Sa + r * P)[g];
        ak.x = fmaf(fk, s.x, ak.x); ak.y = fmaf(fk, s.y, ak.y);
        ak.z = fmaf(fk, s.z, ak.z); ak.w = fmaf(fk, s.w, ak.w);
        aq.x = fmaf(fq, s.x, aq.x); aq.y = fmaf(fq, s.y, aq.y);
        aq.z = fmaf(fq, s.z, aq.z); aq.w = fmaf(fq, s.w, aq.w);
      }
      reinterpret_cast<float4 *>(E + t * P)[g] = ak;
      reinterpret_cast<float4 *>(R + t * P)[g] = aq;
    }
    // ---- weights between the chunk's tokens: A_ts (s < t), <phi~(q_t), phi(k_s)> (s <= t) ----
    for (int e = tid; e < kDC * kDC; e += kDeltaThreads) {
      const int t = e / kDC, s = e % kDC;
      float dk = 0.f, dq = 0.f;
#pragma unroll
      for (int i = 0; i < DK; ++i) {
        dk = fmaf(ks[t * DK + i], ks[s * DK + i], dk);
        dq = fmaf(qs[t * DK + i], ks[s * DK + i], dq);
      }
      A[e] = s < t ? dk * dk : 0.f;
      Bq[e] = s <= t ? dq * dq : 0.f;
    }
    __syncthreads();
    // ---- corrections: forward substitution, one thread per column ----
    if (tid < NC) {
      const int c = tid;
      for (int t = 0; t < n; ++t) {
        const float u = c < DV ? vs[t * DV + c] : 1.f;
        float acc = 0.f;
        for (int s = 0; s < t; ++s) acc = fmaf(A[t * kDC + s], E[s * P + c], acc);
        E[t * P + c] = bs[t] * (u - E[t * P + c] - acc);
      }
      for (int t = n; t < kDC; ++t) E[t * P + c] = 0.f;
    }
    __syncthreads();
    // ---- readout after each write: phi~(q_t)^T S'_t, then y_t ----
    for (int item = tid; item < kDC * NC; item += kDeltaThreads) {
      const int t = item / NC, c = item % NC;
      float acc = R[t * P + c];
      for (int s = 0; s <= t; ++s) acc = fmaf(Bq[t * kDC + s], E[s * P + c], acc);
      R[t * P + c] = acc;
    }
    __syncthreads();
    for (int item = tid; item < n * DV; item += kDeltaThreads) {
      const int t = item / DV, c = item % DV;
      const float den = R[t * P + DV];
      if (c == 0 && !(den > 0.f)) flag_status(status, kStatusNonPositiveNormaliser);
      o[voff + (size_t)(c0 + t) * DV + c] = from_f<Tin>(R[t * P + c] / den);
    }
    // ---- S' += Phi(K)^T E, one state row per thread ----
    for (int r = tid; r < D; r += kDeltaThreads) {
      const int4 e = tab[r];
      float ph[kDC];
#pragma unroll
      for (int t = 0; t < kDC; ++t) ph[t] = ks[t * DK + e.x] * ks[t * DK + e.y];
      for (int c = 0; c < NC; ++c) {
        float acc = Sa[r * P + c];
#pragma unroll
        for (int t = 0; t < kDC; ++t) acc = fmaf(ph[t], E[t * P + c], acc);
        Sa[r * P + c] = acc;
      }
    }
  }
  __syncthreads();
  if (S_out) {
    for (int e = tid; e < D * NC; e += kDeltaThreads)
      S_out[(size_t)bh * D * NC + e] = Sa[(e / NC) * P + e % NC];
  }
}

}  // namespace

template <int DK, int DV, typename Tin>
cudaError_t simt_delta(const DeltaLaunch &a) {
  using L = DeltaSmem<DK, DV>;
  auto kern = delta_kernel<DK, DV, Tin>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::bytes());
  if (e != cudaSuccess) return e;
  ProfileScope prof("simt_delta", a.stream);
  kern<<<(unsigned)a.BH, kDeltaThreads, L::bytes(), a.stream>>>(
      static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v),
      a.beta, static_cast<Tin *>(a.o), a.S0, a.S_out, a.status, a.T);
  return cudaGetLastError();
}

#define KATA_INSTANTIATE_DELTA(DK, DV)                                          \
  template cudaError_t simt_delta<DK, DV, float>(const DeltaLaunch &);         \
  template cudaError_t simt_delta<DK, DV, __nv_bfloat16>(const DeltaLaunch &);
KATA_INSTANTIATE_DELTA(16, 16)
KATA_INSTANTIATE_DELTA(16, 32)
KATA_INSTANTIATE_DELTA(16, 64)
KATA_INSTANTIATE_DELTA(32, 16)
KATA_INSTANTIATE_DELTA(32, 32)
KATA_INSTANTIATE_DELTA(32, 64)

}  // namespace kata
