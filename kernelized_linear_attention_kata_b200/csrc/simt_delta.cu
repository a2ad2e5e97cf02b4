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
// The weights between tokens come in closed form ((a . b)^2 for PSD).
//
// Every column of S' follows the rule on its own (the transition
// I - beta phi phi~^T acts on each column alike), so the columns are split
// over CTAs: CTA (b h, group) owns kCG value columns plus the normaliser
// column, which every group of a head recomputes (it divides the outputs).
// Each CTA walks its head's chunks in order; the delta rule does not add
// increments, so the sequence is not cut into segments.
//
// Per chunk (kDelThreads = 512, 16 warps):
//   1. phi~(k_t)^T S'_0 and phi~(q_t)^T S'_0: warp w takes the state rows
//      r = w mod 16 (every lane reads the same row: broadcasts), lane t the
//      token; the 16 partial sums go through shared memory. The weights
//      between the chunk's tokens in the same phase.
//   2. the triangular solve, one warp per column, lane t holding token t's
//      right-hand side in a register: after E_s is final (a shuffle from
//      lane s) every later lane subtracts its term (right-looking forward
//      substitution, kDC dependent steps); then the readout of the column.
//   3. y = readout / normaliser; S' += Phi(K)^T E, one (state row, four
//      columns) a thread.
//
// Shared memory (fp32): S' [D][kP] (the group's columns, z at column kCG,
// zero padding) | q, k [kDC][DK + 1] (odd stride: lanes on different tokens
// read different banks) | v [kDC][kCG] | the solve's right-hand sides, then E
// [kDC][kP] | the readouts [kDC][kP] | beta_t A_ts stored [s][t] and
// <phi~(q_t), phi(k_s)> stored [s][t] [kDC][kDC] each | beta [kDC] | the
// partial sums of phase 1 [16][kDC][2 kP] | the packed row table [D] (int4).
#include "launch.h"
#include "profile.h"
#include "simt_kernels.cuh"

namespace kata {
namespace {

constexpr int kDC = 32;                 // tokens per chunk (one per lane)
constexpr int kDelThreads = 512;
constexpr int kDelWarps = kDelThreads / 32;
constexpr int kCG = 8;                  // value columns per CTA
constexpr int kNC = kCG + 1;            // with the normaliser column
constexpr int kP = 12;                  // row stride of S' (float4 groups; zero padded)
static_assert(kNC <= kP && kP % 4 == 0, "state row stride");
static_assert(kNC <= kDelWarps, "one solve column per warp");

template <int DK>
struct DeltaSmem {
  static constexpr int D = state_dim(DK, kPSD);
  static constexpr int KS = DK + 1;     // q, k row stride
  static constexpr int S = 0;
  static constexpr int Q = S + D * kP;
  static constexpr int K = Q + kDC * KS;
  static constexpr int V = K + kDC * KS;
  static constexpr int E = V + kDC * kCG;
  static constexpr int R = E + kDC * kP;
  static constexpr int A = R + kDC * kP;
  static constexpr int B = A + kDC * kDC;
  static constexpr int BETA = B + kDC * kDC;
  static constexpr int PART = BETA + kDC;
  static constexpr int TAB = (PART + kDelWarps * kDC * 2 * kP + 3) / 4 * 4;   // int4 entries
  static constexpr size_t bytes() { return sizeof(float) * (size_t)(TAB + 4 * D); }
  static_assert(S % 4 == 0 && E % 4 == 0 && R % 4 == 0 && PART % 4 == 0, "float4 alignment");
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kDelThreads, 1)
delta_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
             const float *__restrict__ beta, Tin *__restrict__ o, const float *__restrict__ S0,
             float *__restrict__ S_out, unsigned *__restrict__ status, int T) {
  using L = DeltaSmem<DK>;
  constexpr int D = L::D, KS = L::KS, NG = DV / kCG, NCOL = DV + 1;
  extern __shared__ __align__(16) float sm[];
  float *Sa = sm + L::S, *qs = sm + L::Q, *ks = sm + L::K, *vs = sm + L::V;
  float *E = sm + L::E, *R = sm + L::R, *At = sm + L::A, *Bt = sm + L::B, *bs = sm + L::BETA;
  float *part = sm + L::PART;
  int4 *tab = reinterpret_cast<int4 *>(sm + L::TAB);
  const int bh = blockIdx.x / NG;
  const int c0 = (blockIdx.x % NG) * kCG;       // first value column of this CTA
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // state column c of this CTA: value column c0 + c for c < kCG, z for c = kCG
  auto gcol = [&](int c) { return c < kCG ? c0 + c : DV; };

  fill_row_table<DK, kPSD>(tab, tid, kDelThreads);
  for (int e = tid; e < D * kP; e += kDelThreads) {
    const int r = e / kP, c = e % kP;
    Sa[e] = (S0 && c < kNC) ? S0[((size_t)bh * D + r) * NCOL + gcol(c)] : 0.f;
  }
  const size_t qoff = (size_t)bh * T * DK, voff = (size_t)bh * T * DV;

  // The inputs of a chunk are fetched into registers one chunk ahead (their
  // global-memory latency hides behind the previous chunk's three phases)
  // and moved to shared memory at the chunk's start.
  constexpr int NQK = (kDC * DK + kDelThreads - 1) / kDelThreads;   // q, k values a thread
  static_assert(kDC * kCG <= kDelThreads && kDC <= kDelThreads, "one v value and one beta a thread");
  float pq[NQK], pk[NQK], pv = 0.f, pb = 0.f;
  auto fetch = [&](int tc) {                    // chunk starting at token tc
    const int nn = min(kDC, T - tc);
#pragma unroll
    for (int j = 0; j < NQK; ++j) {
      const int e = tid + j * kDelThreads;
      const int t = e / DK, i = e % DK;
      const bool in = e < kDC * DK && t < nn;
      pq[j] = in ? to_f(q[qoff + (size_t)(tc + t) * DK + i]) : 0.f;
      pk[j] = in ? to_f(k[qoff + (size_t)(tc + t) * DK + i]) : 0.f;
    }
    if (tid < kDC * kCG) {
      const int t = tid / kCG, c = tid % kCG;
      pv = t < nn ? to_f(v[voff + (size_t)(tc + t) * DV + c0 + c]) : 0.f;
    }
    if (tid < kDC) pb = tid < nn ? beta[(size_t)bh * T + tc + tid] : 0.f;
  };
  if (T > 0) fetch(0);

  for (int t0 = 0; t0 < T; t0 += kDC) {
    const int n = min(kDC, T - t0);
    __syncthreads();                            // previous chunk's readers are done
#pragma unroll
    for (int j = 0; j < NQK; ++j) {
      const int e = tid + j * kDelThreads;
      if (e < kDC * DK) {
        const int t = e / DK, i = e % DK;
        qs[t * KS + i] = pq[j];
        ks[t * KS + i] = pk[j];
      }
    }
    if (tid < kDC * kCG) vs[tid] = pv;
    if (tid < kDC) bs[tid] = pb;
    __syncthreads();
    if (t0 + kDC < T) fetch(t0 + kDC);          // the next chunk, in flight during this one

    // ---- phase 1: partial phi~(k_t)^T S'_0, phi~(q_t)^T S'_0 over rows r = warp mod 16 ----
    {
      const int t = lane;
      const float *kt = ks + t * KS, *qt = qs + t * KS;
      float ak[kP], aq[kP];
#pragma unroll
      for (int c = 0; c < kP; ++c) ak[c] = aq[c] = 0.f;
#pragma unroll 2
      for (int r = warp; r < D; r += kDelWarps) {
        const int4 e = tab[r];
        const float m = __int_as_float(e.z);
        const float fk = m * kt[e.x] * kt[e.y], fq = m * qt[e.x] * qt[e.y];
        const float4 *srow = reinterpret_cast<const float4 *>(Sa + r * kP);
#pragma unroll
        for (int g = 0; g < kP / 4; ++g) {
          const float4 s = srow[g];
          ak[4 * g + 0] = fmaf(fk, s.x, ak[4 * g + 0]);
          ak[4 * g + 1] = fmaf(fk, s.y, ak[4 * g + 1]);
          ak[4 * g + 2] = fmaf(fk, s.z, ak[4 * g + 2]);
          ak[4 * g + 3] = fmaf(fk, s.w, ak[4 * g + 3]);
          aq[4 * g + 0] = fmaf(fq, s.x, aq[4 * g + 0]);
          aq[4 * g + 1] = fmaf(fq, s.y, aq[4 * g + 1]);
          aq[4 * g + 2] = fmaf(fq, s.z, aq[4 * g + 2]);
          aq[4 * g + 3] = fmaf(fq, s.w, aq[4 * g + 3]);
        }
      }
      float4 *dst = reinterpret_cast<float4 *>(part + (warp * kDC + t) * 2 * kP);
#pragma unroll
      for (int g = 0; g < kP / 4; ++g) {
        dst[g] = make_float4(ak[4 * g], ak[4 * g + 1], ak[4 * g + 2], ak[4 * g + 3]);
        dst[kP / 4 + g] = make_float4(aq[4 * g], aq[4 * g + 1], aq[4 * g + 2], aq[4 * g + 3]);
      }
    }
    // weights between the chunk's tokens, stored [s][t]:
    //   At = beta_t (k_t . k_s)^2 for s < t, Bt = (q_t . k_s)^2 for s <= t
    for (int e = tid; e < kDC * kDC; e += kDelThreads) {
      const int s = e / kDC, t = e % kDC;
      float dk = 0.f, dq = 0.f;
#pragma unroll
      for (int i = 0; i < DK; ++i) {
        dk = fmaf(ks[t * KS + i], ks[s * KS + i], dk);
        dq = fmaf(qs[t * KS + i], ks[s * KS + i], dq);
      }
      At[e] = s < t ? bs[t] * dk * dk : 0.f;
      Bt[e] = s <= t ? dq * dq : 0.f;
    }
    __syncthreads();
    // sum of the partials: the solve's right-hand sides (E) and the readouts of S'_0 (R)
    for (int e = tid; e < kDC * kNC; e += kDelThreads) {
      const int t = e / kNC, c = e % kNC;
      float sk = 0.f, sq = 0.f;
#pragma unroll
      for (int w = 0; w < kDelWarps; ++w) {
        sk += part[(w * kDC + t) * 2 * kP + c];
        sq += part[(w * kDC + t) * 2 * kP + kP + c];
      }
      const float u = c < kCG ? vs[t * kCG + c] : 1.f;
      E[t * kP + c] = bs[t] * (u - sk);
      R[t * kP + c] = sq;
    }
    __syncthreads();

    // ---- phase 2: one warp per column: forward substitution, then the readout ----
    if (warp < kNC) {
      const int c = warp;
      float x = E[lane * kP + c];               // lane t: beta_t (u_t - phi~(k_t)^T S'_0)
#pragma unroll 8
      for (int s = 0; s < kDC; ++s) {
        const float es = __shfl_sync(0xffffffffu, x, s);   // E_s is final
        x = fmaf(-At[s * kDC + lane], es, x);
      }
      E[lane * kP + c] = x;
      float acc = R[lane * kP + c];
#pragma unroll 8
      for (int s = 0; s < kDC; ++s)
        acc = fmaf(Bt[s * kDC + lane], __shfl_sync(0xffffffffu, x, s), acc);
      R[lane * kP + c] = acc;
    }
    __syncthreads();

    // ---- phase 3: y = readout / normaliser; S' += Phi(K)^T E ----
    for (int e = tid; e < n * kCG; e += kDelThreads) {
      const int t = e / kCG, c = e % kCG;
      const float den = R[t * kP + kCG];
      if (c == 0 && c0 == 0 && !(den > 0.f)) flag_status(status, kStatusNonPositiveNormaliser);
      o[voff + (size_t)(t0 + t) * DV + c0 + c] = from_f<Tin>(R[t * kP + c] / den);
    }
    for (int e = tid; e < D * (kP / 4); e += kDelThreads) {
      const int r = e / (kP / 4), g = e % (kP / 4);
      const int4 te = tab[r];
      float4 acc = reinterpret_cast<const float4 *>(Sa + r * kP)[g];
#pragma unroll 8
      for (int t = 0; t < kDC; ++t) {
        const float ph = ks[t * KS + te.x] * ks[t * KS + te.y];
        const float4 x = reinterpret_cast<const float4 *>(E + t * kP)[g];
        acc.x = fmaf(ph, x.x, acc.x);
        acc.y = fmaf(ph, x.y, acc.y);
        acc.z = fmaf(ph, x.z, acc.z);
        acc.w = fmaf(ph, x.w, acc.w);
      }
      reinterpret_cast<float4 *>(Sa + r * kP)[g] = acc;
    }
  }
  __syncthreads();
  if (S_out) {
    // every group writes its value columns; group 0 also writes z
    for (int e = tid; e < D * kNC; e += kDelThreads) {
      const int r = e / kNC, c = e % kNC;
      if (c < kCG || c0 == 0) S_out[((size_t)bh * D + r) * NCOL + gcol(c)] = Sa[r * kP + c];
    }
  }
}

}  // namespace

template <int DK, int DV, typename Tin>
cudaError_t simt_delta(const DeltaLaunch &a) {
  static_assert(DV % kCG == 0, "value columns split in groups of kCG");
  using L = DeltaSmem<DK>;
  auto kern = delta_kernel<DK, DV, Tin>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::bytes());
  if (e != cudaSuccess) return e;
  ProfileScope prof("simt_delta", a.stream);
  kern<<<(unsigned)(a.BH * (DV / kCG)), kDelThreads, L::bytes(), a.stream>>>(
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
