// CUDA-core (fp32 FFMA) kernels of the gradient of the chunked causal
// forward, for every supported shape and both element types.
//
// For L = sum_t dy_t . y_t, y_t = n_t / d_t (normalised causal linear
// attention, weights w_ts = phi_q(q_t) . phi(k_s) for s <= t; "線形注意"
// definition, KATA explainer 2.2 for the PSD weight <q, k>^2), let
//   g_t  = dy_t / d_t,   c_t = -(dy_t . y_t) / d_t,   e_ts = g_t . v_s + c_t
// (e_ts = dL/dw_ts). Then
//   dq_t = sum_{s<=t} e_ts dw_ts/dq_t = J_q(q_t)^T (S_t g_t + z_t c_t)
//   dk_s = sum_{t>=s} e_ts dw_ts/dk_s = J_k(k_s)^T (R_s v_s + r_s)
//   dv_s = sum_{t>=s} w_ts g_t        = R_s^T phi(k_s)
// with the forward's prefix state S_t = sum_{s<=t} phi(k_s) v_s^T,
// z_t = sum_{s<=t} phi(k_s), and the suffix state
// R_s = sum_{t>=s} phi_q(q_t) g_t^T, r_s = sum_{t>=s} phi_q(q_t) c_t.
// J_q, J_k are the Jacobians of the query and key features: for the packed
// PSD row (i, j) the feature m q_i q_j (m = 2 off the diagonal on the query
// side, 1 on the key side) sends m u q_j to entry i and m u q_i to entry j
// (2 u q_i when i = j); for the first-order row 1 + i the feature q_i sends
// u to entry i, and the constant row sends nothing.
//
// As in the forward's exact chunked form (explainer 2.3), each sum splits
// into the dense block inside a chunk and the state carried from the other
// chunks; the prefix state is carried forwards and the suffix state
// backwards, both through the forward's two-level segment scan:
//   1. segment_increment_kernel: the increments of (S, z) per segment;
//   2. bwd_dq_kernel: per segment, forwards: d_t and c_t (stored), dq;
//   3. bwd_increment_kernel: the increments of (R, r) per segment;
//   4. bwd_dkdv_kernel: per segment, backwards: dk, dv.
// The chunk inside these kernels is 64 tokens whatever the caller's C (the
// chunk size only schedules the exact form). Arithmetic is fp32 throughout;
// c_t is formed from the recomputed numerator, c_t = -(dy_t . n_t) / d_t^2,
// not from a stored (possibly bf16-rounded) forward output, whose rounding
// the cancellation in e_ts would amplify by 1 / d_t.
#pragma once

#include "launch.h"
#include "profile.h"
#include "simt_kernels.cuh"

namespace kata {

constexpr int kBwdThreads = 256;   // thread = (part 0..3, token 0..63): tid = 64 part + token
constexpr int kBwdChunk = 64;

// Shared memory of the two walking kernels, in floats (every region starts
// on a 16-byte boundary):
//   state [D][DV] (S or R) | vector [D] (z or r) | q, k tiles [64][DK + 1] |
//   v, g tiles [64][DV + 4] | c [64] | partial sums [8][64] |
//   per-thread partial gradients [256][DK + 1] | packed row pairs int [D].
// The padding keeps each thread's reads of its own token row conflict-free.
template <int DK, int DV, int FEAT>
struct BwdSmem {
  static constexpr int D = state_dim(DK, FEAT);
  static constexpr int QS = DK + 1;
  static constexpr int VS = DV + 4;
  static constexpr int kState = 0;
  static constexpr int kVec = kState + D * DV;
  static constexpr int kQ = kVec + round4(D);
  static constexpr int kK = kQ + round4(kBwdChunk * QS);
  static constexpr int kV = kK + round4(kBwdChunk * QS);
  static constexpr int kG = kV + kBwdChunk * VS;
  static constexpr int kC = kG + kBwdChunk * VS;
  static constexpr int kRed = kC + kBwdChunk;
  static constexpr int kAcc = kRed + 8 * kBwdChunk;
  static constexpr int kTab = kAcc + round4(kBwdThreads * (DK + 1));
  static constexpr size_t bytes = sizeof(float) * ((size_t)kTab + (size_t)round4(D));
  static_assert((D * DV) % 4 == 0 && VS % 4 == 0, "float4 rows");
};

// Packed row r -> (i, j) as one int: i in the low byte (signed: -1 is the
// first-order constant row), j in the next.
template <int DK, int FEAT>
__device__ __forceinline__ void fill_pair_table(int *tab, int tid, int nthreads) {
  constexpr int D = state_dim(DK, FEAT);
  for (int r = tid; r < D; r += nthreads) {
    int i, j;
    row_indices<DK, FEAT>(r, i, j);
    tab[r] = (i & 0xff) | (j << 8);
  }
}
__device__ __forceinline__ void unpack_pair(int e, int &i, int &j) {
  i = (int)(signed char)(e & 0xff);
  j = (e >> 8) & 0xff;
}

// w_ts from the two token rows.
template <int DK, int FEAT>
__device__ __forceinline__ float pair_weight(const float *qt, const float *ks) {
  float d0 = 0.f, d1 = 0.f;
#pragma unroll
  for (int a = 0; a < DK; a += 2) {
    d0 = fmaf(qt[a], ks[a], d0);
    d1 = fmaf(qt[a + 1], ks[a + 1], d1);
  }
  const float d = d0 + d1;
  return FEAT == kPSD ? d * d : 1.f + d;
}

// Loads one 64-token chunk: q, k into [64][DK + 1], v and dy into
// [64][DV + 4] (dy in the g tile); rows >= n are zero.
template <int DK, int DV, typename Tin>
__device__ __forceinline__ void bwd_load_chunk(float *qs, float *ks, float *vs, float *gs,
                                               const Tin *q, const Tin *k, const Tin *v,
                                               const Tin *dy, int n, int tid) {
  constexpr int QS = DK + 1, VS = DV + 4;
  for (int e = tid; e < kBwdChunk * DK; e += kBwdThreads) {
    const int r = e / DK, i = e % DK;
    const bool in = r < n;
    qs[r * QS + i] = in ? to_f(q[e]) : 0.f;
    ks[r * QS + i] = in ? to_f(k[e]) : 0.f;
  }
  for (int e = tid; e < kBwdChunk * DV; e += kBwdThreads) {
    const int r = e / DV, c = e % DV;
    const bool in = r < n;
    vs[r * VS + c] = in ? to_f(v[e]) : 0.f;
    gs[r * VS + c] = in ? to_f(dy[e]) : 0.f;
  }
}

// Sum of the four parts' partial gradients of each token of the chunk,
// written as rows of the output [.., DK].
template <int DK, typename Tin>
__device__ __forceinline__ void bwd_reduce_rows(const float *acc, Tin *out, int n, int tid) {
  for (int e = tid; e < kBwdChunk * DK; e += kBwdThreads) {
    const int t = e / DK, a = e % DK;
    if (t < n) {
      const float s = (acc[t * (DK + 1) + a] + acc[(64 + t) * (DK + 1) + a]) +
                      (acc[(128 + t) * (DK + 1) + a] + acc[(192 + t) * (DK + 1) + a]);
      out[(size_t)t * DK + a] = from_f<Tin>(s);
    }
  }
}

// state[r][:] += sum_t f_r(x_t) w_t and vec[r] += sum_t f_r(x_t) c_t over the
// chunk's tokens, f the key feature (mult = false) or the query feature with
// its multiplicity (mult = true); c may be null (then vec gets sum_t f_r).
// Item = (row, 16-column block).
template <int DK, int DV, int FEAT>
__device__ __forceinline__ void bwd_state_update(float *state, float *vec, const int *tab,
                                                 const float *xs, const float *ws, const float *cs,
                                                 bool mult, int n, int tid) {
  constexpr int D = state_dim(DK, FEAT);
  constexpr int QS = DK + 1, VS = DV + 4;
  for (int item = tid; item < D * (DV / 16); item += kBwdThreads) {
    const int r = item % D, cb = item / D;
    int i, j;
    unpack_pair(tab[r], i, j);
    const float m = mult ? query_mult<FEAT>(i, j) : 1.f;
    float4 *srow = reinterpret_cast<float4 *>(state + r * DV + cb * 16);
    float a[16];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const float4 x = srow[c4];
      a[4 * c4 + 0] = x.x;
      a[4 * c4 + 1] = x.y;
      a[4 * c4 + 2] = x.z;
      a[4 * c4 + 3] = x.w;
    }
    float va = 0.f;
    for (int t = 0; t < n; ++t) {
      const float f = m * key_feature_row<DK, FEAT>(xs + t * QS, i, j);
      va = fmaf(f, cs ? cs[t] : 1.f, va);
      const float4 *wr = reinterpret_cast<const float4 *>(ws + t * VS + cb * 16);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const float4 x = wr[c4];
        a[4 * c4 + 0] = fmaf(f, x.x, a[4 * c4 + 0]);
        a[4 * c4 + 1] = fmaf(f, x.y, a[4 * c4 + 1]);
        a[4 * c4 + 2] = fmaf(f, x.z, a[4 * c4 + 2]);
        a[4 * c4 + 3] = fmaf(f, x.w, a[4 * c4 + 3]);
      }
    }
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      srow[c4] = make_float4(a[4 * c4 + 0], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]);
    if (cb == 0) vec[r] += va;
  }
}

// ---------------------------------------------------------------------------
// 2. dq, walking each segment's chunks forwards from the carried (S, z).
//    Also stores every token's d_t and c_t for kernels 3 and 4.
// ---------------------------------------------------------------------------
template <int DK, int DV, int FEAT, typename Tin>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dq_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const Tin *__restrict__ dy, Tin *__restrict__ dq, const float *__restrict__ aggS,
              float *__restrict__ den_out, float *__restrict__ c_out, unsigned *status, int T,
              int G, int seg_len) {
  using L = BwdSmem<DK, DV, FEAT>;
  constexpr int D = L::D, QS = L::QS, VS = L::VS, CB = kBwdChunk;
  extern __shared__ float4 smem_f4[];
  float *sm = reinterpret_cast<float *>(smem_f4);
  float *S = sm + L::kState, *z = sm + L::kVec, *qs = sm + L::kQ, *ks = sm + L::kK;
  float *vs = sm + L::kV, *gs = sm + L::kG, *cs = sm + L::kC, *red = sm + L::kRed;
  float *acc = sm + L::kAcc;
  int *tab = reinterpret_cast<int *>(sm + L::kTab);

  const int g = blockIdx.x % G, bh = blockIdx.x / G;
  const int t0 = g * seg_len, t1 = min(T, t0 + seg_len);
  const int tid = threadIdx.x, part = tid >> 6, tl = tid & 63;
  float *mine = acc + tid * (DK + 1);
  fill_pair_table<DK, FEAT>(tab, tid, kBwdThreads);
  // carry-in: the increments of the earlier segments
  for (int e = tid; e < D * (DV + 1); e += kBwdThreads) {
    float s = 0.f;
    const float *src = aggS + (size_t)bh * G * D * (DV + 1) + e;
    for (int gp = 0; gp < g; ++gp) s += src[(size_t)gp * D * (DV + 1)];
    const int r = e / (DV + 1), c = e % (DV + 1);
    if (c < DV) S[r * DV + c] = s;
    else z[r] = s;
  }
  const size_t qo = (size_t)bh * T * DK, vo = (size_t)bh * T * DV;

  for (int c0 = t0; c0 < t1; c0 += CB) {
    const int n = min(CB, t1 - c0);
    const bool live = tl < n;
    __syncthreads();
    bwd_load_chunk<DK, DV, Tin>(qs, ks, vs, gs, q + qo + (size_t)c0 * DK, k + qo + (size_t)c0 * DK,
                                v + vo + (size_t)c0 * DV, dy + vo + (size_t)c0 * DV, n, tid);
#pragma unroll
    for (int a = 0; a <= DK; ++a) mine[a] = 0.f;
    __syncthreads();

    // ---- d_t = phi_q(q_t) . z_c + sum_{s<=t} w_ts and
    //      dy_t . n_t = phi_q(q_t) . (S_c dy_t) + sum_{s<=t} w_ts (dy_t . v_s) ----
    {
      float dp = 0.f, sp = 0.f;
      if (live) {
        const float *qt = qs + tl * QS;
        float dyr[DV];
        {
          const float4 *g4 = reinterpret_cast<const float4 *>(gs + tl * VS);
#pragma unroll
          for (int c4 = 0; c4 < DV / 4; ++c4) {
            const float4 x = g4[c4];
            dyr[4 * c4 + 0] = x.x;
            dyr[4 * c4 + 1] = x.y;
            dyr[4 * c4 + 2] = x.z;
            dyr[4 * c4 + 3] = x.w;
          }
        }
        for (int r = part; r < D; r += 4) {
          int i, j;
          unpack_pair(tab[r], i, j);
          const float f = query_mult<FEAT>(i, j) * key_feature_row<DK, FEAT>(qt, i, j);
          const float4 *sr = reinterpret_cast<const float4 *>(S + r * DV);
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
          for (int c4 = 0; c4 < DV / 4; ++c4) {
            const float4 x = sr[c4];
            a0 = fmaf(x.x, dyr[4 * c4 + 0], a0);
            a1 = fmaf(x.y, dyr[4 * c4 + 1], a1);
            a2 = fmaf(x.z, dyr[4 * c4 + 2], a2);
            a3 = fmaf(x.w, dyr[4 * c4 + 3], a3);
          }
          dp = fmaf(f, z[r], dp);
          sp = fmaf(f, (a0 + a1) + (a2 + a3), sp);
        }
        for (int s = part; s <= tl; s += 4) {
          const float w = pair_weight<DK, FEAT>(qt, ks + s * QS);
          const float4 *vr = reinterpret_cast<const float4 *>(vs + s * VS);
          float b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
#pragma unroll
          for (int c4 = 0; c4 < DV / 4; ++c4) {
            const float4 x = vr[c4];
            b0 = fmaf(x.x, dyr[4 * c4 + 0], b0);
            b1 = fmaf(x.y, dyr[4 * c4 + 1], b1);
            b2 = fmaf(x.z, dyr[4 * c4 + 2], b2);
            b3 = fmaf(x.w, dyr[4 * c4 + 3], b3);
          }
          dp += w;
          sp = fmaf(w, (b0 + b1) + (b2 + b3), sp);
        }
      }
      red[part * CB + tl] = dp;
      red[(4 + part) * CB + tl] = sp;
    }
    __syncthreads();
    const float den = (red[tl] + red[CB + tl]) + (red[2 * CB + tl] + red[3 * CB + tl]);
    const float dyn = (red[4 * CB + tl] + red[5 * CB + tl]) + (red[6 * CB + tl] + red[7 * CB + tl]);
    const float inv = live ? 1.f / den : 0.f;
    const float ct = -dyn * inv * inv;
    if (live && part == 0) {
      den_out[(size_t)bh * T + c0 + tl] = den;
      c_out[(size_t)bh * T + c0 + tl] = ct;
      if (!(den > 0.f)) flag_status(status, kStatusNonPositiveNormaliser);
    }
    float gr[DV];
    {
      const float4 *g4 = reinterpret_cast<const float4 *>(gs + tl * VS);
#pragma unroll
      for (int c4 = 0; c4 < DV / 4; ++c4) {
        const float4 x = g4[c4];
        gr[4 * c4 + 0] = x.x * inv;
        gr[4 * c4 + 1] = x.y * inv;
        gr[4 * c4 + 2] = x.z * inv;
        gr[4 * c4 + 3] = x.w * inv;
      }
    }

    if (live) {
      const float *qt = qs + tl * QS;
      // ---- carried part: J_q(q_t)^T (S_c g_t + z_c c_t), rows r = part mod 4 ----
      for (int r = part; r < D; r += 4) {
        const float4 *sr = reinterpret_cast<const float4 *>(S + r * DV);
        float u0 = z[r] * ct, u1 = 0.f, u2 = 0.f, u3 = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < DV / 4; ++c4) {
          const float4 x = sr[c4];
          u0 = fmaf(x.x, gr[4 * c4 + 0], u0);
          u1 = fmaf(x.y, gr[4 * c4 + 1], u1);
          u2 = fmaf(x.z, gr[4 * c4 + 2], u2);
          u3 = fmaf(x.w, gr[4 * c4 + 3], u3);
        }
        const float u = (u0 + u1) + (u2 + u3);
        int i, j;
        unpack_pair(tab[r], i, j);
        if constexpr (FEAT == kPSD) {
          const float mu = query_mult<FEAT>(i, j) * u;
          mine[i] = fmaf(mu, qt[j], mine[i]);
          mine[j] = fmaf(mu, qt[i], mine[j]);
        } else {
          if (i >= 0) mine[i] += u;
        }
      }
      // ---- in-chunk part: sum_{s<=t} e_ts dw_ts/dq_t, keys s = part mod 4 ----
      float dqi[DK];
#pragma unroll
      for (int a = 0; a < DK; ++a) dqi[a] = 0.f;
      for (int s = part; s < n; s += 4) {
        const float *kr = ks + s * QS;
        const float4 *vr = reinterpret_cast<const float4 *>(vs + s * VS);
        float e0 = ct, e1 = 0.f, e2 = 0.f, e3 = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < DV / 4; ++c4) {
          const float4 x = vr[c4];
          e0 = fmaf(gr[4 * c4 + 0], x.x, e0);
          e1 = fmaf(gr[4 * c4 + 1], x.y, e1);
          e2 = fmaf(gr[4 * c4 + 2], x.z, e2);
          e3 = fmaf(gr[4 * c4 + 3], x.w, e3);
        }
        float coef = (e0 + e1) + (e2 + e3);
        if constexpr (FEAT == kPSD) {
          float d0 = 0.f, d1 = 0.f;
#pragma unroll
          for (int a = 0; a < DK; a += 2) {
            d0 = fmaf(qt[a], kr[a], d0);
            d1 = fmaf(qt[a + 1], kr[a + 1], d1);
          }
          coef *= 2.f * (d0 + d1);
        }
        coef = s <= tl ? coef : 0.f;
#pragma unroll
        for (int a = 0; a < DK; ++a) dqi[a] = fmaf(coef, kr[a], dqi[a]);
      }
#pragma unroll
      for (int a = 0; a < DK; ++a) mine[a] += dqi[a];
    }
    __syncthreads();
    bwd_reduce_rows<DK, Tin>(acc, dq + qo + (size_t)c0 * DK, n, tid);
    // ---- S += phi(K_c)^T V_c, z += phi(K_c)^T 1 ----
    bwd_state_update<DK, DV, FEAT>(S, z, tab, ks, vs, nullptr, false, n, tid);
  }
}

// ---------------------------------------------------------------------------
// 3. Per-segment increments of the suffix state, segments 1 .. G-1:
//    aggR[bh][g] = ( sum_{t in g} phi_q(q_t) g_t^T , sum_{t in g} phi_q(q_t) c_t )
//    as D rows of (DV + 1) floats. One thread per state row.
// ---------------------------------------------------------------------------
template <int DK, int DV, int FEAT, typename Tin>
__global__ void __launch_bounds__(576)
bwd_increment_kernel(const Tin *__restrict__ q, const Tin *__restrict__ dy,
                     const float *__restrict__ den_in, const float *__restrict__ c_in,
                     float *__restrict__ aggR, int T, int G, int seg_len) {
  constexpr int D = state_dim(DK, FEAT);
  __shared__ __align__(16) float qsh[kAggTile * DK];
  __shared__ __align__(16) float gsh[kAggTile * DV];
  __shared__ float csh[kAggTile], invsh[kAggTile];
  const int g = 1 + (int)(blockIdx.x % (G - 1));
  const int bh = blockIdx.x / (G - 1);
  const int t0 = g * seg_len, t1 = min(T, t0 + seg_len);
  const size_t qo = (size_t)bh * T * DK, vo = (size_t)bh * T * DV;
  const int r = threadIdx.x;
  int ri = 0, rj = 0;
  if (r < D) row_indices<DK, FEAT>(r, ri, rj);
  const float m = query_mult<FEAT>(ri, rj);
  float acc[DV];
#pragma unroll
  for (int c = 0; c < DV; ++c) acc[c] = 0.f;
  float racc = 0.f;

  for (int base = t0; base < t1; base += kAggTile) {
    const int n = min(kAggTile, t1 - base);
    __syncthreads();
    for (int t = threadIdx.x; t < kAggTile; t += blockDim.x) {
      const bool in = t < n;
      invsh[t] = in ? 1.f / den_in[(size_t)bh * T + base + t] : 0.f;
      csh[t] = in ? c_in[(size_t)bh * T + base + t] : 0.f;
    }
    load_rows_f32<Tin, DK>(qsh, q + qo + (size_t)base * DK, n, kAggTile, threadIdx.x, blockDim.x);
    __syncthreads();
    for (int e = threadIdx.x; e < kAggTile * DV; e += blockDim.x) {
      const int t = e / DV;
      gsh[e] = t < n ? to_f(dy[vo + (size_t)base * DV + e]) * invsh[t] : 0.f;
    }
    __syncthreads();
    if (r < D) {
      for (int t = 0; t < n; ++t) {
        const float f = m * key_feature_row<DK, FEAT>(qsh + t * DK, ri, rj);
        racc = fmaf(f, csh[t], racc);
        const float4 *gr = reinterpret_cast<const float4 *>(gsh + t * DV);
#pragma unroll
        for (int c4 = 0; c4 < DV / 4; ++c4) {
          const float4 x = gr[c4];
          acc[4 * c4 + 0] = fmaf(f, x.x, acc[4 * c4 + 0]);
          acc[4 * c4 + 1] = fmaf(f, x.y, acc[4 * c4 + 1]);
          acc[4 * c4 + 2] = fmaf(f, x.z, acc[4 * c4 + 2]);
          acc[4 * c4 + 3] = fmaf(f, x.w, acc[4 * c4 + 3]);
        }
      }
    }
  }
  if (r < D) {
    float *dst = aggR + (((size_t)bh * G + g) * D + r) * (DV + 1);
#pragma unroll
    for (int c = 0; c < DV; ++c) dst[c] = acc[c];
    dst[DV] = racc;
  }
}

// ---------------------------------------------------------------------------
// 4. dk and dv, walking each segment's chunks backwards from the carried
//    suffix state (R, r) of the later segments.
// ---------------------------------------------------------------------------
template <int DK, int DV, int FEAT, typename Tin>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dkdv_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                const Tin *__restrict__ dy, Tin *__restrict__ dk, Tin *__restrict__ dv,
                const float *__restrict__ aggR, const float *__restrict__ den_in,
                const float *__restrict__ c_in, int T, int G, int seg_len) {
  using L = BwdSmem<DK, DV, FEAT>;
  constexpr int D = L::D, QS = L::QS, VS = L::VS, CB = kBwdChunk;
  constexpr int NV = DV / 4;                  // dv columns of one part
  extern __shared__ float4 smem_f4[];
  float *sm = reinterpret_cast<float *>(smem_f4);
  float *R = sm + L::kState, *rv = sm + L::kVec, *qs = sm + L::kQ, *ks = sm + L::kK;
  float *vs = sm + L::kV, *gs = sm + L::kG, *cs = sm + L::kC, *red = sm + L::kRed;
  float *acc = sm + L::kAcc;
  int *tab = reinterpret_cast<int *>(sm + L::kTab);

  const int g = blockIdx.x % G, bh = blockIdx.x / G;
  const int t0 = g * seg_len, t1 = min(T, t0 + seg_len);
  const int tid = threadIdx.x, part = tid >> 6, tl = tid & 63;
  float *mine = acc + tid * (DK + 1);
  fill_pair_table<DK, FEAT>(tab, tid, kBwdThreads);
  // carry-in: the increments of the later segments
  for (int e = tid; e < D * (DV + 1); e += kBwdThreads) {
    float s = 0.f;
    const float *src = aggR + (size_t)bh * G * D * (DV + 1) + e;
    for (int gp = g + 1; gp < G; ++gp) s += src[(size_t)gp * D * (DV + 1)];
    const int r = e / (DV + 1), c = e % (DV + 1);
    if (c < DV) R[r * DV + c] = s;
    else rv[r] = s;
  }
  const size_t qo = (size_t)bh * T * DK, vo = (size_t)bh * T * DV;
  const int nch = (t1 - t0 + CB - 1) / CB;

  for (int ci = nch - 1; ci >= 0; --ci) {
    const int c0 = t0 + ci * CB;
    const int n = min(CB, t1 - c0);
    const bool live = tl < n;
    __syncthreads();
    bwd_load_chunk<DK, DV, Tin>(qs, ks, vs, gs, q + qo + (size_t)c0 * DK, k + qo + (size_t)c0 * DK,
                                v + vo + (size_t)c0 * DV, dy + vo + (size_t)c0 * DV, n, tid);
#pragma unroll
    for (int a = 0; a <= DK; ++a) mine[a] = 0.f;
    __syncthreads();
    // ---- g_t = dy_t / d_t in the g tile; c_t from kernel 2 ----
    {
      const float inv = live ? 1.f / den_in[(size_t)bh * T + c0 + tl] : 0.f;
      if (part == 0) cs[tl] = live ? c_in[(size_t)bh * T + c0 + tl] : 0.f;
      for (int c = part * NV; c < (part + 1) * NV; ++c) gs[tl * VS + c] *= inv;
    }
    __syncthreads();

    if (live) {
      const float *kt = ks + tl * QS;
      float vr[DV];
      {
        const float4 *v4 = reinterpret_cast<const float4 *>(vs + tl * VS);
#pragma unroll
        for (int c4 = 0; c4 < DV / 4; ++c4) {
          const float4 x = v4[c4];
          vr[4 * c4 + 0] = x.x;
          vr[4 * c4 + 1] = x.y;
          vr[4 * c4 + 2] = x.z;
          vr[4 * c4 + 3] = x.w;
        }
      }
      // ---- carried part of dk: J_k(k_s)^T (R_c v_s + r_c), rows r = part mod 4 ----
      for (int r = part; r < D; r += 4) {
        const float4 *rr = reinterpret_cast<const float4 *>(R + r * DV);
        float w0 = rv[r], w1 = 0.f, w2 = 0.f, w3 = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < DV / 4; ++c4) {
          const float4 x = rr[c4];
          w0 = fmaf(x.x, vr[4 * c4 + 0], w0);
          w1 = fmaf(x.y, vr[4 * c4 + 1], w1);
          w2 = fmaf(x.z, vr[4 * c4 + 2], w2);
          w3 = fmaf(x.w, vr[4 * c4 + 3], w3);
        }
        const float w = (w0 + w1) + (w2 + w3);
        int i, j;
        unpack_pair(tab[r], i, j);
        if constexpr (FEAT == kPSD) {
          mine[i] = fmaf(w, kt[j], mine[i]);
          mine[j] = fmaf(w, kt[i], mine[j]);
        } else {
          if (i >= 0) mine[i] += w;
        }
      }
      // ---- in-chunk part of dk: sum_{t>=s} e_ts dw_ts/dk_s, queries t = part mod 4 ----
      float dki[DK];
#pragma unroll
      for (int a = 0; a < DK; ++a) dki[a] = 0.f;
      for (int t = part; t < n; t += 4) {
        const float *qt = qs + t * QS;
        const float4 *gt = reinterpret_cast<const float4 *>(gs + t * VS);
        float e0 = cs[t], e1 = 0.f, e2 = 0.f, e3 = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < DV / 4; ++c4) {
          const float4 x = gt[c4];
          e0 = fmaf(vr[4 * c4 + 0], x.x, e0);
          e1 = fmaf(vr[4 * c4 + 1], x.y, e1);
          e2 = fmaf(vr[4 * c4 + 2], x.z, e2);
          e3 = fmaf(vr[4 * c4 + 3], x.w, e3);
        }
        float coef = (e0 + e1) + (e2 + e3);
        if constexpr (FEAT == kPSD) {
          float d0 = 0.f, d1 = 0.f;
#pragma unroll
          for (int a = 0; a < DK; a += 2) {
            d0 = fmaf(kt[a], qt[a], d0);
            d1 = fmaf(kt[a + 1], qt[a + 1], d1);
          }
          coef *= 2.f * (d0 + d1);
        }
        coef = t >= tl ? coef : 0.f;
#pragma unroll
        for (int a = 0; a < DK; ++a) dki[a] = fmaf(coef, qt[a], dki[a]);
      }
#pragma unroll
      for (int a = 0; a < DK; ++a) mine[a] += dki[a];
    }
    __syncthreads();
    bwd_reduce_rows<DK, Tin>(acc, dk + qo + (size_t)c0 * DK, n, tid);

    // ---- dv_s = R_c^T phi(k_s) + sum_{t>=s} w_ts g_t, this part's NV columns ----
    if (live) {
      const float *kt = ks + tl * QS;
      float dvr[NV];
#pragma unroll
      for (int c = 0; c < NV; ++c) dvr[c] = 0.f;
      for (int r = 0; r < D; ++r) {
        int i, j;
        unpack_pair(tab[r], i, j);
        const float f = key_feature_row<DK, FEAT>(kt, i, j);
        const float4 *rr = reinterpret_cast<const float4 *>(R + r * DV + part * NV);
#pragma unroll
        for (int c4 = 0; c4 < NV / 4; ++c4) {
          const float4 x = rr[c4];
          dvr[4 * c4 + 0] = fmaf(f, x.x, dvr[4 * c4 + 0]);
          dvr[4 * c4 + 1] = fmaf(f, x.y, dvr[4 * c4 + 1]);
          dvr[4 * c4 + 2] = fmaf(f, x.z, dvr[4 * c4 + 2]);
          dvr[4 * c4 + 3] = fmaf(f, x.w, dvr[4 * c4 + 3]);
        }
      }
      for (int t = 0; t < n; ++t) {
        float w = pair_weight<DK, FEAT>(qs + t * QS, kt);
        w = t >= tl ? w : 0.f;
        const float4 *gt = reinterpret_cast<const float4 *>(gs + t * VS + part * NV);
#pragma unroll
        for (int c4 = 0; c4 < NV / 4; ++c4) {
          const float4 x = gt[c4];
          dvr[4 * c4 + 0] = fmaf(w, x.x, dvr[4 * c4 + 0]);
          dvr[4 * c4 + 1] = fmaf(w, x.y, dvr[4 * c4 + 1]);
          dvr[4 * c4 + 2] = fmaf(w, x.z, dvr[4 * c4 + 2]);
          dvr[4 * c4 + 3] = fmaf(w, x.w, dvr[4 * c4 + 3]);
        }
      }
      Tin *drow = dv + vo + (size_t)(c0 + tl) * DV + part * NV;
#pragma unroll
      for (int c = 0; c < NV; ++c) drow[c] = from_f<Tin>(dvr[c]);
    }
    __syncthreads();
    // ---- R += phi_q(Q_c)^T G_c, r += phi_q(Q_c)^T c ----
    bwd_state_update<DK, DV, FEAT>(R, rv, tab, qs, gs, cs, true, n, tid);
  }
}

// The suffix half of the backward (launches 3 and 4): the suffix-state
// increments and the dk, dv walk, from the d_t and c_t of the dq pass.
template <int DK, int DV, int FEAT, typename Tin>
cudaError_t simt_backward_dkdv(const BackwardLaunch &a) {
  constexpr int D = state_dim(DK, FEAT);
  const Tin *q = static_cast<const Tin *>(a.q);
  const Tin *k = static_cast<const Tin *>(a.k);
  const Tin *v = static_cast<const Tin *>(a.v);
  const Tin *dy = static_cast<const Tin *>(a.dout);
  const int inc_threads = (D + 31) / 32 * 32;
  constexpr size_t smem = BwdSmem<DK, DV, FEAT>::bytes;
  cudaError_t e;
  if (a.G > 1) {
    ProfileScope prof("simt_bwd_suffix_increment", a.stream);
    bwd_increment_kernel<DK, DV, FEAT, Tin>
        <<<(unsigned)(a.BH * (a.G - 1)), inc_threads, 0, a.stream>>>(q, dy, a.den, a.c, a.aggR, a.T,
                                                                      a.G, a.seg_len);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  auto kern = bwd_dkdv_kernel<DK, DV, FEAT, Tin>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  ProfileScope prof("simt_bwd_dkdv", a.stream);
  kern<<<(unsigned)(a.BH * a.G), kBwdThreads, smem, a.stream>>>(
      q, k, v, dy, static_cast<Tin *>(a.dk), static_cast<Tin *>(a.dv), a.aggR, a.den, a.c, a.T, a.G,
      a.seg_len);
  return cudaGetLastError();
}

template <int DK, int DV, int FEAT, typename Tin>
cudaError_t simt_backward(const BackwardLaunch &a) {
  constexpr int D = state_dim(DK, FEAT);
  const Tin *q = static_cast<const Tin *>(a.q);
  const Tin *k = static_cast<const Tin *>(a.k);
  const Tin *v = static_cast<const Tin *>(a.v);
  const Tin *dy = static_cast<const Tin *>(a.dout);
  const int inc_threads = (D + 31) / 32 * 32;
  constexpr size_t smem = BwdSmem<DK, DV, FEAT>::bytes;
  cudaError_t e;
  if (a.G > 1) {
    ProfileScope prof("simt_bwd_prefix_increment", a.stream);
    segment_increment_kernel<DK, DV, FEAT, Tin>
        <<<(unsigned)(a.BH * (a.G - 1)), inc_threads, 0, a.stream>>>(k, v, a.aggS, a.T, a.G - 1, a.G,
                                                                      a.seg_len);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    auto kern = bwd_dq_kernel<DK, DV, FEAT, Tin>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return e;
    ProfileScope prof("simt_bwd_dq", a.stream);
    kern<<<(unsigned)(a.BH * a.G), kBwdThreads, smem, a.stream>>>(
        q, k, v, dy, static_cast<Tin *>(a.dq), a.aggS, a.den, a.c, a.status, a.T, a.G, a.seg_len);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return simt_backward_dkdv<DK, DV, FEAT, Tin>(a);
}

#define KATA_INSTANTIATE_BACKWARD(DK, DV, FEAT, TIN)                              \
  template cudaError_t simt_backward<DK, DV, FEAT, TIN>(const BackwardLaunch &);    \
  template cudaError_t simt_backward_dkdv<DK, DV, FEAT, TIN>(const BackwardLaunch &);

}  // namespace kata
