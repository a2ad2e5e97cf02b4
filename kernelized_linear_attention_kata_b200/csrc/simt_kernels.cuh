// General-purpose CUDA-core (fp32 FFMA) kernels for every supported shape and
// both element types: the chunked forward (per-segment increments, then the
// segment pass with its carry-in), the quadratic forward and the decode step.
//
// These kernels carry the fp32 path (which must not be rounded through TF32
// or bf16 tensor-core inputs) and every shape the tensor-core kernels do not
// specialise. Arithmetic is fp32 throughout.
#pragma once

#include "common.cuh"

namespace kata {

// ---------------------------------------------------------------------------
// Tile loads (global -> shared, converted to fp32). Rows >= n are zeroed.
// ---------------------------------------------------------------------------
template <typename Tin, int COLS>
__device__ __forceinline__ void load_rows_f32(float *dst, const Tin *src, int n, int rows, int tid,
                                              int nthreads) {
  for (int e = tid; e < rows * COLS; e += nthreads) {
    int r = e / COLS;
    dst[e] = r < n ? to_f(src[e]) : 0.f;
  }
}

// ---------------------------------------------------------------------------
// Pass 1: per-segment state increments.
//   agg[bh][g] = ( sum_{t in segment g} phi(k_t) v_t^T , sum phi(k_t) )
// stored as D rows of (DV + 1) floats: DV columns of S, then z.
// One thread per state row; tokens streamed through shared memory.
// ---------------------------------------------------------------------------
constexpr int kAggTile = 64;

template <int DK, int DV, int FEAT, typename Tin>
__global__ void __launch_bounds__(576) segment_increment_kernel(const Tin *__restrict__ k, const Tin *__restrict__ v,
                                         float *__restrict__ agg, int T, int G_used, int G_total,
                                         int seg_len) {
  constexpr int D = state_dim(DK, FEAT);
  __shared__ __align__(16) float ks[kAggTile * DK];
  __shared__ __align__(16) float vs[kAggTile * DV];
  const int g = blockIdx.x % G_used;
  const int bh = blockIdx.x / G_used;
  const int t0 = g * seg_len;
  const int t1 = min(T, t0 + seg_len);
  const Tin *kb = k + (size_t)bh * T * DK;
  const Tin *vb = v + (size_t)bh * T * DV;

  const int r = threadIdx.x;
  int ri = 0, rj = 0;
  if (r < D) row_indices<DK, FEAT>(r, ri, rj);
  float acc[DV];
#pragma unroll
  for (int c = 0; c < DV; ++c) acc[c] = 0.f;
  float zacc = 0.f;

  for (int base = t0; base < t1; base += kAggTile) {
    const int n = min(kAggTile, t1 - base);
    __syncthreads();
    load_rows_f32<Tin, DK>(ks, kb + (size_t)base * DK, n, kAggTile, threadIdx.x, blockDim.x);
    load_rows_f32<Tin, DV>(vs, vb + (size_t)base * DV, n, kAggTile, threadIdx.x, blockDim.x);
    __syncthreads();
    if (r < D) {
      for (int t = 0; t < n; ++t) {
        const float ph = key_feature_row<DK, FEAT>(ks + t * DK, ri, rj);
        zacc += ph;
        const float4 *vr = reinterpret_cast<const float4 *>(vs + t * DV);
#pragma unroll
        for (int c4 = 0; c4 < DV / 4; ++c4) {
          float4 x = vr[c4];
          acc[4 * c4 + 0] = fmaf(ph, x.x, acc[4 * c4 + 0]);
          acc[4 * c4 + 1] = fmaf(ph, x.y, acc[4 * c4 + 1]);
          acc[4 * c4 + 2] = fmaf(ph, x.z, acc[4 * c4 + 2]);
          acc[4 * c4 + 3] = fmaf(ph, x.w, acc[4 * c4 + 3]);
        }
      }
    }
  }
  if (r < D) {
    float *dst = agg + (((size_t)bh * G_total + g) * D + r) * (DV + 1);
#pragma unroll
    for (int c = 0; c < DV; ++c) dst[c] = acc[c];
    dst[DV] = zacc;
  }
}

// ---------------------------------------------------------------------------
// Pass 2: one thread block per (b, h, segment). The carry-in is the initial
// state (if given) plus the increments of the earlier segments; the block then walks its chunks in
// order: intra-chunk block + readout of the carried state, then the state
// update, exactly the chunked-state recurrence.
//
// Shared memory: S [D][DV] fp32, z [D], q/k tiles [C][DK], v tile [C][DV].
// ---------------------------------------------------------------------------
constexpr int kSegThreads = 512;

// Shared-memory layout of the segment pass, in floats; every region starts
// on a 16-byte boundary (float4 reads of S rows and of the v tile):
//   S [D][DV] | z [D] | q tile [C][DK + 1] (row stride DK + 1 keeps each
//   thread's own row conflict-free) | k tile [C][DK] | v tile [C][DV] |
//   packed row table [D] of int4 (i, j, query multiplicity bits, -).
__host__ __device__ constexpr int round4(int x) { return (x + 3) / 4 * 4; }

template <int DK, int DV, int FEAT>
struct SegmentSmem {
  static constexpr int D = state_dim(DK, FEAT);
  static __host__ __device__ constexpr int z_off() { return D * DV; }
  static __host__ __device__ constexpr int q_off() { return z_off() + round4(D); }
  static __host__ __device__ constexpr int k_off(int C) { return q_off() + round4(C * (DK + 1)); }
  static __host__ __device__ constexpr int v_off(int C) { return k_off(C) + C * DK; }
  static __host__ __device__ constexpr int tab_off(int C) { return v_off(C) + C * DV; }
  static __host__ __device__ constexpr size_t bytes(int C) {
    return sizeof(float) * ((size_t)tab_off(C) + 4 * (size_t)D);
  }
};

template <int DK, int DV, int FEAT>
__host__ __device__ constexpr size_t segment_pass_smem(int C) {
  return SegmentSmem<DK, DV, FEAT>::bytes(C);
}

// Table of the packed state rows: (i, j, query multiplicity as float bits).
// First-order rows use i = r - 1 (i = -1 for the constant row).
template <int DK, int FEAT>
__device__ __forceinline__ void fill_row_table(int4 *tab, int tid, int nthreads) {
  constexpr int D = state_dim(DK, FEAT);
  for (int r = tid; r < D; r += nthreads) {
    int i, j;
    row_indices<DK, FEAT>(r, i, j);
    tab[r] = make_int4(i, j, __float_as_int(query_mult<FEAT>(i, j)), 0);
  }
}

// phi_q(q)_r for a row-table entry, q read from shared memory.
template <int DK, int FEAT>
__device__ __forceinline__ float query_feature_row(const float *qt, int4 e) {
  if constexpr (FEAT == kPSD || FEAT == kMg2) {
    return __int_as_float(e.z) * qt[e.x] * qt[e.y];
  } else if constexpr (FEAT == kSg2) {
    return __int_as_float(e.z) * fmaf(qt[e.x], qt[e.y], qt[DK / 2 + e.x] * qt[DK / 2 + e.y]);
  } else {
    return e.x < 0 ? 1.f : qt[e.x];
  }
}

template <int DK, int DV, int FEAT, typename Tin>
__global__ void __launch_bounds__(kSegThreads)
segment_pass_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                    const Tin *__restrict__ v, Tin *__restrict__ o,
                    const float *__restrict__ agg, const float *__restrict__ S0,
                    const float *__restrict__ z0, float *__restrict__ S_out,
                    float *__restrict__ z_out, unsigned *status, int T, int C, int G,
                    int seg_len) {
  constexpr int D = state_dim(DK, FEAT);
  constexpr int VB = 16;               // output columns per thread
  constexpr int NVB = DV / VB;
  extern __shared__ float4 smem_f4[];
  using L = SegmentSmem<DK, DV, FEAT>;
  float *S = reinterpret_cast<float *>(smem_f4);
  float *z = S + L::z_off();
  float *qs = S + L::q_off();           // [C][DK + 1]
  float *ks = S + L::k_off(C);
  float *vs = S + L::v_off(C);
  int4 *tab = reinterpret_cast<int4 *>(S + L::tab_off(C));

  const int g = blockIdx.x % G;
  const int bh = blockIdx.x / G;
  const int t0 = g * seg_len;
  const int t1 = min(T, t0 + seg_len);
  const int tid = threadIdx.x;
  fill_row_table<DK, FEAT>(tab, tid, kSegThreads);

  // carry-in: the initial state (if any) plus the exclusive prefix over the
  // earlier segments' increments
  for (int e = tid; e < D * (DV + 1); e += kSegThreads) {
    const int r = e / (DV + 1), c = e % (DV + 1);
    float s = 0.f;
    if (c < DV && S0) s = S0[((size_t)bh * D + r) * DV + c];
    if (c == DV && z0) s = z0[(size_t)bh * D + r];
    const float *src = agg + (size_t)bh * G * D * (DV + 1) + e;
    for (int gp = 0; gp < g; ++gp) s += src[(size_t)gp * D * (DV + 1)];
    if (c < DV) S[r * DV + c] = s;
    else z[r] = s;
  }

  const size_t qoff = (size_t)bh * T * DK;
  const size_t voff = (size_t)bh * T * DV;

  // state row owned by this thread during the update (rows tid, tid + 512)
  for (int c0 = t0; c0 < t1; c0 += C) {
    const int n = min(C, t1 - c0);
    __syncthreads();
    for (int e = tid; e < C * DK; e += kSegThreads) {
      const int r = e / DK, i = e % DK;
      qs[r * (DK + 1) + i] = r < n ? to_f(q[qoff + (size_t)c0 * DK + e]) : 0.f;
    }
    load_rows_f32<Tin, DK>(ks, k + qoff + (size_t)c0 * DK, n, C, tid, kSegThreads);
    load_rows_f32<Tin, DV>(vs, v + voff + (size_t)c0 * DV, n, C, tid, kSegThreads);
    __syncthreads();

    // ---- outputs of this chunk: intra block + readout of S_c ----
    for (int item = tid; item < C * NVB; item += kSegThreads) {
      const int t = item % C;
      const int vb = item / C;
      if (t >= n) continue;
      const float *qt = qs + t * (DK + 1);
      float acc[VB];
#pragma unroll
      for (int c = 0; c < VB; ++c) acc[c] = 0.f;
      float den = 0.f;
      // inter-chunk readout phi_q(q_t)^T S_c, phi_q(q_t)^T z_c
#pragma unroll 4
      for (int r = 0; r < D; ++r) {
        const float ph = query_feature_row<DK, FEAT>(qt, tab[r]);
        const float4 *sr = reinterpret_cast<const float4 *>(S + r * DV + vb * VB);
#pragma unroll
        for (int c4 = 0; c4 < VB / 4; ++c4) {
          float4 x = sr[c4];
          acc[4 * c4 + 0] = fmaf(ph, x.x, acc[4 * c4 + 0]);
          acc[4 * c4 + 1] = fmaf(ph, x.y, acc[4 * c4 + 1]);
          acc[4 * c4 + 2] = fmaf(ph, x.z, acc[4 * c4 + 2]);
          acc[4 * c4 + 3] = fmaf(ph, x.w, acc[4 * c4 + 3]);
        }
        den = fmaf(ph, z[r], den);
      }
      float qv[DK];
#pragma unroll
      for (int i = 0; i < DK; ++i) qv[i] = qt[i];
      // intra-chunk block: the weights of the keys s <= t (closed form)
      for (int s = 0; s <= t; ++s) {
        const float *kr = ks + s * DK;
        const float w = pair_weight<DK, FEAT>(qv, kr);
        den += w;
        const float4 *vr = reinterpret_cast<const float4 *>(vs + s * DV + vb * VB);
#pragma unroll
        for (int c4 = 0; c4 < VB / 4; ++c4) {
          float4 x = vr[c4];
          acc[4 * c4 + 0] = fmaf(w, x.x, acc[4 * c4 + 0]);
          acc[4 * c4 + 1] = fmaf(w, x.y, acc[4 * c4 + 1]);
          acc[4 * c4 + 2] = fmaf(w, x.z, acc[4 * c4 + 2]);
          acc[4 * c4 + 3] = fmaf(w, x.w, acc[4 * c4 + 3]);
        }
      }
      if (!(den > 0.f) && vb == 0) flag_status(status, kStatusNonPositiveNormaliser);
      const float inv = 1.f / den;
      Tin *orow = o + voff + (size_t)(c0 + t) * DV + vb * VB;
#pragma unroll
      for (int c = 0; c < VB; ++c) orow[c] = from_f<Tin>(acc[c] * inv);
    }
    __syncthreads();

    // ---- state update S += phi(K_c)^T V_c, z += phi(K_c)^T 1 ----
    for (int r = tid; r < D; r += kSegThreads) {
      int ri, rj;
      row_indices<DK, FEAT>(r, ri, rj);
      float acc[DV];
#pragma unroll
      for (int c = 0; c < DV; ++c) acc[c] = S[r * DV + c];
      float zacc = z[r];
      for (int t = 0; t < n; ++t) {
        const float ph = key_feature_row<DK, FEAT>(ks + t * DK, ri, rj);
        zacc += ph;
        const float4 *vr = reinterpret_cast<const float4 *>(vs + t * DV);
#pragma unroll
        for (int c4 = 0; c4 < DV / 4; ++c4) {
          float4 x = vr[c4];
          acc[4 * c4 + 0] = fmaf(ph, x.x, acc[4 * c4 + 0]);
          acc[4 * c4 + 1] = fmaf(ph, x.y, acc[4 * c4 + 1]);
          acc[4 * c4 + 2] = fmaf(ph, x.z, acc[4 * c4 + 2]);
          acc[4 * c4 + 3] = fmaf(ph, x.w, acc[4 * c4 + 3]);
        }
      }
#pragma unroll
      for (int c = 0; c < DV; ++c) S[r * DV + c] = acc[c];
      z[r] = zacc;
    }
  }
  __syncthreads();

  if (g == G - 1) {
    if (S_out) {
      float *dst = S_out + (size_t)bh * D * DV;
      for (int e = tid; e < D * DV; e += kSegThreads) dst[e] = S[e];
    }
    if (z_out) {
      float *dst = z_out + (size_t)bh * D;
      for (int e = tid; e < D; e += kSegThreads) dst[e] = z[e];
    }
  }
}

// ---------------------------------------------------------------------------
// Quadratic (flash-style) forward: one block per (b, h, 64-query block),
// key blocks up to the diagonal streamed through shared memory.
// ---------------------------------------------------------------------------
constexpr int kQuadBlock = 64;

template <int DK, int DV, int FEAT, typename Tin>
__global__ void quadratic_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                                 const Tin *__restrict__ v, Tin *__restrict__ o, int T) {
  constexpr int VB = 16;
  __shared__ __align__(16) float ks[kQuadBlock * DK];
  __shared__ __align__(16) float vs[kQuadBlock * DV];
  const int qb = blockIdx.x;
  const int bh = blockIdx.y;
  const int tl = threadIdx.x % kQuadBlock;
  const int vb = threadIdx.x / kQuadBlock;
  const int t = qb * kQuadBlock + tl;
  const size_t qoff = (size_t)bh * T * DK;
  const size_t voff = (size_t)bh * T * DV;

  float qv[DK];
#pragma unroll
  for (int i = 0; i < DK; ++i) qv[i] = t < T ? to_f(q[qoff + (size_t)t * DK + i]) : 0.f;
  float acc[VB];
#pragma unroll
  for (int c = 0; c < VB; ++c) acc[c] = 0.f;
  float den = 0.f;

  for (int kb = 0; kb <= qb; ++kb) {
    const int s0 = kb * kQuadBlock;
    const int n = min(kQuadBlock, T - s0);
    __syncthreads();
    load_rows_f32<Tin, DK>(ks, k + qoff + (size_t)s0 * DK, n, kQuadBlock, threadIdx.x, blockDim.x);
    load_rows_f32<Tin, DV>(vs, v + voff + (size_t)s0 * DV, n, kQuadBlock, threadIdx.x, blockDim.x);
    __syncthreads();
    const int smax = min(n, t - s0 + 1);   // keys s0 .. t within this block
    for (int s = 0; s < smax; ++s) {
      const float *kr = ks + s * DK;
      const float w = pair_weight<DK, FEAT>(qv, kr);
      den += w;
      const float4 *vr = reinterpret_cast<const float4 *>(vs + s * DV + vb * VB);
#pragma unroll
      for (int c4 = 0; c4 < VB / 4; ++c4) {
        float4 x = vr[c4];
        acc[4 * c4 + 0] = fmaf(w, x.x, acc[4 * c4 + 0]);
        acc[4 * c4 + 1] = fmaf(w, x.y, acc[4 * c4 + 1]);
        acc[4 * c4 + 2] = fmaf(w, x.z, acc[4 * c4 + 2]);
        acc[4 * c4 + 3] = fmaf(w, x.w, acc[4 * c4 + 3]);
      }
    }
  }
  if (t < T) {
    const float inv = 1.f / den;
    Tin *orow = o + voff + (size_t)t * DV + vb * VB;
#pragma unroll
    for (int c = 0; c < VB; ++c) orow[c] = from_f<Tin>(acc[c] * inv);
  }
}

// ---------------------------------------------------------------------------
// Decode step: one block per (b, h). The fp32 state is read, updated and
// written back once (HBM-bound); the readout is reduced in shared memory.
// ---------------------------------------------------------------------------
constexpr int kDecThreads = 256;

template <int DK, int DV, int FEAT, typename Tin>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              float *__restrict__ S, float *__restrict__ z, Tin *__restrict__ y) {
  constexpr int D = state_dim(DK, FEAT);
  constexpr int NC4 = DV / 4;                 // float4 columns per row
  constexpr int NRG = kDecThreads / NC4;      // row groups
  __shared__ __align__(16) float qf[DK], kf[DK], vf[DV];
  __shared__ float fk[D], fq[D];              // key feature, query feature (with multiplicity)
  __shared__ float4 red[NRG][NC4];
  __shared__ float den_red[kDecThreads / 32];

  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < DK) {
    qf[tid] = to_f(q[(size_t)bh * DK + tid]);
    kf[tid] = to_f(k[(size_t)bh * DK + tid]);
  }
  if (tid < DV) vf[tid] = to_f(v[(size_t)bh * DV + tid]);
  __syncthreads();
  for (int r = tid; r < D; r += kDecThreads) {
    int i, j;
    row_indices<DK, FEAT>(r, i, j);
    fk[r] = key_feature_row<DK, FEAT>(kf, i, j);
    fq[r] = key_feature_row<DK, FEAT>(qf, i, j) * query_mult<FEAT>(i, j);
  }
  __syncthreads();

  const int c4 = tid % NC4;
  const int rg = tid / NC4;
  const float4 vv = reinterpret_cast<const float4 *>(vf)[c4];
  float4 *Sb = reinterpret_cast<float4 *>(S + (size_t)bh * D * DV);
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int r = rg; r < D; r += NRG) {
    float4 s = Sb[r * NC4 + c4];
    const float a = fk[r];
    s.x = fmaf(a, vv.x, s.x);
    s.y = fmaf(a, vv.y, s.y);
    s.z = fmaf(a, vv.z, s.z);
    s.w = fmaf(a, vv.w, s.w);
    Sb[r * NC4 + c4] = s;
    const float b = fq[r];
    num.x = fmaf(b, s.x, num.x);
    num.y = fmaf(b, s.y, num.y);
    num.z = fmaf(b, s.z, num.z);
    num.w = fmaf(b, s.w, num.w);
  }
  red[rg][c4] = num;

  float dpart = 0.f;
  float *zb = z + (size_t)bh * D;
  for (int r = tid; r < D; r += kDecThreads) {
    const float zz = zb[r] + fk[r];
    zb[r] = zz;
    dpart = fmaf(fq[r], zz, dpart);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dpart += __shfl_xor_sync(0xffffffffu, dpart, off);
  if ((tid & 31) == 0) den_red[tid >> 5] = dpart;
  __syncthreads();

  if (tid < DV) {
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < kDecThreads / 32; ++w) den += den_red[w];
    const int cc = tid / 4, lane = tid % 4;
    float s = 0.f;
    for (int g = 0; g < NRG; ++g) {
      const float4 x = red[g][cc];
      s += lane == 0 ? x.x : lane == 1 ? x.y : lane == 2 ? x.z : x.w;
    }
    y[(size_t)bh * DV + tid] = from_f<Tin>(s / den);
  }
}

}  // namespace kata
