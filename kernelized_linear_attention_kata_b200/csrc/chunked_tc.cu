// Tensor-core (tcgen05 / TMEM / TMA) chunked-state forward for the rank-one
// PSD feature, bf16 inputs, fp32 accumulation: d_k = 32, d_v = 64, C = 128.
//
// The exact O(T) chunked form (KATA explainer section 2.3; arXiv abstract):
// for chunk c with state (S_c, Z_c) carried in from the earlier chunks
//   A    = (Q_c K_c^T)^2 masked to s <= t               intra-chunk block
//   num  = A V_c + phi_q(Q_c) S_c                       tcgen05.mma
//   den  = A 1   + q_t^T Z_c q_t                        (Z = sum k k^T, so
//                                                        q^T Z q = phi_q(q) . z)
//   y    = num / den                                    convex output gate
//   S_c+1 = S_c + phi(K_c)^T V_c,  Z_c+1 = Z_c + K_c^T K_c
// with phi(k) the 528 distinct products k_i k_j (i <= j) and phi_q(q) the same
// products of q with the off-diagonal multiplicity 2.
//
// Parallel carry: the sequence of every (b, h) is cut into G segments of
// whole chunks. A first launch (AGG = true) computes each segment's
// increment (sum of phi(K)^T V and K^T K over its chunks); the second launch
// gives segment g the sum of increments 0 .. g-1 as its carry-in and walks
// its chunks. G = 1 is the sequential carry.
//
// Feature order inside the kernel ("diagonal offset"): feature f = 32 d + l
// (d = 0..15, l = 0..31) is the pair (l, (l + d) mod 32); f = 512 + l
// (l < 16) is (l, l + 16). Every unordered pair i <= j appears once. The
// state is converted to the library's row-major (i <= j) order only where it
// leaves the kernel (S_out, z_out).
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM allocation and
// MMA issue (one lane), warps 2-5 math: thread r owns TMEM lane r, which is
// token r of the chunk for the token-major tiles and feature row r of each
// 128-feature state tile.
//
// Tensor memory (512 columns, fp32):
//   [  0, 320)  S, five 128-feature tiles of 64 columns (tile 4: 16 rows used)
//   [320, 352)  Z (lanes 0..31)
//   [352, 384)  U = Q_c Z_c (den of the inter-chunk part)
//   [384, 512)  Q_c K_c^T; then P (bf16, in place, [384, 448)) and O ([448, 512))
// Shared memory: two TMA stages of (Q, K, V) tiles, the bf16 snapshot of S_c
// (the readout's B operand) and of Z_c, and a two-slot ring of 128-feature
// phi tiles (the readout's A operand for Q, the update's A operand for K).
#include "common.cuh"
#include "launch.h"
#include "profile.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace kata {
namespace {

using namespace tc;

constexpr int kC = 128;            // chunk
constexpr int kDK = 32;
constexpr int kDV = 64;
constexpr int kD = 528;
constexpr int kTiles = 5;          // ceil(528 / 128)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColZ = 320, kColU = 352, kColX = 384, kColO = 448;
constexpr int kAggFloats = kD * kDV + kDK * kDK;      // one segment increment

// Shared memory layout (bytes from a 1024-aligned base).
constexpr int kStageBytes = 32768;                    // Q 8 KB | K 8 KB | V 16 KB
constexpr int kOffQ = 0, kOffK = 8192, kOffV = 16384;
constexpr int kOffStages = 0;
constexpr int kOffSnap = 2 * kStageBytes;             // S_c bf16 [528][64], 128 B rows
constexpr int kSnapBytes = kD * 128;
constexpr int kOffZSnap = kOffSnap + kSnapBytes;      // Z_c bf16 [32][32], 64 B rows
constexpr int kOffSlots = kOffZSnap + 2048;           // two 32 KB phi slots
constexpr int kSlotBytes = 32768;
constexpr int kOffBars = kOffSlots + 2 * kSlotBytes;
enum {
  kBarKvFull = 0, kBarKvEmpty = 2, kBarSFull = 4, kBarPFull, kBarOFull, kBarUpdFull, kBarXFree,
  kBarSnapFull, kBarSlotFull = 10, kBarSlotEmpty = 12, kNumBars = 14
};
constexpr int kOffTmemSlot = kOffBars + 8 * kNumBars;
constexpr int kOffAbort = kOffTmemSlot + 4;
constexpr int kSmemBytes = kOffAbort + 4 + 1024;      // + alignment slack
static_assert(kOffSnap % 1024 == 0 && kOffZSnap % 1024 == 0 && kOffSlots % 1024 == 0, "align");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-row tile
// with the 128-byte swizzle (atoms of 8 rows x 128 B).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}
// Same for 64-byte rows with the 64-byte swizzle.
__device__ __forceinline__ uint32_t sw64(int row, int chunk) {
  return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&a);
  __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162 *>(&b);
  __nv_bfloat162 r = __hmul2(x, y);
  return *reinterpret_cast<uint32_t *>(&r);
}

// Library (row-major i <= j) index of internal feature f.
__device__ __forceinline__ int abi_row(int f) {
  int a, b;
  if (f < 512) {
    a = f & 31;
    b = (a + (f >> 5)) & 31;
  } else {
    a = f - 512;
    b = a + 16;
  }
  const int i = a < b ? a : b, j = a < b ? b : a;
  return i * kDK - i * (i - 1) / 2 + (j - i);
}

// Writes the phi tile of slot s (features 128 s .. 128 s + 127) for one token
// row into a 32 KB slot (two 64-feature groups of 128-byte rows). P[l] holds
// the bf16 pair (x_l, x_(l+1) mod 32); M[l] is the multiplier pair for the
// partner index (x doubled off the diagonal on the query side).
template <bool QUERY>
__device__ __forceinline__ void write_phi_slot(uint8_t *slot, int row, int s, const uint32_t (&P)[32],
                                               const uint32_t (&P2)[32]) {
#pragma unroll
  for (int g2 = 0; g2 < 2; ++g2) {
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const int d = 4 * s + 2 * g2 + (cc >> 2);
      const int l0 = (cc & 3) * 8;
      if (s == 4 && (g2 != 0 || cc >= 2)) continue;         // only (16, l < 16) in slot 4
      uint4 v;
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int l = l0 + 2 * k;
        const int m = (l + d) & 31;
        w[k] = bmul2(P[l], (QUERY && d != 0) ? P2[m] : P[m]);
      }
      v.x = w[0];
      v.y = w[1];
      v.z = w[2];
      v.w = w[3];
      *reinterpret_cast<uint4 *>(slot + g2 * 16384 + sw128(row, cc)) = v;
    }
  }
}

// Pairs P[l] = (x_l, x_(l+1) mod 32) from a 64-byte row in the 64-byte swizzle.
__device__ __forceinline__ void load_pairs(const uint8_t *tile, int row, uint32_t (&X)[16],
                                           uint32_t (&P)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4 *>(tile + sw64(row, c));
    X[4 * c + 0] = v.x;
    X[4 * c + 1] = v.y;
    X[4 * c + 2] = v.z;
    X[4 * c + 3] = v.w;
  }
#pragma unroll
  for (int w = 0; w < 16; ++w) {
    P[2 * w] = X[w];
    P[2 * w + 1] = __byte_perm(X[w], X[(w + 1) & 15], 0x5432);
  }
}

template <bool AGG>
__global__ void __launch_bounds__(kThreads, 1)
chunked_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, __nv_bfloat16 *__restrict__ o,
                  float *__restrict__ agg, float *__restrict__ S_out, float *__restrict__ z_out,
                  unsigned *__restrict__ status, int T, int G_grid, int G_total, int seg_len) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffTmemSlot);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffAbort);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int g = blockIdx.x % G_grid;
  const int bh = blockIdx.x / G_grid;
  const int t0 = g * seg_len;
  const int t1 = min(T, t0 + seg_len);
  const int nchunks = (t1 - t0 + kC - 1) / kC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kBarKvFull + s], 1);
      mbar_init(&bars[kBarKvEmpty + s], 1 + 128);
      mbar_init(&bars[kBarSlotFull + s], 128);
      mbar_init(&bars[kBarSlotEmpty + s], 1);
    }
    mbar_init(&bars[kBarSFull], 1);
    mbar_init(&bars[kBarPFull], 128);
    mbar_init(&bars[kBarOFull], 1);
    mbar_init(&bars[kBarUpdFull], 1);
    mbar_init(&bars[kBarXFree], 128);
    mbar_init(&bars[kBarSnapFull], 128);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      if (!AGG) tma_prefetch_desc(&tmq);
      const uint32_t bytes = AGG ? 8192 + 16384 : 8192 * 2 + 16384;
      for (int i = 0; i < nchunks; ++i) {
        const int st = i & 1;
        if (i >= 2 && !mbar_wait(&bars[kBarKvEmpty + st], ((i >> 1) - 1) & 1, abort_flag)) break;
        uint8_t *stage = smem + kOffStages + st * kStageBytes;
        const int row = t0 + i * kC;
        mbar_arrive_expect_tx(&bars[kBarKvFull + st], bytes);
        if (!AGG) tma_load_3d(stage + kOffQ, &tmq, &bars[kBarKvFull + st], 0, row, bh);
        tma_load_3d(stage + kOffK, &tmk, &bars[kBarKvFull + st], 0, row, bh);
        tma_load_3d(stage + kOffV, &tmv, &bars[kBarKvFull + st], 0, row, bh);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t id_pv = idesc_bf16(128, kDV, false, true);
      constexpr uint32_t id_u = idesc_bf16(128, 32, false, false);
      constexpr uint32_t id_ro = idesc_bf16(128, kDV, false, true);
      constexpr uint32_t id_up = idesc_bf16(128, kDV, true, true);
      constexpr uint32_t id_z = idesc_bf16(128, 32, true, true);
      const uint32_t snap = smem_u32(smem + kOffSnap);
      const uint32_t zsnap = smem_u32(smem + kOffZSnap);
      const uint32_t slots = smem_u32(smem + kOffSlots);
      int u = 0;                                   // slot uses so far
      bool ok = true;
      for (int i = 0; ok && i < nchunks; ++i) {
        const int st = i & 1;
        const uint32_t stage = smem_u32(smem + kOffStages + st * kStageBytes);
        if (!(ok = mbar_wait(&bars[kBarKvFull + st], (i >> 1) & 1, abort_flag))) break;
        if (!AGG) {
          if (i > 0 && !(ok = mbar_wait(&bars[kBarXFree], (i - 1) & 1, abort_flag))) break;
          tc_fence_after();
          // S_qk = Q K^T  (both K-major, 64-byte swizzle)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(tbase + kColX, smem_desc(stage + kOffQ + 32 * kk, 16, 512, kSw64),
                   smem_desc(stage + kOffK + 32 * kk, 16, 512, kSw64), id_qk, kk);
          mma_commit(&bars[kBarSFull]);
          if (!(ok = mbar_wait(&bars[kBarPFull], i & 1, abort_flag))) break;
          tc_fence_after();
          // O = P V  (P from TMEM)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tbase + kColO, tbase + kColX + 8 * kk,
                   smem_desc(stage + kOffV + 2048 * kk, 16384, 1024, kSw128), id_pv, kk);
        }
        if ((!AGG || i == 0) && !(ok = mbar_wait(&bars[kBarSnapFull], i & 1, abort_flag))) break;
        tc_fence_after();
        if (!AGG) {
          // U = Q Z_c
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(tbase + kColU, smem_desc(stage + kOffQ + 32 * kk, 16, 512, kSw64),
                   smem_desc(zsnap + 32 * kk, 16, 512, kSw64), id_u, kk);
          // O += phi_q(Q) S_c, five feature slots
          for (int s = 0; s < kTiles && ok; ++s, ++u) {
            const int b = u & 1;
            if (!(ok = mbar_wait(&bars[kBarSlotFull + b], (u >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            const uint32_t slot = slots + b * kSlotBytes;
            const int nk = s == 4 ? 1 : 8;
            for (int kk = 0; kk < nk; ++kk) {
              const uint32_t a = slot + (kk >> 2) * 16384 + (kk & 3) * 32;
              mma_ss(tbase + kColO, smem_desc(a, 16, 1024, kSw128),
                     smem_desc(snap + (128 * s + 16 * kk) * 128, 16384, 1024, kSw128), id_ro, 1);
            }
            mma_commit(&bars[kBarSlotEmpty + b]);
          }
          if (!ok) break;
          mma_commit(&bars[kBarOFull]);
        }
        // S += phi(K)^T V, five feature tiles
        for (int m = 0; m < kTiles && ok; ++m, ++u) {
          const int b = u & 1;
          if (!(ok = mbar_wait(&bars[kBarSlotFull + b], (u >> 1) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t slot = slots + b * kSlotBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tbase + kColS + 64 * m, smem_desc(slot + 2048 * kk, 16384, 1024, kSw128),
                   smem_desc(stage + kOffV + 2048 * kk, 16384, 1024, kSw128), id_up, 1);
          mma_commit(&bars[kBarSlotEmpty + b]);
        }
        if (!ok) break;
        // Z += K^T K (A rows 32..127 alias other shared memory; unused lanes)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tbase + kColZ, smem_desc(stage + kOffK + 1024 * kk, 8192, 512, kSw64),
                 smem_desc(stage + kOffK + 1024 * kk, 8192, 512, kSw64), id_z, 1);
        mma_commit(&bars[kBarKvEmpty + st]);
        if (!AGG || i == nchunks - 1) mma_commit(&bars[kBarUpdFull]);
      }
    }
  } else {
    // ------------------------------------------------------------ math
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                    // TMEM lane / token / feature row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t *snap = smem + kOffSnap;
    uint8_t *zsnap = smem + kOffZSnap;
    bool ok = true;

    // ---- carry-in: sum of the increments of segments 0 .. g-1 ----
    {
      const float *seg0 = agg + (size_t)bh * G_total * kAggFloats;
      for (int m = 0; m < kTiles; ++m) {
        const int f = 128 * m + r;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {              // 16 columns at a time
          float acc[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[c] = 0.f;
          if (!AGG && f < kD) {
            for (int gp = 0; gp < g; ++gp) {
              const float4 *src =
                  reinterpret_cast<const float4 *>(seg0 + (size_t)gp * kAggFloats + f * kDV + 16 * q4);
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const float4 x = src[c4];
                acc[4 * c4 + 0] += x.x;
                acc[4 * c4 + 1] += x.y;
                acc[4 * c4 + 2] += x.z;
                acc[4 * c4 + 3] += x.w;
              }
            }
          }
          uint32_t bits[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) bits[c] = __float_as_uint(acc[c]);
          tmem_st16(tbase + lane_off + kColS + 64 * m + 16 * q4, bits);
          if (!AGG && f < kD) {
            uint4 v0, v1;
            v0.x = pack_bf16x2(acc[0], acc[1]);
            v0.y = pack_bf16x2(acc[2], acc[3]);
            v0.z = pack_bf16x2(acc[4], acc[5]);
            v0.w = pack_bf16x2(acc[6], acc[7]);
            v1.x = pack_bf16x2(acc[8], acc[9]);
            v1.y = pack_bf16x2(acc[10], acc[11]);
            v1.z = pack_bf16x2(acc[12], acc[13]);
            v1.w = pack_bf16x2(acc[14], acc[15]);
            *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4)) = v0;
            *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4 + 1)) = v1;
          }
        }
      }
      // Z rows live in lanes 0..31 (quarter 0); the other lanes hold zeros
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        float acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = 0.f;
        if (!AGG && r < kDK) {
          for (int gp = 0; gp < g; ++gp) {
            const float *src = seg0 + (size_t)gp * kAggFloats + kD * kDV + r * kDK + 16 * q2;
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[c] += src[c];
          }
        }
        uint32_t bits[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) bits[c] = __float_as_uint(acc[c]);
        tmem_st16(tbase + lane_off + kColZ + 16 * q2, bits);
        if (!AGG && r < kDK) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 v;
            v.x = pack_bf16x2(acc[8 * h + 0], acc[8 * h + 1]);
            v.y = pack_bf16x2(acc[8 * h + 2], acc[8 * h + 3]);
            v.z = pack_bf16x2(acc[8 * h + 4], acc[8 * h + 5]);
            v.w = pack_bf16x2(acc[8 * h + 6], acc[8 * h + 7]);
            *reinterpret_cast<uint4 *>(zsnap + sw64(r, 2 * q2 + h)) = v;
          }
        }
      }
      fence_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[kBarSnapFull]);
    }

    int u = 0;
    for (int i = 0; i < nchunks; ++i) {
      const int st = i & 1;
      uint8_t *stage = smem + kOffStages + st * kStageBytes;
      const int c0 = t0 + i * kC;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarKvFull + st], (i >> 1) & 1, abort_flag));
      if (!ok) break;
      float l_intra = 0.f;
      uint32_t XQ[16];
      if (!AGG) {
        // ---- intra-chunk block: P = (Q K^T)^2 masked, in place in TMEM ----
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarSFull], i & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t x[32];
          tmem_ld32(tbase + lane_off + kColX + 32 * c, x);
          tmem_wait_ld();
          uint32_t p[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int s0 = 32 * c + 2 * k;
            const float a0 = __uint_as_float(x[2 * k]);
            const float a1 = __uint_as_float(x[2 * k + 1]);
            float w0 = a0 * a0, w1 = a1 * a1;
            if (s0 > r || c0 + s0 >= T) w0 = 0.f;
            if (s0 + 1 > r || c0 + s0 + 1 >= T) w1 = 0.f;
            l_intra += w0 + w1;
            p[k] = pack_bf16x2(w0, w1);
          }
          tmem_st16(tbase + lane_off + kColX + 16 * c, p);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[kBarPFull]);

        // ---- phi_q(Q_c) slots ----
        uint32_t P[32], P2[32];
        load_pairs(stage + kOffQ, r, XQ, P);
#pragma unroll
        for (int l = 0; l < 32; ++l) P2[l] = bmul2(P[l], 0x40004000u);   // x 2 (bf16 2.0)
#pragma unroll
        for (int s = 0; s < kTiles; ++s) {
          const int us = u + s, b = us & 1;
          if (ok && us >= 2)
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars[kBarSlotEmpty + b], ((us >> 1) - 1) & 1, abort_flag));
          if (ok) {
            write_phi_slot<true>(smem + kOffSlots + b * kSlotBytes, r, s, P, P2);
            fence_async_smem();
            mbar_arrive(&bars[kBarSlotFull + b]);
          }
        }
        u += kTiles;
        if (!ok) break;
      }
      // ---- phi(K_c) slots ----
      {
        uint32_t XK[16], P[32];
        load_pairs(stage + kOffK, r, XK, P);
#pragma unroll
        for (int s = 0; s < kTiles; ++s) {
          const int us = u + s, b = us & 1;
          if (ok && us >= 2)
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars[kBarSlotEmpty + b], ((us >> 1) - 1) & 1, abort_flag));
          if (ok) {
            write_phi_slot<false>(smem + kOffSlots + b * kSlotBytes, r, s, P, P);
            fence_async_smem();
            mbar_arrive(&bars[kBarSlotFull + b]);
          }
        }
        u += kTiles;
        if (!ok) break;
      }
      mbar_arrive(&bars[kBarKvEmpty + st]);     // Q and K tiles no longer read here

      if (!AGG) {
        // ---- epilogue: y = (O) / (l_intra + q^T U) ----
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarOFull], i & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t uu[32];
        tmem_ld32(tbase + lane_off + kColU, uu);
        uint32_t oo[32], oo2[32];
        tmem_ld32(tbase + lane_off + kColO, oo);
        tmem_ld32(tbase + lane_off + kColO + 32, oo2);
        tmem_wait_ld();
        float den = l_intra;
#pragma unroll
        for (int w = 0; w < 16; ++w) {
          const __nv_bfloat162 qq = *reinterpret_cast<const __nv_bfloat162 *>(&XQ[w]);
          den = fmaf(__low2float(qq), __uint_as_float(uu[2 * w]), den);
          den = fmaf(__high2float(qq), __uint_as_float(uu[2 * w + 1]), den);
        }
        tc_fence_before();
        mbar_arrive(&bars[kBarXFree]);
        const int t = c0 + r;
        if (!(den > 0.f) && t < T) flag_status(status, kStatusNonPositiveNormaliser);
        if (t < T) {
          const float inv = 1.f / den;
          uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)bh * T + t) * kDV);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(oo[8 * q4 + 0]) * inv, __uint_as_float(oo[8 * q4 + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(oo[8 * q4 + 2]) * inv, __uint_as_float(oo[8 * q4 + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(oo[8 * q4 + 4]) * inv, __uint_as_float(oo[8 * q4 + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(oo[8 * q4 + 6]) * inv, __uint_as_float(oo[8 * q4 + 7]) * inv);
            dst[q4] = v;
          }
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(oo2[8 * q4 + 0]) * inv, __uint_as_float(oo2[8 * q4 + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(oo2[8 * q4 + 2]) * inv, __uint_as_float(oo2[8 * q4 + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(oo2[8 * q4 + 4]) * inv, __uint_as_float(oo2[8 * q4 + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(oo2[8 * q4 + 6]) * inv, __uint_as_float(oo2[8 * q4 + 7]) * inv);
            dst[4 + q4] = v;
          }
        }
      }

      // ---- wait for S_c+1, Z_c+1 (increments only need the final state) ----
      const bool last = i == nchunks - 1;
      if (AGG && !last) continue;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarUpdFull], AGG ? 0 : (i & 1), abort_flag));
      if (!ok) break;
      tc_fence_after();
      if (!last && !AGG) {
        // snapshot S_c+1 -> bf16 B operand of the next readout; Z_c+1 likewise
        for (int m = 0; m < kTiles; ++m) {
          if (m == 4 && quarter != 0) continue;          // tile 4: rows 512..527 (lanes 0..15)
          const int f = 128 * m + r;
          uint32_t a[32], b2[32];
          tmem_ld32(tbase + lane_off + kColS + 64 * m, a);
          tmem_ld32(tbase + lane_off + kColS + 64 * m + 32, b2);
          tmem_wait_ld();
          if (f < kD) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(a[8 * q4 + 0]), __uint_as_float(a[8 * q4 + 1]));
              v.y = pack_bf16x2(__uint_as_float(a[8 * q4 + 2]), __uint_as_float(a[8 * q4 + 3]));
              v.z = pack_bf16x2(__uint_as_float(a[8 * q4 + 4]), __uint_as_float(a[8 * q4 + 5]));
              v.w = pack_bf16x2(__uint_as_float(a[8 * q4 + 6]), __uint_as_float(a[8 * q4 + 7]));
              *reinterpret_cast<uint4 *>(snap + sw128(f, q4)) = v;
              uint4 v2;
              v2.x = pack_bf16x2(__uint_as_float(b2[8 * q4 + 0]), __uint_as_float(b2[8 * q4 + 1]));
              v2.y = pack_bf16x2(__uint_as_float(b2[8 * q4 + 2]), __uint_as_float(b2[8 * q4 + 3]));
              v2.z = pack_bf16x2(__uint_as_float(b2[8 * q4 + 4]), __uint_as_float(b2[8 * q4 + 5]));
              v2.w = pack_bf16x2(__uint_as_float(b2[8 * q4 + 6]), __uint_as_float(b2[8 * q4 + 7]));
              *reinterpret_cast<uint4 *>(snap + sw128(f, 4 + q4)) = v2;
            }
          }
        }
        if (quarter == 0) {
          uint32_t zr[32];
          tmem_ld32(tbase + lane_off + kColZ, zr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(zr[8 * c + 0]), __uint_as_float(zr[8 * c + 1]));
            v.y = pack_bf16x2(__uint_as_float(zr[8 * c + 2]), __uint_as_float(zr[8 * c + 3]));
            v.z = pack_bf16x2(__uint_as_float(zr[8 * c + 4]), __uint_as_float(zr[8 * c + 5]));
            v.w = pack_bf16x2(__uint_as_float(zr[8 * c + 6]), __uint_as_float(zr[8 * c + 7]));
            *reinterpret_cast<uint4 *>(zsnap + sw64(r, c)) = v;
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[kBarSnapFull]);
      }
    }

    // ---- state leaving the kernel ----
    const bool write_agg = AGG;
    const bool write_out = !AGG && g == G_total - 1 && (S_out || z_out);
    if (ok && nchunks > 0 && (write_agg || write_out)) {
      float *dst_agg = agg + ((size_t)bh * G_total + g) * kAggFloats;
      for (int m = 0; m < kTiles; ++m) {
        if (m == 4 && quarter != 0) continue;
        const int f = 128 * m + r;
        uint32_t a[32], b2[32];
        tmem_ld32(tbase + lane_off + kColS + 64 * m, a);
        tmem_ld32(tbase + lane_off + kColS + 64 * m + 32, b2);
        tmem_wait_ld();
        if (f < kD) {
          float *row = write_agg ? dst_agg + (size_t)f * kDV
                                 : (S_out ? S_out + ((size_t)bh * kD + abi_row(f)) * kDV : nullptr);
          if (row) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              *reinterpret_cast<float4 *>(row + c) =
                  make_float4(__uint_as_float(a[c]), __uint_as_float(a[c + 1]),
                              __uint_as_float(a[c + 2]), __uint_as_float(a[c + 3]));
              *reinterpret_cast<float4 *>(row + 32 + c) =
                  make_float4(__uint_as_float(b2[c]), __uint_as_float(b2[c + 1]),
                              __uint_as_float(b2[c + 2]), __uint_as_float(b2[c + 3]));
            }
          }
        }
      }
      if (quarter == 0) {
        uint32_t zr[32];
        tmem_ld32(tbase + lane_off + kColZ, zr);
        tmem_wait_ld();
        if (write_agg) {
          float *row = dst_agg + kD * kDV + r * kDK;
#pragma unroll
          for (int c = 0; c < 32; ++c) row[c] = __uint_as_float(zr[c]);
        } else if (z_out) {
          // z_(i,j) = Z_ij for i <= j; row r of Z gives the pairs (r, j >= r)
#pragma unroll
          for (int j = 0; j < kDK; ++j)
            if (j >= r)
              z_out[(size_t)bh * kD + r * kDK - r * (r - 1) / 2 + (j - r)] = __uint_as_float(zr[j]);
        }
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) flag_status(status, kStatusDeviceTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

}  // namespace

// Shapes handled by the tensor-core chunked forward.
bool tc_chunked_supported(const ChunkedLaunch &a, int d_k, int d_v, int C, int feature) {
  if (feature != kPSD || d_k != kDK || d_v != kDV || C != kC || a.T <= 0) return false;
  for (const void *p : {a.q, a.k, a.v, (const void *)a.o})
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return false;
  if ((a.S_out && reinterpret_cast<uintptr_t>(a.S_out) % 16) != 0) return false;
  if (a.seg_len % kC != 0) return false;
  return true;
}

size_t tc_chunked_agg_floats() { return (size_t)kAggFloats; }

cudaError_t tc_chunked(const ChunkedLaunch &a) {
  CUtensorMap tq, tk, tv;
  if (!make_tma_3d_bf16(&tq, a.q, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tk, a.k, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tv, a.v, kDV, a.T, a.BH, kC))
    return cudaErrorNotSupported;
  cudaError_t e;
  if (a.G > 1) {
    auto kagg = chunked_tc_kernel<true>;
    e = cudaFuncSetAttribute(kagg, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    ProfileScope prof("tc_segment_increment", a.stream);
    kagg<<<(unsigned)(a.BH * (a.G - 1)), kThreads, kSmemBytes, a.stream>>>(
        tq, tk, tv, static_cast<__nv_bfloat16 *>(a.o), a.agg, nullptr, nullptr, a.status, a.T,
        a.G - 1, a.G, a.seg_len);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  auto kpass = chunked_tc_kernel<false>;
  e = cudaFuncSetAttribute(kpass, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_segment_pass", a.stream);
  kpass<<<(unsigned)(a.BH * a.G), kThreads, kSmemBytes, a.stream>>>(
      tq, tk, tv, static_cast<__nv_bfloat16 *>(a.o), a.agg, a.S_out, a.z_out, a.status, a.T, a.G,
      a.G, a.seg_len);
  return cudaGetLastError();
}

}  // namespace kata
