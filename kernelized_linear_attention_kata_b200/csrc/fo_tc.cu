// Tensor-core (tcgen05 / TMEM / TMA) chunked-state forward for the
// first-order feature, bf16 inputs, fp32 accumulation: d_k = d_v = 64.
//
// The first-order (Lorentz) feature phi(u) = [1, u] gives the weight
// 1 + q . k (first-order reading of the arXiv abstract; KATA explainer
// sections 2.1 and 2.3 for the chunked form and its scan). With the ones
// column appended to V, one accumulator carries numerator and normaliser:
//
//   S' = [K | 1]^T [V | 1]          (65 x 65: rows k_1..k_64 and the constant
//                                    feature; columns v_1..v_64 and the count)
//   O' = P [V | 1] + [Q | 1] S'_c   with P = (1 + Q K^T) masked to s <= t
//   y  = O'[:, 0:64] / O'[:, 64]    (the convex output gate)
//
// so a tile of 128 tokens is five MMA streams of N = 80 (65 columns padded to
// a multiple of 16) and one of N = 128 (Q K^T). The chunk size C of the
// exact chunked form only schedules the work: C = 64 and C = 128 both run
// on 128-token tiles (the result is the same up to rounding).
//
// Parallel carry as in the PSD kernel: a first launch (AGG) computes each
// segment's increment of S', the second gives segment g the sum of the
// increments of segments 0 .. g-1 as its carry-in.
//
// Warp roles (352 threads): warp 0 TMA (Q, K, V, three stages each); warp 1
// TMEM allocation and the MMAs of Q K^T, P V and the readout (in the
// increment kernel, the update); warp 10 the update of S' in the pass (one
// thread issues an MMA only every ~80 cycles, so the two streams go
// side by side); warps 2-5 the query side (P); warps 6-9 the state side (the
// bf16 snapshot of S' after each update, the epilogue and the TMA store of
// y, the carry-in, the state written out). The readout of tile i reads the
// snapshot of S'_i, so the snapshot of S'_i+1 (double-buffered) is taken
// while it runs. Math thread r owns TMEM lane r: token r of the tile, or
// feature row r of S'.
//
// Tensor memory (512 columns): S' [0, 80) (lanes 0..64 used), O' [128, 208),
// Q K^T of even / odd tiles [256, 384) / [384, 512) (P in place as bf16).
#include "common.cuh"
#include "launch.h"
#include "profile.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace kata {
namespace {

using namespace tc;

constexpr int kTile = 128;         // tokens per tile
constexpr int kDh = 64;            // d_k = d_v
constexpr int kNa = 80;            // augmented width (65 padded to a multiple of 16)
constexpr int kRows = 65;          // rows / columns of S' that carry data
constexpr int kThreads = 352;      // 11 warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 128, kColX = 256;   // X of tile i at kColX + 128 (i & 1)
constexpr int kAggFloats = kRows * kRows;                 // one segment increment: S'[0..64][0..64]
constexpr int kStages = 3;                                // Q, K, V tiles in flight

// Shared memory (bytes from a 1024-aligned base):
//   pass: Q 3 x 16 KB | K 3 x 16 KB | V 3 x 16 KB | ones 16 KB | ones(A) 4 KB |
//         S' snapshots 2 x (2 x 10 KB) | y stage 16 KB
//   increments: K 3 x 16 KB | V 3 x 16 KB | ones 16 KB
// "ones": 128 rows of 128 B whose element 0 is 1 (SW128): the second
// 64-element group of the MN-major operands [K | 1]^T (feature 64 = the
// constant) and [V | 1] (column 64 = the count). "ones(A)": 128 rows of 32 B
// (SW32, K-major) whose element 0 is 1: the constant feature of [Q | 1].
template <bool AGG>
struct FoLayout {
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = AGG ? 0 : kStages * 16384;
  static constexpr int kOffV = kOffK + kStages * 16384;
  static constexpr int kOffOnes = kOffV + kStages * 16384;
  static constexpr int kOffOnesA = kOffOnes + 16384;
  static constexpr int kOffSnap = kOffOnesA + (AGG ? 0 : 4096);
  static constexpr int kSnapGroup = kNa * 128;                // 10 KB per 64-column group
  static constexpr int kSnapBytes = 2 * kSnapGroup;            // one snapshot (two groups)
  static constexpr int kOffStage = kOffSnap + (AGG ? 0 : 2 * kSnapBytes);   // two snapshots
  static constexpr int kOffBars = kOffStage + (AGG ? 0 : 16384);
  static constexpr int kSmemBytes = kOffBars + 1024 + 1024;
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffOnes % 1024 == 0 &&
                    kOffOnesA % 1024 == 0 && kOffSnap % 1024 == 0 && kOffStage % 1024 == 0,
                "swizzle atoms need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};
enum {
  kBarQFull = 0, kBarQEmpty = kBarQFull + kStages, kBarKvFull = kBarQEmpty + kStages,
  kBarKvEmpty = kBarKvFull + kStages, kBarSFull = kBarKvEmpty + kStages, kBarPFull = kBarSFull + 2,
  kBarOFull, kBarOFree, kBarSnapFull, kBarSnapFree, kBarStageFull, kBarStageFree, kBarUpdFull, kNumBars
};
constexpr int kBarBytes = 8 * kNumBars;

__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint4 pack8(const uint32_t *a) {
  return make_uint4(pack_bf16x2(__uint_as_float(a[0]), __uint_as_float(a[1])),
                    pack_bf16x2(__uint_as_float(a[2]), __uint_as_float(a[3])),
                    pack_bf16x2(__uint_as_float(a[4]), __uint_as_float(a[5])),
                    pack_bf16x2(__uint_as_float(a[6]), __uint_as_float(a[7])));
}
__device__ __forceinline__ uint4 pack8_scaled(const uint32_t *a, float2 s) {
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 v = __fmul2_rn(make_float2(__uint_as_float(a[2 * j]), __uint_as_float(a[2 * j + 1])), s);
    w[j] = pack_bf16x2(v.x, v.y);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

constexpr uint32_t kSetArrivals = 128;
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

template <bool AGG>
__global__ void __launch_bounds__(kThreads, 1)
fo_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
             const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
             float *__restrict__ agg, const float *__restrict__ S0, const float *__restrict__ z0,
             float *__restrict__ S_out, float *__restrict__ z_out,
             unsigned *__restrict__ status, int T, int G_grid, int G_total, int seg_len) {
  using L = FoLayout<AGG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffBars + kBarBytes);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffBars + kBarBytes + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int g = blockIdx.x % G_grid;
  const int bh = blockIdx.x / G_grid;
  const int t0 = g * seg_len;
  const int t1 = min(T, t0 + seg_len);
  const int ntiles = (t1 - t0 + kTile - 1) / kTile;

  // constant operands (zero elsewhere), then the barriers
  for (int i = threadIdx.x; i < 16384 / 16; i += kThreads) {
    const int row = i >> 3, chunk = i & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (chunk == (row & 7)) v.x = 0x3f80u;               // logical chunk 0 of the row: element 0 = 1
    *reinterpret_cast<uint4 *>(smem + L::kOffOnes + i * 16) = v;
  }
  if (!AGG) {
    for (int i = threadIdx.x; i < 4096 / 16; i += kThreads) {
      const int row = i >> 1, chunk = i & 1;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (chunk == ((row >> 2) & 1)) v.x = 0x3f80u;
      *reinterpret_cast<uint4 *>(smem + L::kOffOnesA + i * 16) = v;
    }
    // snapshot rows 65..79 and the unused chunks of the second group stay zero
    for (int i = threadIdx.x; i < 2 * L::kSnapBytes / 16; i += kThreads)
      *reinterpret_cast<uint4 *>(smem + L::kOffSnap + i * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_async_smem();
  if (threadIdx.x == 0) {
    constexpr uint32_t A = kSetArrivals;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[kBarQFull + s], 1);
      mbar_init(&bars[kBarQEmpty + s], 1);
      mbar_init(&bars[kBarKvFull + s], 1);
      mbar_init(&bars[kBarKvEmpty + s], AGG ? 1 : 2);     // pass: both issuing warps
    }
    for (int s = 0; s < 2; ++s) mbar_init(&bars[kBarSFull + s], 1);
    mbar_init(&bars[kBarPFull], A);
    mbar_init(&bars[kBarOFull], 1);
    mbar_init(&bars[kBarOFree], A);
    mbar_init(&bars[kBarSnapFull], A);
    mbar_init(&bars[kBarSnapFree], 2);              // both issuing warps
    mbar_init(&bars[kBarStageFull], A);
    mbar_init(&bars[kBarStageFree], 1);
    mbar_init(&bars[kBarUpdFull], 1);
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
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % kStages, row = t0 + i * kTile;
        const uint32_t par = ((i / kStages) - 1) & 1;
        if (!AGG) {
          if (i >= kStages && !mbar_wait(&bars[kBarQEmpty + st], par, abort_flag)) break;
          mbar_arrive_expect_tx(&bars[kBarQFull + st], 16384);
          tma_load_3d(smem + L::kOffQ + 16384 * st, &tmq, &bars[kBarQFull + st], 0, row, bh);
        }
        if (i >= kStages && !mbar_wait(&bars[kBarKvEmpty + st], par, abort_flag)) break;
        mbar_arrive_expect_tx(&bars[kBarKvFull + st], 32768);
        tma_load_3d(smem + L::kOffK + 16384 * st, &tmk, &bars[kBarKvFull + st], 0, row, bh);
        tma_load_3d(smem + L::kOffV + 16384 * st, &tmv, &bars[kBarKvFull + st], 0, row, bh);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t id_pv = idesc_bf16(128, kNa, false, true);
      constexpr uint32_t id_ro = idesc_bf16(128, kNa, false, true);
      constexpr uint32_t id_up = idesc_bf16(128, kNa, true, true);
      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
      const uint32_t a_q = smem_u32(smem + L::kOffQ), a_k = smem_u32(smem + L::kOffK);
      const uint32_t a_v = smem_u32(smem + L::kOffV), a_ones = smem_u32(smem + L::kOffOnes);
      // [V | 1] and [K | 1]^T, MN-major: the second 64-element group is the ones tile
      uint64_t d_v1[kStages], d_k1[kStages], d_kk[kStages], d_q[kStages];
      for (int s = 0; s < kStages; ++s) {
        d_v1[s] = smem_desc(a_v + 16384 * s, a_ones - (a_v + 16384 * s), 1024, kSw128);
        d_k1[s] = smem_desc(a_k + 16384 * s, a_ones - (a_k + 16384 * s), 1024, kSw128);
        d_kk[s] = smem_desc(a_k + 16384 * s, 16, 1024, kSw128);     // K, K-major (Q K^T's B)
        d_q[s] = smem_desc(a_q + 16384 * s, 16, 1024, kSw128);      // Q, K-major
      }
      const uint64_t d_q1 = smem_desc(smem_u32(smem + L::kOffOnesA), 16, 256, kSw32);
      const uint64_t d_snap = smem_desc(smem_u32(smem + L::kOffSnap), L::kSnapGroup, 1024, kSw128);
      bool ok = true;
      if (AGG) {
        for (int i = 0; ok && i < ntiles; ++i) {
          const int st = i % kStages;
          if (!(ok = mbar_wait(&bars[kBarKvFull + st], (i / kStages) & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tbase + kColS, adv(d_k1[st], 2048 * kk), adv(d_v1[st], 2048 * kk), id_up,
                   (i > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars[kBarKvEmpty + st]);
        }
        if (ok && ntiles > 0) mma_commit(&bars[kBarUpdFull]);
      } else {
        auto issue_qk = [&](int i) {
          const int st = i % kStages, xb = i & 1;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tbase + kColX + 128 * xb, adv(d_q[st], 32 * kk), adv(d_kk[st], 32 * kk), id_qk, kk);
          mma_commit(&bars[kBarSFull + xb]);
        };
        if (ntiles > 0) {
          ok = mbar_wait(&bars[kBarQFull], 0, abort_flag) && mbar_wait(&bars[kBarKvFull], 0, abort_flag);
          if (ok) {
            tc_fence_after();
            issue_qk(0);
          }
        }
        // PFull(i) also says: the snapshot of S'_i is in place, tile i + 1's
        // Q, K, V are loaded, and O' was read by the previous epilogue.
        for (int i = 0; ok && i < ntiles; ++i) {
          const int st = i % kStages;
          if (!(ok = mbar_wait(&bars[kBarPFull], i & 1, abort_flag))) break;
          tc_fence_after();
          if (i + 1 < ntiles) issue_qk(i + 1);
          // O' = P [V | 1]  (P from tensor memory)
          const uint32_t x = tbase + kColX + 128 * (i & 1);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tbase + kColO, x + 8 * kk, adv(d_v1[st], 2048 * kk), id_pv, kk);
          // tile i - 1's readout (issued before) has read the other snapshot
          // buffer; K_i (Q K^T) and V_i (P V) are read. Warp 10 adds its
          // commits for the update of S'.
          mma_commit(&bars[kBarSnapFree]);
          mma_commit(&bars[kBarKvEmpty + st]);
          // O' += [Q | 1] S'_i
          const uint64_t d_sn = adv(d_snap, (i & 1) * L::kSnapBytes);
#pragma unroll
          for (int kk = 0; kk < 5; ++kk)
            mma_ss(tbase + kColO, kk < 4 ? adv(d_q[st], 32 * kk) : d_q1, adv(d_sn, 2048 * kk), id_ro, 1);
          mma_commit(&bars[kBarOFull]);
          mma_commit(&bars[kBarQEmpty + st]);
        }
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------ MMA issue: the update
    // S' += [K | 1]^T [V | 1], issued beside warp 1's stream (one thread
    // issues an MMA only every ~80 cycles). The readout of tile i reads the
    // snapshot of S'_i in shared memory, so the state side takes the snapshot
    // of S'_i+1 while it runs.
    if (!AGG && lane == 0) {
      constexpr uint32_t id_up = idesc_bf16(128, kNa, true, true);
      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
      const uint32_t a_k = smem_u32(smem + L::kOffK), a_v = smem_u32(smem + L::kOffV);
      const uint32_t a_ones = smem_u32(smem + L::kOffOnes);
      bool ok = true;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i % kStages;
        const uint64_t d_v1 = smem_desc(a_v + 16384 * st, a_ones - (a_v + 16384 * st), 1024, kSw128);
        const uint64_t d_k1 = smem_desc(a_k + 16384 * st, a_ones - (a_k + 16384 * st), 1024, kSw128);
        // PFull(i): the snapshot of S'_i is taken and tile i's K, V are loaded
        if (!(ok = mbar_wait(&bars[kBarPFull], i & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tbase + kColS, adv(d_k1, 2048 * kk), adv(d_v1, 2048 * kk), id_up, 1);
        mma_commit(&bars[kBarSnapFree]);
        mma_commit(&bars[kBarKvEmpty + st]);
      }
      if (ok && ntiles > 0) mma_commit(&bars[kBarUpdFull]);
    }
  } else if (warp < 6) {
    // ------------------------------------------------ query side (warps 2..5)
    if (!AGG) {
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      for (int i = 0; i < ntiles; ++i) {
        const int xb = i & 1, c0 = t0 + i * kTile;
        if (!warp_wait(&bars[kBarSFull + xb], (i >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        // ---- P = (1 + Q K^T) masked to keys s <= min(r, t1 - 1 - c0) ----
        const uint32_t x = tbase + lane_off + kColX + 128 * xb;
        const int lim = min(r, t1 - 1 - c0);
        const int lim_lo = __reduce_min_sync(0xffffffffu, lim);
        const int lim_hi = __reduce_max_sync(0xffffffffu, lim);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t p[16];
          if (32 * c > lim_hi) {
#pragma unroll
            for (int k = 0; k < 16; ++k) p[k] = 0u;
          } else {
            uint32_t xv[32];
            tmem_ld32(x + 32 * c, xv);
            tmem_wait_ld();
            const bool full = 32 * c + 31 <= lim_lo;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int s0 = 32 * c + 2 * k;
              float a = 1.f + __uint_as_float(xv[2 * k]), b = 1.f + __uint_as_float(xv[2 * k + 1]);
              if (!full) {
                a = s0 <= lim ? a : 0.f;
                b = s0 + 1 <= lim ? b : 0.f;
              }
              p[k] = pack_bf16x2(a, b);
            }
          }
          tmem_st16(x + 16 * c, p);
        }
        tmem_wait_st();
        tc_fence_before();
        // fold the MMA warp's other dependencies into PFull: the snapshot of
        // S'_i, O' read by the previous epilogue, tile i + 1's Q, K, V
        bool ok = warp_wait(&bars[kBarSnapFull], i & 1, abort_flag);
        if (ok && i > 0) ok = warp_wait(&bars[kBarOFree], (i - 1) & 1, abort_flag);
        if (ok && i + 1 < ntiles) {
          const int sn = (i + 1) % kStages;
          const uint32_t pn = ((i + 1) / kStages) & 1;
          ok = warp_wait(&bars[kBarQFull + sn], pn, abort_flag) && warp_wait(&bars[kBarKvFull + sn], pn, abort_flag);
        }
        if (!ok) break;
        mbar_arrive(&bars[kBarPFull]);
      }
    }
  } else {
    // -------------------------------------------------- state side (warps 6..9)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                  // TMEM lane = feature row of S'
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t *snap = smem + L::kOffSnap;
    const bool rows = quarter < 3;                      // warps holding rows 0..64 (row 64 in quarter 2)
    bool ok = true;
    // snapshot of S' rows 0..64 (80 columns) as the readout's bf16 B operand
    auto snapshot = [&](int buf) {
      if (!rows) return;
      uint8_t *sn = snap + buf * L::kSnapBytes;
      uint32_t a[32], b[32], c[16];
      tmem_ld32(tbase + lane_off + kColS, a);
      tmem_ld32(tbase + lane_off + kColS + 32, b);
      tmem_ld16(tbase + lane_off + kColS + 64, c);
      tmem_wait_ld();
      if (r < kRows) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          *reinterpret_cast<uint4 *>(sn + sw128(r, q4)) = pack8(a + 8 * q4);
          *reinterpret_cast<uint4 *>(sn + sw128(r, 4 + q4)) = pack8(b + 8 * q4);
        }
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2)
          *reinterpret_cast<uint4 *>(sn + L::kSnapGroup + sw128(r, q2)) = pack8(c + 8 * q2);
      }
    };

    // ---- carry-in: S' = the initial state (library layout, if any) plus the
    //      increments of segments 0 .. g-1 ----
    if (!AGG) {
      const float *seg0 = agg + (size_t)bh * G_total * kAggFloats;
      float acc[kNa];
#pragma unroll
      for (int c = 0; c < kNa; ++c) acc[c] = 0.f;
      if (r < kRows) {
        // library row 0 is the constant feature (internal row 64), row 1 + f is k_f
        const int lr = r == kDh ? 0 : r + 1;
        if (S0) {
          const float *s0 = S0 + ((size_t)bh * kRows + lr) * kDh;
#pragma unroll
          for (int c = 0; c < kDh; ++c) acc[c] = s0[c];
        }
        if (z0) acc[kDh] = z0[(size_t)bh * kRows + lr];
      }
      if (r < kRows)
        for (int gp = 0; gp < g; ++gp) {
          const float *src = seg0 + (size_t)gp * kAggFloats + (size_t)r * kRows;
#pragma unroll
          for (int c = 0; c < kRows; ++c) acc[c] += src[c];
        }
      uint32_t bits[kNa];
#pragma unroll
      for (int c = 0; c < kNa; ++c) bits[c] = __float_as_uint(acc[c]);
      tmem_st32(tbase + lane_off + kColS, *reinterpret_cast<uint32_t(*)[32]>(bits));
      tmem_st32(tbase + lane_off + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(bits + 32));
      tmem_st16(tbase + lane_off + kColS + 64, *reinterpret_cast<uint32_t(*)[16]>(bits + 64));
      tmem_wait_st();
      snapshot(0);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[kBarSnapFull]);
    }

    uint8_t *stage = smem + L::kOffStage;
    for (int i = 0; !AGG && ok && i < ntiles; ++i) {
      const int c0 = t0 + i * kTile;
      // snapshot of S'_i+1 (into buffer (i + 1) & 1) once tile i's update is
      // done, which also means tile i - 1's readout has read that buffer
      if (i + 1 < ntiles) {
        if (!(ok = warp_wait(&bars[kBarSnapFree], i & 1, abort_flag))) break;
        tc_fence_after();
        snapshot((i + 1) & 1);
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[kBarSnapFull]);
      }
      // ---- epilogue: y = O'[:, 0:64] / O'[:, 64] (row r = token r) ----
      if (!(ok = warp_wait(&bars[kBarOFull], i & 1, abort_flag))) break;
      tc_fence_after();
      uint32_t oa[32], ob[32], oc[16];
      tmem_ld32(tbase + lane_off + kColO, oa);
      tmem_ld32(tbase + lane_off + kColO + 32, ob);
      tmem_ld16(tbase + lane_off + kColO + 64, oc);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars[kBarOFree]);                   // O' may be overwritten
      const float den = __uint_as_float(oc[0]);
      if (!(den > 0.f) && c0 + r < t1) flag_status(status, kStatusNonPositiveNormaliser);
      const float inv = 1.f / den;                      // rows past the segment are not stored
      const float2 inv2 = make_float2(inv, inv);
      if (i > 0 && !(ok = warp_wait(&bars[kBarStageFree], (i - 1) & 1, abort_flag))) break;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        *reinterpret_cast<uint4 *>(stage + sw128(r, q4)) = pack8_scaled(oa + 8 * q4, inv2);
        *reinterpret_cast<uint4 *>(stage + sw128(r, 4 + q4)) = pack8_scaled(ob + 8 * q4, inv2);
      }
      fence_async_smem();
      mbar_arrive(&bars[kBarStageFull]);
      // y of tile i leaves by one TMA store (one thread)
      if (r == 0) {
        ok = mbar_wait(&bars[kBarStageFull], i & 1, abort_flag);
        if (ok) {
          tma_store_3d(&tmo, stage, 0, t0 + i * kTile, bh);
          bulk_commit_group();
          bulk_wait_read_all();
          mbar_arrive(&bars[kBarStageFree]);
        }
      }
      ok = __all_sync(0xffffffffu, ok);
    }
    if (!AGG && r == 0) bulk_wait_all();

    // ---- state leaving the kernel ----
    const bool write_out = !AGG && g == G_total - 1 && (S_out || z_out);
    if (ok && ntiles > 0 && (AGG || write_out) && warp_wait(&bars[kBarUpdFull], 0, abort_flag)) {
      tc_fence_after();
      if (rows) {
        uint32_t a[32], b[32], c[16];
        tmem_ld32(tbase + lane_off + kColS, a);
        tmem_ld32(tbase + lane_off + kColS + 32, b);
        tmem_ld16(tbase + lane_off + kColS + 64, c);
        tmem_wait_ld();
        if (r < kRows) {
          if (AGG) {
            float *dst = agg + ((size_t)bh * G_total + g) * kAggFloats + (size_t)r * kRows;
#pragma unroll
            for (int j = 0; j < 32; ++j) dst[j] = __uint_as_float(a[j]);
#pragma unroll
            for (int j = 0; j < 32; ++j) dst[32 + j] = __uint_as_float(b[j]);
            dst[64] = __uint_as_float(c[0]);
          } else {
            // library order: row 0 is the constant feature (internal row 64),
            // row 1 + f is k_f (internal row f)
            const int abi = r == kDh ? 0 : r + 1;
            if (S_out) {
              float *row = S_out + ((size_t)bh * kRows + abi) * kDh;
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                *reinterpret_cast<float4 *>(row + j) =
                    make_float4(__uint_as_float(a[j]), __uint_as_float(a[j + 1]),
                                __uint_as_float(a[j + 2]), __uint_as_float(a[j + 3]));
                *reinterpret_cast<float4 *>(row + 32 + j) =
                    make_float4(__uint_as_float(b[j]), __uint_as_float(b[j + 1]),
                                __uint_as_float(b[j + 2]), __uint_as_float(b[j + 3]));
              }
            }
            if (z_out) {
              // the last tile is padded to 128 rows whose constant feature
              // also counted; remove the padding from the count
              float zc = __uint_as_float(c[0]);
              if (r == kDh) zc -= (float)(ntiles * kTile - (t1 - t0));
              z_out[(size_t)bh * kRows + abi] = zc;
            }
          }
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

bool fo_tc_supported(const ChunkedLaunch &a, int d_k, int d_v, int C, int feature) {
  if (feature != kFirstOrder || d_k != kDh || d_v != kDh || (C != 64 && C != 128) || a.T <= 0)
    return false;
  for (const void *p : {a.q, a.k, a.v, (const void *)a.o})
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return false;
  if (a.S_out && reinterpret_cast<uintptr_t>(a.S_out) % 16 != 0) return false;
  return true;
}

cudaError_t fo_tc(const ChunkedLaunch &a) {
  // segments of whole 128-token tiles, no more of them than the caller sized
  // the workspace for
  int G, seg_len;
  tile_segments(a.T, kTile, a.G, &G, &seg_len);
  // the state-only call reads neither q nor o: their maps are built on k, v
  // and never used by the increment kernel
  CUtensorMap tq, tk, tv, to;
  if (!make_tma_3d_bf16(&tq, a.state_only ? a.k : a.q, kDh, a.T, a.BH, kTile) ||
      !make_tma_3d_bf16(&tk, a.k, kDh, a.T, a.BH, kTile) ||
      !make_tma_3d_bf16(&tv, a.v, kDh, a.T, a.BH, kTile) ||
      !make_tma_3d_bf16(&to, a.state_only ? a.v : a.o, kDh, a.T, a.BH, kTile))
    return cudaErrorInvalidValue;              // accepted shape: a failure, not a fallback
  cudaError_t e;
  // increments of segments 0 .. G-2 (all G for the state-only call)
  const int G_inc = a.state_only ? G : G - 1;
  if (G_inc > 0) {
    auto kagg = fo_tc_kernel<true>;
    e = cudaFuncSetAttribute(kagg, cudaFuncAttributeMaxDynamicSharedMemorySize, FoLayout<true>::kSmemBytes);
    if (e != cudaSuccess) return e;
    ProfileScope prof("tc_fo_increment", a.stream);
    kagg<<<(unsigned)(a.BH * G_inc), kThreads, FoLayout<true>::kSmemBytes, a.stream>>>(
        tq, tk, tv, to, a.agg, nullptr, nullptr, nullptr, nullptr, a.status, a.T, G_inc, G, seg_len);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.state_only) {
    // the constant feature of the last segment's padded rows entered the count
    const int t0_last = (G - 1) * seg_len;
    const int last_tiles = (a.T - t0_last + kTile - 1) / kTile;
    const float pad = (float)(last_tiles * kTile - (a.T - t0_last));
    return state_reduce(kAggFoTc, a.agg, a.BH, G, kRows, kDh, kDh, a.S_out, a.z_out, pad, a.stream);
  }
  auto kpass = fo_tc_kernel<false>;
  e = cudaFuncSetAttribute(kpass, cudaFuncAttributeMaxDynamicSharedMemorySize, FoLayout<false>::kSmemBytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_fo_pass", a.stream);
  kpass<<<(unsigned)(a.BH * G), kThreads, FoLayout<false>::kSmemBytes, a.stream>>>(
      tq, tk, tv, to, a.agg, a.S0, a.z0, a.S_out, a.z_out, a.status, a.T, G, G, seg_len);
  return cudaGetLastError();
}

size_t fo_tc_agg_floats() { return (size_t)kAggFloats; }

}  // namespace kata
