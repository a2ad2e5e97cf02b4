// Segment increments of the PSD chunked-state forward on the tensor cores
// (bf16, d_k = 32, d_v = 64): for a run of whole 128-token chunks,
//   dS = sum_t phi(k_t) v_t^T   (528 x 64),   dZ = sum_t k_t k_t^T   (32 x 32),
// the quantity the scan across chunks adds up (KATA explainer section 2.3;
// the state is a sum over tokens, so any split of the tokens into pieces
// can be summed in any order).
//
// The update dS += phi(K_c)^T V_c is an MMA with M = 128 features per state
// tile, N = 64 value columns and K = 128 tokens. Its A operand, the key
// features, is built in tensor memory (a TS MMA): lane f of the tile holds
// feature f, columns hold the chunk's tokens two bf16 per column. The
// shared memory then carries only the TMA tiles of K and V, and the
// tensor core reads only V from it. The key-side warps transpose the K tile
// into K^T (dimension rows, two tokens per word) in shared memory; thread l
// of key-side warp q then forms tile m's feature (l, (l + d) mod 32),
// d = 4 m + q, from rows l and (l + d) mod 32 of K^T: warp q writes exactly
// the tensor-memory lanes 32 q .. 32 q + 31 that it may address.
//
// Warps (224 threads): 0 TMA producer; 1 and 6 the MMAs (warp 1 also TMEM
// allocation, Z by an SS MMA on the K tile and state tiles 0, 2, 4; warp 6
// tiles 1, 3; TS MMAs); 2-5 the key features, four 32-column half-tile
// buffers in tensor memory, and the increment written out (features
// doubled off the diagonal, the layout the pass kernels read).
//
// Tensor memory: [0, 320) dS, five tiles of 64 columns; [320, 352) dZ (lanes
// 0..31); [384, 512) the four half-tile key-feature buffers.
#include "common.cuh"
#include "launch.h"
#include "profile.h"
#include "psd_tc_common.cuh"
#include "tma_host.h"

namespace kata {
namespace {

using namespace tc;
using namespace psd;

constexpr int kIncThreads = 224;
constexpr uint32_t kIncTmemCols = 512;
constexpr uint32_t kColS = 0, kColZ = 320, kColKey = 384;
constexpr int kKeyBufs = 4;          // 32-column half-tile buffers at kColKey

// Shared memory: K 2 x 8 KB | V 2 x 16 KB | K^T 2 x 8.5 KB | barriers. The
// Z MMA reads its A operand (K^T, M = 128 of which 32 rows are K's
// dimensions) through 8 KB-strided atoms that run into the V buffers: those
// rows only feed accumulator lanes 32..127, which are never read.
constexpr int kOffK = 0, kOffV = 16384, kOffKt = 49152;
constexpr int kOffBars = (kOffKt + 2 * kKtBytes + 1023) / 1024 * 1024;
constexpr int kIncSmemBytes = kOffBars + 1024 + 1024;

enum {
  kBarKvFull = 0,
  kBarKvEmpty = 2,
  kBarKeyFull = 4,
  kBarKeyEmpty = kBarKeyFull + kKeyBufs,
  kBarUpdFull = kBarKeyEmpty + kKeyBufs,
  kBarKtFull = kBarUpdFull + 1,
  kNumIncBars = kBarKtFull + 2
};

// Grid: B*H x (segments x pieces). Block (bh, g, j) covers chunks
// [g cps + j ppc, min(g cps + (j + 1) ppc, (g + 1) cps)) of head bh (cps
// chunks per segment, ppc chunks per piece, P pieces per segment) and
// writes increment number g P + j of that head.
__global__ void __launch_bounds__(kIncThreads, 1)
psd_increment_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     float *__restrict__ agg, unsigned *__restrict__ status, int T, int n_pieces,
                     int P, int cps, int ppc, int incs_per_head) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBars + 8 * kNumIncBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBars + 8 * kNumIncBars + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int piece = blockIdx.x % n_pieces;
  const int bh = blockIdx.x / n_pieces;
  const int g = piece / P, j = piece % P;
  const int c_begin = g * cps + j * ppc;
  const int c_end = min(c_begin + ppc, (g + 1) * cps);
  const int nchunks = max(0, min(c_end, (T + kC - 1) / kC) - c_begin);

  if (threadIdx.x == 0) {
    for (int st = 0; st < 2; ++st) {
      mbar_init(&bars[kBarKvFull + st], 1);
      mbar_init(&bars[kBarKvEmpty + st], 4 + 2);     // key warps + both issuers' commits
    }
    for (int b = 0; b < kKeyBufs; ++b) {
      mbar_init(&bars[kBarKeyFull + b], 4);
      mbar_init(&bars[kBarKeyEmpty + b], 1);
    }
    mbar_init(&bars[kBarUpdFull], 2);
    for (int b = 0; b < 2; ++b) mbar_init(&bars[kBarKtFull + b], 4);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kIncTmemCols);
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
      for (int i = 0; i < nchunks; ++i) {
        const int st = i & 1;
        const int row = (c_begin + i) * kC;
        if (i >= 2 && !mbar_wait(&bars[kBarKvEmpty + st], ((i >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&bars[kBarKvFull + st], 8192 + 16384);
        tma_load_3d(smem + kOffK + 8192 * st, &tmk, &bars[kBarKvFull + st], 0, row, bh);
        tma_load_3d(smem + kOffV + 16384 * st, &tmv, &bars[kBarKvFull + st], 0, row, bh);
      }
    }
  } else if (warp == 1 || warp == 6) {
    // ------------------------------------------------------------ MMA issue
    // Two issuing threads, each with its own tiles (warp 1: Z and tiles 0,
    // 2, 4; warp 6: tiles 1, 3), so that each tile accumulates in a fixed
    // order and one thread's barrier waits are covered by the other's MMAs.
    if (lane == 0) {
      const int mine = warp == 1 ? 0 : 1;
      constexpr uint32_t id_up = idesc_bf16(128, kDV, false, true);   // A from TMEM
      constexpr uint32_t id_z = idesc_bf16(128, 32, true, true);
      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
      const uint64_t d_k_mn = smem_desc(smem_u32(smem + kOffK), 8192, 512, kSw64);     // K, MN-major
      const uint64_t d_v = smem_desc(smem_u32(smem + kOffV), 16384, 1024, kSw128);    // V, MN-major
      bool ok = true;
      for (int i = 0; ok && i < nchunks; ++i) {
        const int st = i & 1;
        for (int m = mine; m < kTiles; m += 2) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int u = 2 * (kTiles * i + m) + h, b = u % kKeyBufs;
            // the key warps publish tile 0 after K_i, V_i have landed
            if (!(ok = mbar_wait(&bars[kBarKeyFull + b], (u / kKeyBufs) & 1, abort_flag))) break;
            tc_fence_after();
            if (m == 0 && h == 0) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_ss(tbase + kColZ, adv(d_k_mn, 8192 * st + 1024 * kk),
                       adv(d_k_mn, 8192 * st + 1024 * kk), id_z, 1);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tbase + kColS + 64 * m, tbase + kColKey + 32 * b + 8 * kk,
                     adv(d_v, 16384 * st + 2048 * (4 * h + kk)), id_up, 1);
            mma_commit(&bars[kBarKeyEmpty + b]);
          }
          if (!ok) break;
        }
        if (!ok) break;
        mma_commit(&bars[kBarKvEmpty + st]);
      }
      mma_commit(&bars[kBarUpdFull]);             // every MMA of this thread is done
    }
  } else if (warp >= 2 && warp < 6) {
    // -------------------------------------------- key side (warps 2..5)
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    // the accumulators start at zero
    {
      uint32_t zeros[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) zeros[c] = 0u;
      for (int c0 = 0; c0 < (int)(kColZ + 32); c0 += 32) tmem_st32(tbase + lane_off + c0, zeros);
      tmem_wait_st();
      tc_fence_before();
    }
    for (int i = 0; ok && i < nchunks; ++i) {
      const int st = i & 1;
      if (!(ok = warp_wait(&bars[kBarKvFull + st], (i >> 1) & 1, abort_flag))) break;
      // K^T of chunk i (buffer i & 1; the key warps' previous use of it,
      // chunk i - 2, ended before the barrier of chunk i - 1)
      uint8_t *kt = smem + kOffKt + kKtBytes * (i & 1);
      transpose_k(smem + kOffK + 8192 * st, kt, 32 * quarter + lane);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[kBarKvEmpty + st]);
        mbar_arrive(&bars[kBarKtFull + (i & 1)]);
      }
      // every key warp's part of K^T is written (a bounded wait, like all others)
      if (!(ok = warp_wait(&bars[kBarKtFull + (i & 1)], (i >> 1) & 1, abort_flag))) break;
      uint32_t X[64];
      load_kt_row(kt, lane, X);                 // this thread's dimension, all 128 tokens
      for (int m = 0; m < kTiles && ok; ++m) {
        // tile m: offset d = 4 m + quarter, partner lane l + d; tile 4: the
        // pairs (l, l + 16), l < 16, in lanes 0..15 of the first warp
        const int src = m < 4 ? (lane + 4 * m + quarter) & 31 : (lane + 16) & 31;
        const bool write = m < 4 || quarter == 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int u = 2 * (kTiles * i + m) + h, b = u % kKeyBufs;
          if (u >= kKeyBufs &&
              !(ok = warp_wait(&bars[kBarKeyEmpty + b], ((u / kKeyBufs) - 1) & 1, abort_flag)))
            break;
          tc_fence_after();
          const uint32_t taddr = tbase + lane_off + kColKey + 32 * b;
          if (write) {
            if (h == 0) key_half<0>(taddr, X, src, m == 4 && lane >= 16);
            else key_half<1>(taddr, X, src, m == 4 && lane >= 16);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kBarKeyFull + b]);
        }
      }
    }
    // ---- the increment leaves in the pass kernels' layout ----
    if (ok && warp_wait(&bars[kBarUpdFull], 0, abort_flag)) {
      tc_fence_after();
      float *dst = agg + ((size_t)bh * incs_per_head + piece) * kAggFloats;
#pragma unroll 1
      for (int m = 0; m < kTiles; ++m) {
        if (m == 4 && quarter != 0) continue;
        const int f = 128 * m + 32 * quarter + lane;
        uint32_t a[32], b2[32];
        tmem_ld32(tbase + lane_off + kColS + 64 * m, a);
        tmem_ld32(tbase + lane_off + kColS + 64 * m + 32, b2);
        tmem_wait_ld();
        if (f < kD) {
          const float sc = f < kDK ? 1.f : 2.f;       // off-diagonal features doubled
          float *row = dst + (size_t)f * kDV;
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            *reinterpret_cast<float4 *>(row + c) =
                make_float4(sc * __uint_as_float(a[c]), sc * __uint_as_float(a[c + 1]),
                            sc * __uint_as_float(a[c + 2]), sc * __uint_as_float(a[c + 3]));
            *reinterpret_cast<float4 *>(row + 32 + c) =
                make_float4(sc * __uint_as_float(b2[c]), sc * __uint_as_float(b2[c + 1]),
                            sc * __uint_as_float(b2[c + 2]), sc * __uint_as_float(b2[c + 3]));
          }
        }
      }
      if (quarter == 0) {
        uint32_t zr[32];
        tmem_ld32(tbase + lane_off + kColZ, zr);
        tmem_wait_ld();
        float *row = dst + kD * kDV + lane * kDK;
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          *reinterpret_cast<float4 *>(row + c) =
              make_float4(__uint_as_float(zr[c]), __uint_as_float(zr[c + 1]),
                          __uint_as_float(zr[c + 2]), __uint_as_float(zr[c + 3]));
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) flag_status(status, kStatusDeviceTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kIncTmemCols);
}

}  // namespace

cudaError_t psd_tc_increments(const CUtensorMap &tk, const CUtensorMap &tv, float *agg,
                              unsigned *status, long long BH, int T, int G_inc, int P, int cps,
                              int incs_per_head, cudaStream_t stream) {
  if (G_inc <= 0) return cudaSuccess;
  const int ppc = (cps + P - 1) / P;
  const int n_pieces = G_inc * P;
  auto k = psd_increment_kernel;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kIncSmemBytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_segment_increment", stream);
  k<<<(unsigned)(BH * n_pieces), kIncThreads, kIncSmemBytes, stream>>>(tk, tv, agg, status, T, n_pieces,
                                                                      P, cps, ppc, incs_per_head);
  return cudaGetLastError();
}

}  // namespace kata
