// Tensor-core chunked-state forward for the rank-one PSD feature (bf16
// inputs, fp32 accumulation; d_k = 32, d_v = 64; 128-token chunks) on a
// cluster of two CTAs per (head, segment).
//
// The exact O(T) chunked form (KATA explainer section 2.3; arXiv abstract):
// for chunk c with state (S_c, Z_c) carried in from the earlier chunks
//   A     = (Q_c K_c^T)^2 masked to s <= t              intra-chunk block
//   num   = A V_c + phi_q(Q_c) S_c                      tcgen05.mma
//   den   = A 1   + q_t^T Z_c q_t                       (Z = sum k k^T, so
//                                                        q^T Z q = phi_q(q) . z)
//   y     = num / den                                   convex output gate
//   S_c+1 = S_c + phi(K_c)^T V_c,  Z_c+1 = Z_c + K_c^T K_c
// with phi(k) the 528 distinct products k_i k_j (i <= j) and phi_q(q) the
// same products of q with the off-diagonal multiplicity 2.
//
// The two CTAs split the 528 features (order and tiles as in
// psd_tc_common.cuh), so each holds half of the state and the whole chunk's
// query features for its half in tensor memory:
//   rank 0: state tiles 0, 1 (features 0..255), readout slots 0..3, the
//           intra-chunk block (Q K^T, P = (Q K^T)^2 masked, P V) and the
//           output y = (O_0 + O_1) / (l_intra + q^T Z_c q);
//   rank 1: state tiles 2, 3, 4 (features 256..527), readout slots 4..8,
//           Z and U = Q Z_c. Its partial numerator O_1 and q^T Z_c q go to
//           rank 0 through distributed shared memory (st.shared::cluster,
//           one remote mbarrier arrival per thread), and rank 0 frees the
//           buffer the same way.
// Both CTAs load Q, K, V themselves (the second load of a tile is an L2
// hit); no load is multicast.
//
// The state update is a TS MMA: the key features are built in tensor memory
// (lane = feature, columns = tokens) from a transposed copy of the K tile
// in shared memory (thread l of a key-side warp reads dimension rows l and
// its partner's); the
// readout is a TS MMA with the query features in tensor memory and a bf16
// snapshot of the state (double-buffered) as the shared-memory operand.
// The state in tensor memory is the raw sum S_f = sum k_i k_j v; the
// snapshot holds m_f S_f (m_f = 2 off the diagonal), so that plain query
// products give phi_q(q) . S.
//
// Warps (384 threads): 0 TMA producer; 1 TMEM allocation and the readout
// side's MMAs (rank 0: Q K^T, P V, readout; rank 1: U, readout); 2 and 3
// the update MMAs (each its own tiles; rank 1's warp 2 also Z); 4-7 query
// side (thread = token of the chunk); 8-11 key side (thread = key
// dimension / state row).
//
// Tensor memory (512 columns of each CTA):
//   rank 0: [0,128) S tiles 0,1 | [128,256) query features, slots 0..3 |
//           [256,320) key features (two 32-column half-tile buffers) |
//           [320,448) Q K^T, then P (bf16) in
//           [320,384) | [448,512) O_0
//   rank 1: [0,192) S tiles 2,3,4 | [192,320) query features, slots 4..7 |
//           [320,384) key features (two half-tile buffers) |
//           [384,416) Z (lanes 0..31) |
//           [416,448) U | [448,512) O_1
// Slot 8 (16 features) of rank 1 is a 4 KB shared-memory A operand.
//
// Every wait is bounded (2 s): on expiry the CTA raises its abort flag,
// later waits return at once, the peer's waits run out in turn, and both
// CTAs free their tensor memory and report KATA_ERR_DEVICE_TIMEOUT.
#include "common.cuh"
#include "launch.h"
#include "profile.h"
#include "psd_tc_common.cuh"
#include "tma_host.h"

namespace kata {
namespace {

using namespace tc;
using namespace psd;

constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
// tensor memory
constexpr uint32_t k0S = 0, k0QF = 128, k0Key = 256, k0X = 320, k0O = 448;
constexpr uint32_t k1S = 0, k1QF = 192, k1Key = 320, k1Z = 384, k1U = 416, k1O = 448;

// Shared memory (bytes from a 1024-aligned base):
//   Q 2 x 8 KB | K 2 x 8 KB | V 2 x 16 KB | snapshots 2 x 35 KB (up to 272
//   rows of 128 B) | rank 0: the exchange buffer (rank 1's partial O,
//   [128][64] fp32 in 256-byte rows with 16-byte chunks rotated by the row,
//   then q^T Z q [128]) | rank 1: Z snapshot 2 KB, slot 8 (4 KB) |
//   barriers.
// The Z MMA (rank 1) reads its A operand (K^T, M = 128 of which 32 rows
// carry K's dimensions) through 8 KB-strided atoms that run into the V
// buffers; those rows feed only accumulator lanes 32..127, never read.
constexpr int kOffQ = 0, kOffK = 16384, kOffV = 32768, kOffSnap = 65536;
constexpr int kSnapBytes = 35 * 1024;
constexpr int kOffX = kOffSnap + 2 * kSnapBytes;
constexpr int kXDen = 128 * 256;
constexpr int kXBytes = kXDen + 512;
constexpr int kOffZSnap = kOffX;
constexpr int kOffSlot8 = kOffZSnap + 2048;
constexpr int kOffKt = (kOffX + kXBytes + 1023) / 1024 * 1024;     // K^T, 2 buffers
constexpr int kOffBars = (kOffKt + 2 * kKtBytes + 1023) / 1024 * 1024;
constexpr int kSmemBytes = kOffBars + 1024 + 1024;
static_assert(kOffSlot8 + 4096 <= kOffKt, "rank 1 layout");
static_assert(kOffSnap % 1024 == 0 && kSnapBytes % 1024 == 0 && kOffX % 1024 == 0,
              "swizzle atoms need 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");

enum {
  bQKvFull = 0,
  bQKvEmpty = bQKvFull + 2,
  bSFull = bQKvEmpty + 2,
  bPFull,
  bQFFull,
  bRoDone,
  bSnapFull,
  bSnapFree = bSnapFull + 2,
  bTileDone = bSnapFree + 2,
  bKeyFull = bTileDone + 3,
  bKeyFree = bKeyFull + 2,
  bUpdDone = bKeyFree + 2,
  bUReady,
  bUFull,
  bZDone,
  bXFull,
  bXEmpty,
  bKtFull,
  kNumBars = bKtFull + 2
};
constexpr int kBarBytes = 8 * kNumBars;
static_assert(kBarBytes + 8 <= 1024, "barrier area");

// 16-byte chunk c of exchange row r (chunks rotated so that 32 threads
// writing or reading chunk c of 32 rows spread over the banks).
__device__ __forceinline__ uint32_t xchunk(int r, int c) {
  return (uint32_t)(r * 256 + ((c ^ (r & 15)) << 4));
}

__device__ __forceinline__ void warp_arrive1(uint64_t *bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
psd_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, __nv_bfloat16 *__restrict__ out,
                const float *__restrict__ agg, const float *__restrict__ S0,
                const float *__restrict__ z0, float *__restrict__ S_out, float *__restrict__ z_out,
                unsigned *__restrict__ status, int T, int G, int seg_len, int P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBars + kBarBytes);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBars + kBarBytes + 4);

  const int rank = (int)cluster_ctarank();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int pair = blockIdx.x >> 1;
  const int g = pair % G;
  const int bh = pair / G;
  const int t0 = g * seg_len;
  const int t1 = min(T, t0 + seg_len);
  const int nchunks = (t1 - t0 + kC - 1) / kC;
  const int nt = rank == 0 ? 2 : 3;           // state tiles of this CTA
  const int m0 = rank == 0 ? 0 : 2;           // its first tile

  if (threadIdx.x == 0) {
    for (int st = 0; st < 2; ++st) {
      mbar_init(&bars[bQKvFull + st], 1);
      mbar_init(&bars[bQKvEmpty + st], 1 + 2 + 4 + 4);   // three issuers + query and key warps
      mbar_init(&bars[bKeyFull + st], 4);
      mbar_init(&bars[bKeyFree + st], 1);
      mbar_init(&bars[bSnapFull + st], 4);
      mbar_init(&bars[bSnapFree + st], 1);
    }
    mbar_init(&bars[bSFull], 1);
    mbar_init(&bars[bPFull], 4);
    mbar_init(&bars[bQFFull], 4);
    mbar_init(&bars[bRoDone], 1);
    for (int m = 0; m < 3; ++m) mbar_init(&bars[bTileDone + m], 1);
    mbar_init(&bars[bUpdDone], 2);
    mbar_init(&bars[bUReady], 4);
    mbar_init(&bars[bUFull], 1);
    mbar_init(&bars[bZDone], 1);
    mbar_init(&bars[bXFull], 128);
    mbar_init(&bars[bXEmpty], 128);
    for (int b = 0; b < 2; ++b) mbar_init(&bars[bKtFull + b], 4);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();                 // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      for (int i = 0; i < nchunks; ++i) {
        const int st = i & 1;
        const int row = t0 + i * kC;
        if (i >= 2 && !mbar_wait(&bars[bQKvEmpty + st], ((i >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&bars[bQKvFull + st], 8192 + 8192 + 16384);
        tma_load_3d(smem + kOffQ + 8192 * st, &tmq, &bars[bQKvFull + st], 0, row, bh);
        tma_load_3d(smem + kOffK + 8192 * st, &tmk, &bars[bQKvFull + st], 0, row, bh);
        tma_load_3d(smem + kOffV + 16384 * st, &tmv, &bars[bQKvFull + st], 0, row, bh);
      }
    }
  } else if (warp >= 1 && warp <= 3) {
    if (lane == 0) {
      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
      const uint64_t d_q = smem_desc(smem_u32(smem + kOffQ), 16, 512, kSw64);       // K-major
      const uint64_t d_k = smem_desc(smem_u32(smem + kOffK), 16, 512, kSw64);       // K-major
      const uint64_t d_k_mn = smem_desc(smem_u32(smem + kOffK), 8192, 512, kSw64);  // MN-major
      const uint64_t d_v = smem_desc(smem_u32(smem + kOffV), 16384, 1024, kSw128);  // MN-major
      const uint64_t d_snap = smem_desc(smem_u32(smem + kOffSnap), 16384, 1024, kSw128);
      const uint64_t d_z = smem_desc(smem_u32(smem + kOffZSnap), 16, 512, kSw64);
      const uint64_t d_slot8 = smem_desc(smem_u32(smem + kOffSlot8), 16, 256, kSw32);
      constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t id_n64 = idesc_bf16(128, kDV, false, true);   // P V, readout, update
      constexpr uint32_t id_u = idesc_bf16(128, 32, false, false);
      constexpr uint32_t id_z = idesc_bf16(128, 32, true, true);
      bool ok = true;
      if (warp == 1 && rank == 0) {
        // ---------------- rank 0: Q K^T, P V, readout of slots 0..3 ----------------
        auto issue_qk = [&](int i) -> bool {
          const int st = i & 1;
          if (!mbar_wait(&bars[bQKvFull + st], (i >> 1) & 1, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(tbase + k0X, adv(d_q, 8192 * st + 32 * kk), adv(d_k, 8192 * st + 32 * kk), id_qk, kk);
          mma_commit(&bars[bSFull]);
          return true;
        };
        if (nchunks > 0) ok = issue_qk(0);
        for (int i = 0; ok && i < nchunks; ++i) {
          const int st = i & 1, b = i & 1;
          // P_i written, O free (the previous chunk's output has been read)
          if (!(ok = mbar_wait(&bars[bPFull], i & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tbase + k0O, tbase + k0X + 8 * kk, adv(d_v, 16384 * st + 2048 * kk), id_n64, kk);
          mma_commit(&bars[bQKvEmpty + st]);            // Q_i, K_i (Q K^T) and V_i (P V) read
          // the pipe runs this thread's MMAs in order: P V has read P before
          // the next Q K^T overwrites its columns
          if (i + 1 < nchunks && !(ok = issue_qk(i + 1))) break;
          if (!(ok = mbar_wait(&bars[bQFFull], i & 1, abort_flag))) break;
          tc_fence_after();
          for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tbase + k0O, tbase + k0QF + 32 * s + 8 * kk,
                     adv(d_snap, kSnapBytes * b + (64 * s + 16 * kk) * 128), id_n64, 1);
          mma_commit(&bars[bRoDone]);
          mma_commit(&bars[bSnapFree + b]);
        }
      } else if (warp == 1) {
        // ---------------- rank 1: U = Q Z_c, readout of slots 4..8 ----------------
        for (int i = 0; ok && i < nchunks; ++i) {
          const int st = i & 1, b = i & 1;
          // Q_i landed and the Z_i snapshot written
          if (!(ok = mbar_wait(&bars[bUReady], i & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(tbase + k1U, adv(d_q, 8192 * st + 32 * kk), adv(d_z, 32 * kk), id_u, kk);
          mma_commit(&bars[bUFull]);                    // U_i ready, Z snapshot read
          mma_commit(&bars[bQKvEmpty + st]);            // this thread's reads of Q_i done
          // query features written, U read, O free, snapshot i ready
          if (!(ok = mbar_wait(&bars[bQFFull], i & 1, abort_flag))) break;
          tc_fence_after();
          for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tbase + k1O, tbase + k1QF + 32 * s + 8 * kk,
                     adv(d_snap, kSnapBytes * b + (64 * s + 16 * kk) * 128), id_n64, (s | kk) != 0);
          mma_ss(tbase + k1O, d_slot8, adv(d_snap, kSnapBytes * b + 256 * 128), id_n64, 1);
          mma_commit(&bars[bRoDone]);
          mma_commit(&bars[bSnapFree + b]);
        }
      } else {
        // ---------------- update: S tile += phi(K)^T V (rank 1 also Z) ----------------
        // Two issuing threads with their own tiles (warp 2: local tiles 0
        // and 2, and Z; warp 3: local tile 1), so that each tile accumulates
        // in a fixed order and one thread's waits are covered by the
        // other's MMAs. A tile arrives in two halves of 64 tokens.
        const uint32_t sbase = rank == 0 ? k0S : k1S;
        const uint32_t kbuf = rank == 0 ? k0Key : k1Key;
        const int mine = warp == 2 ? 0 : 1;
        for (int i = 0; ok && i < nchunks; ++i) {
          const int st = i & 1;
          for (int mt = mine; mt < nt && ok; mt += 2) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int u = 2 * (nt * i + mt) + h, b = u & 1;
              // the key warps publish a tile after K_i, V_i landed and after
              // the state it updates has been read into the snapshot
              if (!(ok = mbar_wait(&bars[bKeyFull + b], (u >> 1) & 1, abort_flag))) break;
              tc_fence_after();
              if (rank == 1 && mt == 0 && h == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  mma_ss(tbase + k1Z, adv(d_k_mn, 8192 * st + 1024 * kk),
                         adv(d_k_mn, 8192 * st + 1024 * kk), id_z, 1);
                mma_commit(&bars[bZDone]);
              }
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ts(tbase + sbase + 64 * mt, tbase + kbuf + 32 * b + 8 * kk,
                       adv(d_v, 16384 * st + 2048 * (4 * h + kk)), id_n64, 1);
              mma_commit(&bars[bKeyFree + b]);
            }
            if (ok) mma_commit(&bars[bTileDone + mt]);
          }
          if (!ok) break;
          mma_commit(&bars[bQKvEmpty + st]);
        }
        mma_commit(&bars[bUpdDone]);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------ query side (warps 4..7)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                   // token of the chunk = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    if (rank == 0) {
      // y of chunk i: rank 0's O plus rank 1's partial, over the normaliser
      auto epilogue = [&](int i, float l_intra) -> bool {
        if (!warp_wait(&bars[bRoDone], i & 1, abort_flag)) return false;
        tc_fence_after();
        uint32_t o0[32], o1[32];
        tmem_ld32(tbase + lane_off + k0O, o0);
        tmem_ld32(tbase + lane_off + k0O + 32, o1);
        tmem_wait_ld();
        tc_fence_before();
        if (!__all_sync(0xffffffffu, mbar_wait_cluster(&bars[bXFull], i & 1, abort_flag)))
          return false;
        const uint8_t *xb = smem + kOffX;
        float y[64];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float4 p = *reinterpret_cast<const float4 *>(xb + xchunk(r, c));
          const uint32_t *src = c < 8 ? o0 + 4 * c : o1 + 4 * (c - 8);
          y[4 * c + 0] = __uint_as_float(src[0]) + p.x;
          y[4 * c + 1] = __uint_as_float(src[1]) + p.y;
          y[4 * c + 2] = __uint_as_float(src[2]) + p.z;
          y[4 * c + 3] = __uint_as_float(src[3]) + p.w;
        }
        const float den = l_intra + *reinterpret_cast<const float *>(xb + kXDen + 4 * r);
        // the exchange buffer may take the next chunk
        mbar_arrive_cluster(mapa_shared(smem_u32(&bars[bXEmpty]), 1));
        const int t = t0 + i * kC + r;
        if (t < T) {
          if (!(den > 0.f)) flag_status(status, kStatusNonPositiveNormaliser);
          const float inv = 1.f / den;
          uint4 *dst = reinterpret_cast<uint4 *>(out + ((size_t)bh * T + t) * kDV);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_uint4(pack_bf16x2(y[8 * c] * inv, y[8 * c + 1] * inv),
                                pack_bf16x2(y[8 * c + 2] * inv, y[8 * c + 3] * inv),
                                pack_bf16x2(y[8 * c + 4] * inv, y[8 * c + 5] * inv),
                                pack_bf16x2(y[8 * c + 6] * inv, y[8 * c + 7] * inv));
        }
        return true;
      };
      float l_prev = 0.f;
      for (int i = 0; i < nchunks; ++i) {
        const int st = i & 1;
        const int c0 = t0 + i * kC;
        if (!(ok = warp_wait(&bars[bSFull], i & 1, abort_flag))) break;
        tc_fence_after();
        // ---- P = (Q K^T)^2 masked to keys s <= min(r, T-1-c0), in place as bf16 ----
        const int lim = min(r, T - 1 - c0);
        const int lim_lo = __reduce_min_sync(0xffffffffu, lim);
        const int lim_hi = __reduce_max_sync(0xffffffffu, lim);
        float2 lsum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t p[16];
          if (32 * c > lim_hi) {
#pragma unroll
            for (int k = 0; k < 16; ++k) p[k] = 0u;
          } else {
            uint32_t x[32];
            tmem_ld32(tbase + lane_off + k0X + 32 * c, x);
            tmem_wait_ld();
            if (32 * c + 31 <= lim_lo) {
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                const float2 a = make_float2(__uint_as_float(x[2 * k]), __uint_as_float(x[2 * k + 1]));
                const float2 w = __fmul2_rn(a, a);
                lsum[k & 3] = __fadd2_rn(lsum[k & 3], w);
                p[k] = pack_bf16x2(w.x, w.y);
              }
            } else {
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                const int s0 = 32 * c + 2 * k;
                const float2 a = make_float2(__uint_as_float(x[2 * k]), __uint_as_float(x[2 * k + 1]));
                float2 w = __fmul2_rn(a, a);
                w.x = s0 <= lim ? w.x : 0.f;
                w.y = s0 + 1 <= lim ? w.y : 0.f;
                lsum[k & 3] = __fadd2_rn(lsum[k & 3], w);
                p[k] = pack_bf16x2(w.x, w.y);
              }
            }
          }
          tmem_st16(tbase + lane_off + k0X + 16 * c, p);
        }
        const float2 l01 = __fadd2_rn(lsum[0], lsum[1]), l23 = __fadd2_rn(lsum[2], lsum[3]);
        const float2 lt = __fadd2_rn(l01, l23);
        const float l_intra = lt.x + lt.y;
        tmem_wait_st();
        tc_fence_before();
        // ---- y of the previous chunk, which frees O for this chunk's P V ----
        if (i > 0 && !(ok = epilogue(i - 1, l_prev))) break;
        warp_arrive1(&bars[bPFull]);
        l_prev = l_intra;
        // ---- query features of slots 0..3 into tensor memory ----
        if (!(ok = warp_wait(&bars[bQKvFull + st], (i >> 1) & 1, abort_flag))) break;
        uint32_t XQ[16], P[32], R[32];
        load_pairs(smem + kOffQ + 8192 * st, r, XQ, P);
        warp_arrive1(&bars[bQKvEmpty + st]);
#pragma unroll
        for (int l = 0; l < 32; ++l) R[l] = P[l];
        // the previous readout has read the query features (waited for in
        // its epilogue above; chunk 0 has no predecessor)
#pragma unroll 1
        for (int s = 0; s < 4; ++s) {
          uint32_t w[32];
          q_slot_words(P, R, false, w);
          tmem_st32(tbase + lane_off + k0QF + 32 * s, w);
          rotate_left(R, 2);
        }
        tmem_wait_st();
        tc_fence_before();
        if (!(ok = warp_wait(&bars[bSnapFull + (i & 1)], (i >> 1) & 1, abort_flag))) break;
        warp_arrive1(&bars[bQFFull]);
      }
      if (ok && nchunks > 0) ok = epilogue(nchunks - 1, l_prev);
    } else {
      // rank 1's partial numerator and q^T Z_c q of chunk i into rank 0's buffer
      const uint32_t xremote = mapa_shared(smem_u32(smem + kOffX), 0);
      const uint32_t xfull_remote = mapa_shared(smem_u32(&bars[bXFull]), 0);
      auto exchange = [&](int i, float den) -> bool {
        if (!warp_wait(&bars[bRoDone], i & 1, abort_flag)) return false;
        tc_fence_after();
        uint32_t o0[32], o1[32];
        tmem_ld32(tbase + lane_off + k1O, o0);
        tmem_ld32(tbase + lane_off + k1O + 32, o1);
        tmem_wait_ld();
        tc_fence_before();
        if (i >= 1 &&
            !__all_sync(0xffffffffu, mbar_wait_cluster(&bars[bXEmpty], (i - 1) & 1, abort_flag)))
          return false;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t *src = c < 8 ? o0 + 4 * c : o1 + 4 * (c - 8);
          st_cluster_v4(xremote + xchunk(r, c), make_uint4(src[0], src[1], src[2], src[3]));
        }
        st_cluster_u32(xremote + kXDen + 4 * r, __float_as_uint(den));
        mbar_arrive_cluster(xfull_remote);
        return true;
      };
      uint8_t *slot8 = smem + kOffSlot8;
      float den_prev = 0.f;
      for (int i = 0; i < nchunks; ++i) {
        const int st = i & 1;
        // ---- q^T Z_i q = q . u ----
        if (!(ok = warp_wait(&bars[bUFull], i & 1, abort_flag))) break;
        tc_fence_after();
        uint32_t uu[32];
        tmem_ld32(tbase + lane_off + k1U, uu);
        tmem_wait_ld();
        tc_fence_before();
        if (!(ok = warp_wait(&bars[bQKvFull + st], (i >> 1) & 1, abort_flag))) break;
        uint32_t XQ[16], P[32], R[32];
        load_pairs(smem + kOffQ + 8192 * st, r, XQ, P);
        warp_arrive1(&bars[bQKvEmpty + st]);
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < 16; ++w) {
          const __nv_bfloat162 qq = *reinterpret_cast<const __nv_bfloat162 *>(&XQ[w]);
          den = fmaf(__low2float(qq), __uint_as_float(uu[2 * w]), den);
          den = fmaf(__high2float(qq), __uint_as_float(uu[2 * w + 1]), den);
        }
        // ---- the previous chunk's partial leaves; O and the slots are free ----
        if (i > 0 && !(ok = exchange(i - 1, den_prev))) break;
        den_prev = den;
        // ---- query features of slots 4..8 (slot 8 in shared memory) ----
#pragma unroll
        for (int l = 0; l < 32; ++l) R[l] = P[l];
        rotate_left(R, 8);
#pragma unroll 1
        for (int s = 4; s < 8; ++s) {
          uint32_t w[32];
          q_slot_words(P, R, false, w);
          tmem_st32(tbase + lane_off + k1QF + 32 * (s - 4), w);
          rotate_left(R, 2);
        }
        {
          uint32_t w[32];
          q_slot_words(P, R, true, w);          // features (l, l + 16), l < 16: words 0..7
#pragma unroll
          for (int c = 0; c < 2; ++c)
            *reinterpret_cast<uint4 *>(slot8 + r * 32 + ((c ^ ((r >> 2) & 1)) << 4)) =
                make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
        fence_async_smem();
        tmem_wait_st();
        tc_fence_before();
        if (!(ok = warp_wait(&bars[bSnapFull + (i & 1)], (i >> 1) & 1, abort_flag))) break;
        warp_arrive1(&bars[bQFFull]);
      }
      if (ok && nchunks > 0) ok = exchange(nchunks - 1, den_prev);
    }
  } else if (warp >= 8) {
    // -------------------------------------------------- key side (warps 8..11)
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t sbase = rank == 0 ? k0S : k1S;
    const uint32_t kbuf = rank == 0 ? k0Key : k1Key;
    uint8_t *snap = smem + kOffSnap;
    uint8_t *zsnap = smem + kOffZSnap;
    bool ok = true;
    // row of local tile mt this thread owns: global feature f, valid if f < 528
    auto feature_of = [&](int mt) { return 128 * (m0 + mt) + 32 * quarter + lane; };

    // ---- carry-in: the initial state (library layout) plus the increments
    //      of the segments before this one (P pieces each), into tensor
    //      memory (raw) and snapshot 0 (m_f S_f) ----
    {
      const float *inc0 = agg + (size_t)bh * G * P * kAggFloats;
      const int ninc = g * P;
      for (int mt = 0; mt < nt; ++mt) {
        const int f = feature_of(mt);
        const bool valid = f < kD;
        const float mf = f < kDK ? 1.f : 2.f;
        const float inv_mf = f < kDK ? 1.f : 0.5f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float acc[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[c] = 0.f;
          if (valid) {
            if (S0) {
              const float *s0 = S0 + ((size_t)bh * kD + abi_row(f)) * kDV + 16 * q4;
#pragma unroll
              for (int c = 0; c < 16; ++c) acc[c] = s0[c];
            }
            for (int gp = 0; gp < ninc; ++gp) {
              const float4 *src =
                  reinterpret_cast<const float4 *>(inc0 + (size_t)gp * kAggFloats + f * kDV + 16 * q4);
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const float4 x = src[c4];
                acc[4 * c4 + 0] = fmaf(x.x, inv_mf, acc[4 * c4 + 0]);
                acc[4 * c4 + 1] = fmaf(x.y, inv_mf, acc[4 * c4 + 1]);
                acc[4 * c4 + 2] = fmaf(x.z, inv_mf, acc[4 * c4 + 2]);
                acc[4 * c4 + 3] = fmaf(x.w, inv_mf, acc[4 * c4 + 3]);
              }
            }
          }
          uint32_t bits[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) bits[c] = __float_as_uint(acc[c]);
          tmem_st16(tbase + lane_off + sbase + 64 * mt + 16 * q4, bits);
          if (valid) {
            const int fl = f - 128 * m0;
            const float2 m2 = make_float2(mf, mf);
            *reinterpret_cast<uint4 *>(snap + sw128(fl, 2 * q4)) = pack8_scaled(bits, m2);
            *reinterpret_cast<uint4 *>(snap + sw128(fl, 2 * q4 + 1)) = pack8_scaled(bits + 8, m2);
          }
        }
      }
      if (rank == 1) {
        // Z rows live in lanes 0..31 (quarter 0)
        float acc[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) acc[c] = 0.f;
        if (quarter == 0) {
          const int rr = lane;
          if (z0) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int i = rr < c ? rr : c, j = rr < c ? c : rr;
              acc[c] = z0[(size_t)bh * kD + i * kDK - i * (i - 1) / 2 + (j - i)];
            }
          }
          for (int gp = 0; gp < ninc; ++gp) {
            const float4 *src =
                reinterpret_cast<const float4 *>(inc0 + (size_t)gp * kAggFloats + kD * kDV + rr * kDK);
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
              const float4 x = src[c4];
              acc[4 * c4 + 0] += x.x;
              acc[4 * c4 + 1] += x.y;
              acc[4 * c4 + 2] += x.z;
              acc[4 * c4 + 3] += x.w;
            }
          }
        }
        uint32_t bits[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) bits[c] = __float_as_uint(acc[c]);
        tmem_st32(tbase + lane_off + k1Z, bits);
        if (quarter == 0) {
#pragma unroll
          for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(zsnap + sw64(lane, c)) = pack8(bits + 8 * c);
        }
      }
      fence_async_smem();
      tmem_wait_st();
      tc_fence_before();
      warp_arrive1(&bars[bSnapFull + 0]);       // snapshot of chunk 0
    }

    for (int i = 0; ok && i < nchunks; ++i) {
      const int st = i & 1, b = i & 1;
      if (!(ok = warp_wait(&bars[bQKvFull + st], (i >> 1) & 1, abort_flag))) break;
      // K^T of chunk i (buffer i & 1; the key warps' previous use of it,
      // chunk i - 2, ended before the barrier of chunk i - 1)
      uint8_t *kt = smem + kOffKt + kKtBytes * (i & 1);
      transpose_k(smem + kOffK + 8192 * st, kt, 32 * quarter + lane);
      warp_arrive1(&bars[bQKvEmpty + st]);
      // every key warp's part of K^T is written (a bounded wait, like all others)
      warp_arrive1(&bars[bKtFull + (i & 1)]);
      if (!(ok = warp_wait(&bars[bKtFull + (i & 1)], (i >> 1) & 1, abort_flag))) break;
      uint32_t X[64];
      load_kt_row(kt, lane, X);                 // this thread's dimension, all 128 tokens
      if (rank == 1) {
        // ---- snapshot Z_i (after the Z update of chunk i - 1) for U_i ----
        if (i > 0) {
          if (!(ok = warp_wait(&bars[bZDone], (i - 1) & 1, abort_flag))) break;
          // U_(i-1) has read the snapshot; waiting for it also keeps this
          // warp from completing UReady twice before the issuer tests it
          if (!(ok = warp_wait(&bars[bUFull], (i - 1) & 1, abort_flag))) break;
          tc_fence_after();
          if (quarter == 0) {
            uint32_t zr[32];
            tmem_ld32(tbase + lane_off + k1Z, zr);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4 *>(zsnap + sw64(lane, c)) = pack8(zr + 8 * c);
          }
          fence_async_smem();
          tc_fence_before();
        }
        warp_arrive1(&bars[bUReady]);           // Q_i has landed (waited above), Z_i in zsnap
      }
      for (int mt = 0; mt < nt; ++mt) {
        const int u = nt * i + mt;
        const int f = feature_of(mt);
        const int m = m0 + mt;
        // ---- snapshot of S_i tile mt (after the update of chunk i - 1) ----
        if (i > 0) {
          if (!(ok = warp_wait(&bars[bTileDone + mt], (i - 1) & 1, abort_flag))) break;
          tc_fence_after();
          if (mt == 0 && i >= 2 &&
              !(ok = warp_wait(&bars[bSnapFree + b], ((i >> 1) - 1) & 1, abort_flag)))
            break;
          if (m < 4 || quarter == 0) {               // tile 4: rows 512..527 in lanes 0..15
            uint32_t a[32], b2[32];
            tmem_ld32(tbase + lane_off + sbase + 64 * mt, a);
            tmem_ld32(tbase + lane_off + sbase + 64 * mt + 32, b2);
            tmem_wait_ld();
            if (f < kD) {
              const int fl = f - 128 * m0;
              const float mf = f < kDK ? 1.f : 2.f;
              const float2 m2 = make_float2(mf, mf);
              uint8_t *sb = snap + kSnapBytes * b;
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                *reinterpret_cast<uint4 *>(sb + sw128(fl, q4)) = pack8_scaled(a + 8 * q4, m2);
                *reinterpret_cast<uint4 *>(sb + sw128(fl, 4 + q4)) = pack8_scaled(b2 + 8 * q4, m2);
              }
            }
          }
          fence_async_smem();
          tc_fence_before();
          if (mt == nt - 1) warp_arrive1(&bars[bSnapFull + b]);
        }
        // ---- key features of tile mt for chunk i, two halves of 64 tokens
        //      through two 32-column buffers ----
        const int src = m < 4 ? (lane + 4 * m + quarter) & 31 : (lane + 16) & 31;
        const bool write = m < 4 || quarter == 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int uh = 2 * u + h, bb = uh & 1;
          if (uh >= 2 && !(ok = warp_wait(&bars[bKeyFree + bb], ((uh >> 1) - 1) & 1, abort_flag)))
            break;
          tc_fence_after();
          const uint32_t taddr = tbase + lane_off + kbuf + 32 * bb;
          if (write) {
            if (h == 0) key_half<0>(taddr, X, src, m == 4 && lane >= 16);
            else key_half<1>(taddr, X, src, m == 4 && lane >= 16);
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive1(&bars[bKeyFull + bb]);
        }
        if (!ok) break;
      }
    }

    // ---- the state after the last segment, in the library layout ----
    if (ok && g == G - 1 && (S_out || z_out) && warp_wait(&bars[bUpdDone], 0, abort_flag)) {
      tc_fence_after();
      for (int mt = 0; mt < nt; ++mt) {
        const int f = feature_of(mt);
        if (m0 + mt == 4 && quarter != 0) continue;
        uint32_t a[32], b2[32];
        tmem_ld32(tbase + lane_off + sbase + 64 * mt, a);
        tmem_ld32(tbase + lane_off + sbase + 64 * mt + 32, b2);
        tmem_wait_ld();
        if (S_out && f < kD) {
          float *row = S_out + ((size_t)bh * kD + abi_row(f)) * kDV;
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
      if (rank == 1 && quarter == 0 && z_out) {
        uint32_t zr[32];
        tmem_ld32(tbase + lane_off + k1Z, zr);
        tmem_wait_ld();
        // z_(i,j) = Z_ij for i <= j; row l of Z gives the pairs (l, j >= l)
#pragma unroll
        for (int j = 0; j < kDK; ++j)
          if (j >= lane)
            z_out[(size_t)bh * kD + lane * kDK - lane * (lane - 1) / 2 + (j - lane)] = __uint_as_float(zr[j]);
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) flag_status(status, kStatusDeviceTimeout);
  tc_fence_before();
  cluster_sync_all();                 // no CTA leaves while its peer may still touch its memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

}  // namespace

// Shapes handled by the tensor-core chunked forward. The chunk size of the
// exact chunked form only schedules the work: C = 64 and C = 128 both run on
// 128-token chunks (the same result up to rounding).
bool tc_chunked_supported(const ChunkedLaunch &a, int d_k, int d_v, int C, int feature) {
  if (feature != kPSD || d_k != kDK || d_v != kDV || (C != 64 && C != kC) || a.T <= 0) return false;
  for (const void *p : {a.q, a.k, a.v, (const void *)a.o})
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return false;
  if ((a.S_out && reinterpret_cast<uintptr_t>(a.S_out) % 16) != 0) return false;
  return true;
}

size_t tc_chunked_agg_floats() { return (size_t)kAggFloats; }

void tc_chunked_layout(long long BH, int T, int sms, bool sequential, int *G, int *seg_len,
                       int *P) {
  // one wave of CTA pairs: G segments of whole 128-token chunks per head
  const long long pairs = sms / 2;
  const int g_req = (sequential || BH >= pairs) ? 1 : (int)(pairs / BH);
  tile_segments(T, kC, g_req, G, seg_len);
  // each segment increment the pass needs (G - 1 of them per head) is cut
  // into P pieces so that the increment launch also fills the SMs
  const int cps = *seg_len / kC;
  const long long units = BH * (long long)(*G > 1 ? *G - 1 : 1);
  int p = units < sms ? (int)(sms / units) : 1;
  *P = p < 1 ? 1 : (p > cps ? cps : p);
}

cudaError_t tc_chunked(const ChunkedLaunch &a) {
  int G, seg_len, P;
  tc_chunked_layout(a.BH, a.T, a.sms, a.sequential, &G, &seg_len, &P);
  // the state-only call reads neither q nor o: its q map is built on k and
  // never used by the increment kernel
  CUtensorMap tq, tk, tv;
  if (!make_tma_3d_bf16(&tq, a.state_only ? a.k : a.q, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tk, a.k, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tv, a.v, kDV, a.T, a.BH, kC))
    return cudaErrorInvalidValue;              // accepted shape: a failure, not a fallback
  // increments of segments 0 .. G-2 (all G for the state-only call), P pieces each
  const int G_inc = a.state_only ? G : G - 1;
  cudaError_t e = psd_tc_increments(tk, tv, a.agg, a.status, a.BH, a.T, G_inc, P, seg_len / kC,
                                    G * P, a.stream);
  if (e != cudaSuccess) return e;
  if (a.state_only)
    return state_reduce(kAggPsdTc, a.agg, a.BH, G * P, kD, kDK, kDV, a.S_out, a.z_out, 0.f,
                        a.stream);
  auto kpass = psd_pair_kernel;
  e = cudaFuncSetAttribute(kpass, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  if (a.BH * G * 2 > 0x7fffffffLL) return cudaErrorInvalidValue;
  ProfileScope prof("tc_segment_pass", a.stream);
  kpass<<<(unsigned)(a.BH * G * 2), kThreads, kSmemBytes, a.stream>>>(
      tq, tk, tv, reinterpret_cast<__nv_bfloat16 *>(a.o), a.agg, a.S0, a.z0, a.S_out, a.z_out,
      a.status, a.T, G, seg_len, P);
  return cudaGetLastError();
}

}  // namespace kata
