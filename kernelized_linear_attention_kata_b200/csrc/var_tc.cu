// Tensor-core (tcgen05 / TMEM / TMA) chunked forward of the two-factor
// variants KATA-Mg and KATA-Sigma-g (g = 2), bf16 inputs, d_k = 32, d_v = 64,
// fp32 accumulation.
//
// The KATA explainer (section 2.3) names the variants; the library reads the
// two factors of a head vector x as its halves a = x[0:16], b = x[16:32]:
//   Mg2:  phi(x) = [psi(a), psi(b)],  weight (q_a . k_a)^2 + (q_b . k_b)^2,
//         272 state rows (136 packed pairs of each half);
//   Sg2:  Psi(x) = a a^T + b b^T,     weight sum over the four (q_u . k_w)^2,
//         136 state rows.
// The exact chunked form per 128-token chunk with the state (S, Z) carried
// in (Z = sum k k^T, 32 x 32):
//   intra: A_uw = Q_u K_w^T (16-wide blocks; Mg2 u = w, Sg2 all four),
//          P = sum A_uw^2 masked to s <= t, l = P 1, O = P V
//   readout: O += phi_q(Q) S_c (query features through shared memory),
//          den = l + q^T Zd q with Zd the block-diagonal part of Z_c
//          (Mg2: diag(Z_aa, Z_bb); Sg2: (Z_aa + Z_bb) on both blocks)
//   y = O / den;  S += phi(K)^T V, Z += K^T K.
// The segment scan is the PSD kernels': an increment launch (update only)
// gives each segment the sum of the earlier segments' increments.
//
// Internal feature order of a 16-wide half: f = 16 d + l (d = 0..7, l =
// 0..15) is the pair (l, (l + d) mod 16); f = 128 + l (l < 8) is (l, l + 8).
// Mg2 lays out half a's 128 main pairs, half b's, then a's 8 extra pairs and
// b's (272); Sg2 the 128 main pairs then the 8 extra ones (136). As in the
// PSD kernels the state rows are kept doubled off the diagonal (m_f S_f), so
// the readout multiplies plain query products, and the state is converted
// to the library's order (i <= j row-major per half) only where it enters
// or leaves the kernel.
//
// Synchronous structure: 256 threads (two warps per TMEM lane quarter; half
// h = warp / 4 splits the columns of each phase), threads 0 and 32 issue
// each round of MMAs (each accumulator's chain from one of them) and commit
// it to one barrier every thread waits on. Independent MMAs share rounds:
// per chunk
//   A: U = Q Zd and the blocks of keys 0..63
//   B: P V (keys 0..63, P in U's columns), the blocks of keys 64..127,
//      readout groups 0, 1
//   C: P V (keys 64..127), readout groups 2 (, 3), the update of state tiles
//      0, 1 and Z
//   D (Mg2): readout group 4, the update of tile 2
// (four rounds for Mg2, three for Sg2), the operands of the next round
// written by the threads in between.
//
// Tensor memory (512 columns, fp32): S (NT tiles of 64 columns) | Z (32) |
// U = Q Zd, then P of keys 0..63 (32) | O (64) | work (the intra-chunk
// blocks of 64 keys; Mg2 keeps P of keys 64..127 after them).
#include "common.cuh"
#include "launch.h"
#include "profile.h"
#include "tc_common.cuh"
#include "tma_host.h"
#include "psd_tc_common.cuh"

#include <type_traits>

namespace kata {
namespace {

using namespace tc;
using psd::sw128;
using psd::sw64;
using psd::bmul2;
using psd::pack8;

constexpr int kVC = 128, kVDK = 32, kVDV = 64, kVH = 16;
template <int N> using IC = std::integral_constant<int, N>;
constexpr int kVThreads = 256;
constexpr uint32_t kVTmemCols = 512;

template <int V>
struct VarShape {
  static constexpr int D = V == kMg2 ? 272 : 136;     // state rows
  static constexpr int NT = V == kMg2 ? 3 : 2;        // 128-feature state tiles
  static constexpr int NG = V == kMg2 ? 5 : 3;        // 64-feature groups
  static constexpr int NA = V == kMg2 ? 2 : 4;        // intra-chunk 16-wide blocks
  static constexpr uint32_t ColS = 0, ColZ = 64 * NT, ColU = ColZ + 32, ColO = ColU + 32,
                            ColW = ColO + 64;
  static_assert(ColW + 64 * NA <= kVTmemCols, "tensor memory");
};

struct VarSmem {
  static constexpr int Q = 0;                  // [128][32] bf16, 64-byte swizzle
  static constexpr int K = 8192;
  static constexpr int V = 16384;              // [128][64] bf16, 128-byte swizzle
  static constexpr int Snap = 32768;           // S_c bf16 [384][64] (rows past D zero)
  static constexpr int ZSnap = Snap + 384 * 128;   // Zd bf16 [32][32]
  static constexpr int Buf = ZSnap + 2048;     // 2 x 32 KB key-feature tiles (update A operand)
  static constexpr int Slot = Buf + 65536;     // 2 x 16 KB query-feature slots (readout A operand)
  static constexpr int Lx = Slot + 32768;      // [128] fp32: half 1's partial l
  static constexpr int Bars = Lx + 512;
  static constexpr int Bytes = Bars + 64 + 1024;
  static_assert(Snap % 1024 == 0 && ZSnap % 1024 == 0 && Buf % 1024 == 0 && Slot % 1024 == 0,
                "swizzle atoms");
  static_assert(Bytes <= 232448, "shared memory budget");
};
enum { kVBarLoadQ = 0, kVBarLoadKV, kVBarLoadKV1, kVBarMma, kVNumBars };
// The increment kernel double-buffers K, V: its second stage sits in the
// snapshot area (unused there), kKvStage1 bytes above the first.
constexpr int kKvStage1 = VarSmem::Snap - VarSmem::K;
static_assert(VarSmem::K + kKvStage1 + 8192 <= VarSmem::V + kKvStage1 &&
                  VarSmem::V + kKvStage1 + 16384 <= VarSmem::ZSnap && (VarSmem::V + kKvStage1) % 1024 == 0,
              "second K, V stage inside the snapshot area");

// Pairs of one 16-wide half h of a row: P[l] = (x_(16h+l), x_(16h+(l+1) mod 16)),
// from the row's 16 bf16x2 words X.
__device__ __forceinline__ void half_pairs(const uint32_t (&X)[16], int h, uint32_t (&P)[16]) {
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    P[2 * w] = X[8 * h + w];
    P[2 * w + 1] = __byte_perm(X[8 * h + w], X[8 * h + ((w + 1) & 7)], 0x5432);
  }
}

// The row's 16 bf16x2 words from a 64-byte-swizzled tile.
__device__ __forceinline__ void row_words(const uint8_t *tile, int row, uint32_t (&X)[16]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4 *>(tile + sw64(row, c));
    X[4 * c] = v.x;
    X[4 * c + 1] = v.y;
    X[4 * c + 2] = v.z;
    X[4 * c + 3] = v.w;
  }
}

__device__ __forceinline__ float2 bf2f(uint32_t w) {
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&w);
  return make_float2(__low2float(b), __high2float(b));
}

// Two adjacent features (l, l + d) and (l + 1, l + 1 + d) of the pair arrays,
// as one bf16x2 word: Mg2 one half's products; Sg2 the sum over the halves
// (fp32 products of the bf16 inputs, one rounding). KEY doubles the
// off-diagonal features (the state's m_f).
template <int V, bool KEY>
__device__ __forceinline__ uint32_t pair_word(const uint32_t (&Pa)[16], const uint32_t (&Pb)[16],
                                              int half, int l, int d) {
  const bool dbl = KEY && d != 0;
  if constexpr (V == kMg2) {
    const uint32_t w = half ? bmul2(Pb[l], Pb[(l + d) & 15]) : bmul2(Pa[l], Pa[(l + d) & 15]);
    return dbl ? bmul2(w, 0x40004000u) : w;
  } else {
    const float2 a0 = bf2f(Pa[l]), a1 = bf2f(Pa[(l + d) & 15]);
    const float2 b0 = bf2f(Pb[l]), b1 = bf2f(Pb[(l + d) & 15]);
    const float s = dbl ? 2.f : 1.f;
    return pack_bf16x2(s * fmaf(a0.x, a1.x, b0.x * b1.x), s * fmaf(a0.y, a1.y, b0.y * b1.y));
  }
}

// The 32 words (features 2c, 2c + 1) of 64-feature group GR of one row (GR
// a constant, so that every register index is static).
template <int V, bool KEY, int GR>
__device__ __forceinline__ void group_words_c(const uint32_t (&Pa)[16], const uint32_t (&Pb)[16],
                                              uint32_t (&w)[32]) {
  constexpr int NG = VarShape<V>::NG;
  if constexpr (GR < NG - 1) {
    // main pairs: Mg2 groups 0, 1 are half a's offsets 0..3, 4..7, groups
    // 2, 3 half b's; Sg2 groups 0, 1 the summed offsets 0..3, 4..7
    constexpr int half = V == kMg2 ? (GR >> 1) : 0;
    constexpr int d0 = 4 * (GR & 1);
#pragma unroll
    for (int dd = 0; dd < 4; ++dd)
#pragma unroll
      for (int j = 0; j < 8; ++j) w[8 * dd + j] = pair_word<V, KEY>(Pa, Pb, half, 2 * j, d0 + dd);
  } else {
    // the extra pairs (l, l + 8), l < 8: Mg2 half a's then half b's, Sg2 summed
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j] = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = pair_word<V, KEY>(Pa, Pb, 0, 2 * j, 8);
    if constexpr (V == kMg2) {
#pragma unroll
      for (int j = 0; j < 4; ++j) w[4 + j] = pair_word<V, KEY>(Pa, Pb, 1, 2 * j, 8);
    }
  }
}

// One row of group g into a buffer of 128-byte rows (128-byte swizzle).
__device__ __forceinline__ void store_words(uint8_t *buf, int row, const uint32_t (&w)[32]) {
#pragma unroll
  for (int cc = 0; cc < 8; ++cc)
    *reinterpret_cast<uint4 *>(buf + sw128(row, cc)) =
        make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
}

// Library row of internal feature f, and the pair's (i, j) within its half
// (for the multiplicity), for the variant's state order.
__device__ __forceinline__ int psd16_row(int i, int j) {
  const int a = i < j ? i : j, b = i < j ? j : i;
  return a * kVH - a * (a - 1) / 2 + (b - a);
}
template <int V>
__device__ __forceinline__ int var_abi_row(int f, bool &diag) {
  int blk, l, d;
  if (f < (V == kMg2 ? 256 : 128)) {
    blk = V == kMg2 ? f >> 7 : 0;
    d = (f & 127) >> 4;
    l = f & 15;
  } else {
    const int e = f - (V == kMg2 ? 256 : 128);
    blk = V == kMg2 ? e >> 3 : 0;
    l = e & 7;
    d = 8;
  }
  diag = d == 0;
  return blk * 136 + psd16_row(l, (l + d) & 15);
}

template <int V, bool AGG>
__global__ void __launch_bounds__(kVThreads, 1)
var_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv, float *__restrict__ agg,
              __nv_bfloat16 *__restrict__ o, const float *__restrict__ S0,
              const float *__restrict__ z0, float *__restrict__ S_out, float *__restrict__ z_out,
              unsigned *__restrict__ status, int T, int G_grid, int G_total, int seg_len) {
  using L = VarSmem;
  using SH = VarShape<V>;
  constexpr int D = SH::D, NT = SH::NT, NG = SH::NG, NA = SH::NA;
  constexpr size_t kInc = (size_t)D * kVDV + kVDK * kVDK;   // floats of one increment
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::Bars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::Bars + 8 * kVNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::Bars + 8 * kVNumBars + 4);
  float *lx = reinterpret_cast<float *>(smem + L::Lx);
  uint8_t *snap = smem + L::Snap;
  uint8_t *zsnap = smem + L::ZSnap;
  uint8_t *buf = smem + L::Buf;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int quarter = warp & 3, half = warp >> 2;
  const int r = quarter * 32 + lane;
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  const int g = blockIdx.x % G_grid, bh = blockIdx.x / G_grid;
  const int t0 = g * seg_len, t1 = min(T, t0 + seg_len);
  const int nchunks = (t1 - t0 + kVC - 1) / kVC;
  // the pass's last segment updates after its last chunk only to return the state
  const bool state_out = !AGG && g == G_total - 1 && (S_out || z_out);

  if (threadIdx.x == 0) {
    mbar_init(&bars[kVBarLoadQ], 1);
    mbar_init(&bars[kVBarLoadKV], 1);
    mbar_init(&bars[kVBarLoadKV1], 1);
    mbar_init(&bars[kVBarMma], 2);                // one commit per issuing thread
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kVTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  auto load_q = [&](int i) {
    mbar_arrive_expect_tx(&bars[kVBarLoadQ], 8192);
    tma_load_3d(smem + L::Q, &tmq, &bars[kVBarLoadQ], 0, t0 + i * kVC, bh);
  };
  // K and V of chunk i; the increment kernel alternates two stages
  auto load_kv = [&](int i) {
    const int st = AGG ? (i & 1) : 0;
    uint64_t *bar = &bars[kVBarLoadKV + st];
    mbar_arrive_expect_tx(bar, 8192 + 16384);
    tma_load_3d(smem + L::K + kKvStage1 * st, &tmk, bar, 0, t0 + i * kVC, bh);
    tma_load_3d(smem + L::V + kKvStage1 * st, &tmv, bar, 0, t0 + i * kVC, bh);
  };
  if (threadIdx.x == 0 && nchunks > 0) {
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    if (!AGG) {
      tma_prefetch_desc(&tmq);
      load_q(0);
    }
    load_kv(0);
    if (AGG && nchunks > 1) load_kv(1);
  }

  uint32_t mph = 0;
  auto round = [&](auto issue) -> bool {
    tmem_wait_ld();
    tmem_wait_st();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 || threadIdx.x == 32) {    // issue(0), issue(1): one accumulator each
      tc_fence_after();
      issue(threadIdx.x >> 5);
      mma_commit(&bars[kVBarMma]);
    }
    const bool ok = mbar_wait(&bars[kVBarMma], mph, abort_flag);
    mph ^= 1;
    tc_fence_after();
    return __syncthreads_and(ok);
  };
  auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
    return __syncthreads_and(mbar_wait(bar, parity, abort_flag));
  };

  auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
  const uint64_t d_q = smem_desc(smem_u32(smem + L::Q), 16, 512, kSw64);          // K-major
  const uint64_t d_k = smem_desc(smem_u32(smem + L::K), 16, 512, kSw64);          // K-major
  const uint64_t d_k_mn = smem_desc(smem_u32(smem + L::K), 8192, 512, kSw64);     // MN-major
  const uint64_t d_v_mn = smem_desc(smem_u32(smem + L::V), 16384, 1024, kSw128);  // MN-major
  const uint64_t d_snap = smem_desc(smem_u32(snap), 16384, 1024, kSw128);         // MN-major
  const uint64_t d_z = smem_desc(smem_u32(zsnap), 16, 512, kSw64);
  const uint64_t d_slot = smem_desc(smem_u32(smem + L::Slot), 16, 1024, kSw128);   // K-major
  const uint64_t d_tile = smem_desc(smem_u32(buf), 16384, 1024, kSw128);          // MN-major
  constexpr uint32_t id_n64 = idesc_bf16(128, 64, false, false);
  constexpr uint32_t id_n32 = idesc_bf16(128, 32, false, false);
  constexpr uint32_t id_pv = idesc_bf16(128, 64, false, true);
  constexpr uint32_t id_ro = idesc_bf16(128, 64, false, true);
  constexpr uint32_t id_up = idesc_bf16(128, 64, true, true);
  constexpr uint32_t id_z = idesc_bf16(128, 32, true, true);

  // ---- carry-in: S, Z = the initial state (library order, if any) plus the
  //      increments of the earlier segments; the snapshot's rows past D are
  //      zero (the last readout K-step reads 16 rows) ----
  {
    // (the increment kernel has no readout, and holds its second K, V stage
    // in the snapshot area)
    if (!AGG)
      for (int e = threadIdx.x; e < (384 - D) * 8; e += kVThreads)
        *reinterpret_cast<uint4 *>(snap + (size_t)(D + e / 8) * 128 + (e % 8) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    const float *seg0 = agg + (size_t)bh * G_total * kInc;
    for (int mt = half; mt < NT; mt += 2) {
      const int f = 128 * mt + r;
      bool diag = false;
      const int row = f < D ? var_abi_row<V>(f, diag) : 0;
      const float mf = diag ? 1.f : 2.f;
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        float acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = 0.f;
        if (!AGG && f < D) {
          if (S0) {
            const float *s0 = S0 + ((size_t)bh * D + row) * kVDV + 16 * q4;
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[c] = mf * s0[c];
          }
          for (int gp = 0; gp < g; ++gp) {
            const float4 *src =
                reinterpret_cast<const float4 *>(seg0 + (size_t)gp * kInc + (size_t)f * kVDV + 16 * q4);
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
        tmem_st16(tbase + lane_off + SH::ColS + 64 * mt + 16 * q4, bits);
        if (!AGG && f < D) {
          *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4)) = pack8(bits);
          *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4 + 1)) = pack8(bits + 8);
        }
      }
    }
    if (half) {
      // Z: z0 gives the diagonal blocks (Mg2: Z_aa, Z_bb; Sg2: their sum,
      // kept in Z_aa); the cross blocks are never read
      float acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = 0.f;
      if (!AGG && r < kVDK) {
        if (z0) {
          const int hr = r / kVH;
          const float *zr0 = z0 + (size_t)bh * D + (V == kMg2 ? hr * 136 : 0);
          if (hr == 0) {
#pragma unroll
            for (int c = 0; c < kVH; ++c) acc[c] = zr0[psd16_row(r, c)];
          } else if (V == kMg2) {
#pragma unroll
            for (int c = 0; c < kVH; ++c) acc[kVH + c] = zr0[psd16_row(r - kVH, c)];
          }
        }
        for (int gp = 0; gp < g; ++gp) {
          const float4 *src =
              reinterpret_cast<const float4 *>(seg0 + (size_t)gp * kInc + (size_t)D * kVDV + r * kVDK);
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
      tmem_st32(tbase + lane_off + SH::ColZ, bits);
    }
  }

  // Zd snapshot (the readout's B operand for U = Q Zd) from Z in tensor memory:
  // quarter-0 lanes of half 1 hold the rows of Z
  auto snap_z = [&] {
    if (half && quarter == 0) {
      uint32_t zr[32];
      tmem_ld32(tbase + lane_off + SH::ColZ, zr);
      tmem_wait_ld();
      float zd[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float own = __uint_as_float(zr[c]);
        // the partner row of the other half, same column within its block
        const float other = __shfl_xor_sync(0xffffffffu, __uint_as_float(zr[c ^ 16]), 16);
        const bool same_block = (c >> 4) == (r >> 4);
        zd[c] = !same_block ? 0.f : (V == kMg2 ? own : own + other);
      }
      uint32_t bits[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) bits[c] = __float_as_uint(zd[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(zsnap + sw64(r, c)) = pack8(bits + 8 * c);
    }
  };
  if (!AGG) {
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    snap_z();
  }

  bool ok = true;
  for (int i = 0; ok && i < nchunks; ++i) {
    const int c0 = t0 + i * kVC;
    const bool valid = c0 + r < T;
    const int kvs = AGG ? (i & 1) : 0;                  // K, V stage of this chunk
    const uint32_t kvo = (uint32_t)(kKvStage1 * kvs);
    if (!(ok = wait_all(&bars[kVBarLoadKV + kvs], AGG ? (i >> 1) & 1 : i & 1))) break;
    // key tile M of the update (groups 2 M, 2 M + 1) into tile buffer tb
    auto tile_groups = [&](auto mc, uint8_t *tb) {
      constexpr int M = decltype(mc)::value;
      uint32_t XK[16], Ka[16], Kb[16], w[32];
      row_words(smem + L::K + kvo, r, XK);
      half_pairs(XK, 0, Ka);
      half_pairs(XK, 1, Kb);
      if constexpr (2 * M < NG) {
        group_words_c<V, true, 2 * M>(Ka, Kb, w);
        store_words(tb, r, w);
      }
      if constexpr (2 * M + 1 < NG) {
        group_words_c<V, true, 2 * M + 1>(Ka, Kb, w);
        store_words(tb + 16384, r, w);
      }
    };
    // S tile M += (tile buffer hb)^T V; Z += K^T K with the first tile
    auto issue_update = [&](int M, int hb, bool with_z) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss(tbase + SH::ColS + 64 * M, adv(d_tile, 32768 * hb + 2048 * kk),
               adv(d_v_mn, kvo + 2048 * kk), id_up, 1u);
      if (with_z) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tbase + SH::ColZ, adv(d_k_mn, kvo + 1024 * kk), adv(d_k_mn, kvo + 1024 * kk), id_z, 1u);
      }
    };

    if constexpr (AGG) {
      // ---- increment: the update only, two key tiles a round ----
      auto update_round = [&](auto m0c) -> bool {
        constexpr int M0 = decltype(m0c)::value;
        if (half) {
          if constexpr (M0 + 1 < NT) tile_groups(IC<M0 + 1>{}, buf + 32768);
        } else {
          tile_groups(IC<M0>{}, buf);
        }
        return round([&](int who) {
          if (who == 0) {
            issue_update(M0, 0, M0 == 0);
          } else {
            if constexpr (M0 + 1 < NT) issue_update(M0 + 1, 1, false);
          }
        });
      };
      ok = update_round(IC<0>{});
      if constexpr (NT > 2) {
        if (ok) ok = update_round(IC<2>{});
      }
      if (!ok) break;
      // this stage's K, V are no longer read: chunk i + 2 goes into it
      if (threadIdx.x == 0 && i + 2 < nchunks) load_kv(i + 2);
      continue;
    } else {
      if (!(ok = wait_all(&bars[kVBarLoadQ], i & 1))) break;
      // the state after this chunk is needed by the next chunk, or returned
      const bool upd = i < nchunks - 1 || state_out;
      uint32_t XQ[16], Pa[16], Pb[16];
      row_words(smem + L::Q, r, XQ);
      half_pairs(XQ, 0, Pa);
      half_pairs(XQ, 1, Pb);
      // query-feature group G into this half's readout slot
      auto slot_group = [&](auto gc) {
        constexpr int G = decltype(gc)::value;
        if constexpr (G < NG) {
          uint32_t w[32];
          group_words_c<V, false, G>(Pa, Pb, w);
          store_words(smem + L::Slot + 16384 * (G & 1), r, w);
        }
      };
      // O += slot (group G) x snapshot rows of group G
      auto issue_readout = [&](int G) {
        const int nk = G == NG - 1 ? 1 : 4;
        for (int kk = 0; kk < nk; ++kk)
          mma_ss(tbase + SH::ColO, adv(d_slot, 16384 * (G & 1) + 32 * kk),
                 adv(d_snap, (64 * G + 16 * kk) * 128), id_ro, 1u);
      };
      // intra-chunk blocks Q_u K_w^T for keys 64 b .. 64 b + 63 into the work columns
      auto issue_intra = [&](int b) {
#pragma unroll
        for (int j = 0; j < NA; ++j) {
          // block (u, w): Mg2 (0,0), (1,1); Sg2 (0,0), (0,1), (1,0), (1,1)
          const int u = V == kMg2 ? j : j >> 1, w = V == kMg2 ? j : j & 1;
          mma_ss(tbase + SH::ColW + 64 * j, adv(d_q, 32 * u), adv(d_k, 4096 * b + 32 * w), id_n64, 0);
        }
      };
      // P V for keys 64 b .. 64 b + 63, P (bf16) at column pc
      auto issue_pv = [&](int b, uint32_t pc) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tbase + SH::ColO, tbase + pc + 8 * kk, adv(d_v_mn, 8192 * b + 2048 * kk), id_pv,
                 (b > 0 || kk > 0) ? 1u : 0u);
      };
      // sum of squares of the blocks for this half's 32 keys, masked; P words
      float l_part = 0.f;
      auto weights = [&](int b, uint32_t (&p)[16]) {
        float wsum[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) wsum[c] = 0.f;
#pragma unroll
        for (int j = 0; j < NA; ++j) {
          uint32_t a[32];
          tmem_ld32(tbase + lane_off + SH::ColW + 64 * j + 32 * half, a);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float x = __uint_as_float(a[c]);
            wsum[c] = fmaf(x, x, wsum[c]);
          }
        }
        const int s0 = 64 * b + 32 * half;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float w0 = s0 + 2 * c <= r ? wsum[2 * c] : 0.f;
          const float w1 = s0 + 2 * c + 1 <= r ? wsum[2 * c + 1] : 0.f;
          l_part += w0 + w1;
          p[c] = pack_bf16x2(w0, w1);
        }
      };
      // P of the second key half: Mg2 after its two blocks, Sg2 over its
      // first block (read before the store)
      constexpr uint32_t kColP1 = V == kMg2 ? SH::ColW + 128 : SH::ColW;
      static_assert(V != kMg2 || SH::ColW + 160 <= kVTmemCols, "P of the second key half");

      // MMA round A: U = Q Zd, the blocks of keys 0..63
      ok = round([&](int who) {
        if (who == 0) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(tbase + SH::ColU, adv(d_q, 32 * kk), adv(d_z, 32 * kk), id_n32, kk);
        } else {
          issue_intra(0);
        }
      });
      if (!ok) break;
      float den_inter = 0.f;
      {
        uint32_t p[16];
        weights(0, p);
        if (half == 0) {
          uint32_t u[32];
          tmem_ld32(tbase + lane_off + SH::ColU, u);
          tmem_wait_ld();
#pragma unroll
          for (int w = 0; w < 16; ++w) {
            const float2 qq = bf2f(XQ[w]);
            den_inter = fmaf(qq.x, __uint_as_float(u[2 * w]), den_inter);
            den_inter = fmaf(qq.y, __uint_as_float(u[2 * w + 1]), den_inter);
          }
        }
        __syncthreads();       // U and the blocks are read: P of keys 0..63 goes to U's columns
        tmem_st16(tbase + lane_off + SH::ColU + 16 * half, p);
      }
      if (half) slot_group(IC<1>{}); else slot_group(IC<0>{});
      // MMA round B: P V (keys 0..63), the blocks of keys 64..127, readout groups 0, 1
      ok = round([&](int who) {
        if (who == 0) {                          // the O accumulator
          issue_pv(0, SH::ColU);
          issue_readout(0);
          issue_readout(1);
        } else {
          issue_intra(1);
        }
      });
      if (!ok) break;
      {
        uint32_t p[16];
        weights(1, p);
        __syncthreads();       // every thread has read the blocks
        tmem_st16(tbase + lane_off + kColP1 + 16 * half, p);
      }
      if (half) lx[r] = l_part;
      if (half) slot_group(IC<3>{}); else slot_group(IC<2>{});
      if (upd) {
        if (half) tile_groups(IC<1>{}, buf + 32768); else tile_groups(IC<0>{}, buf);
      }
      // MMA round C: P V (keys 64..127), readout groups 2, 3, update of tiles 0, 1 and Z
      ok = round([&](int who) {
        if (who == 0) {                          // O, and state tile 1
          issue_pv(1, kColP1);
          issue_readout(2);
          if (NG > 4) issue_readout(3);
          if (upd) issue_update(1, 1, false);
        } else if (upd) {                        // state tile 0 and Z
          issue_update(0, 0, true);
        }
      });
      if (!ok) break;
      if constexpr (NG > 4) {
        // MMA round D (Mg2): readout group 4, update of tile 2
        if (!half) slot_group(IC<4>{});
        if (upd && !half) tile_groups(IC<2>{}, buf);
        ok = round([&](int who) {
          if (who == 0) {
            issue_readout(4);
          } else if (upd) {
            issue_update(2, 0, false);
          }
        });
        if (!ok) break;
      }
      if (threadIdx.x == 0 && i + 1 < nchunks) {
        load_q(i + 1);                                           // Q, K, V no longer read
        load_kv(i + 1);
      }

      // ---- y = O / (l + q^T Zd q) ----
      if (!half) {
        const float den = l_part + lx[r] + den_inter;
        if (valid && !(den > 0.f)) flag_status(status, kStatusNonPositiveNormaliser);
        const float inv = 1.f / den;
        const float2 inv2 = make_float2(inv, inv);
#pragma unroll 1
        for (int hv = 0; hv < 2; ++hv) {
          uint32_t acc[32];
          tmem_ld32(tbase + lane_off + SH::ColO + 32 * hv, acc);
          tmem_wait_ld();
          if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)bh * T + c0 + r) * kVDV + 32 * hv);
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[c] = psd::pack8_scaled(acc + 8 * c, inv2);
          }
        }
      }
      // ---- snapshot S_c+1 and Zd_c+1 (not after the last chunk) ----
      if (i < nchunks - 1) {
        for (int mt = half; mt < NT; mt += 2) {
          const int f = 128 * mt + r;
          uint32_t a[32], b2[32];
          tmem_ld32(tbase + lane_off + SH::ColS + 64 * mt, a);
          tmem_ld32(tbase + lane_off + SH::ColS + 64 * mt + 32, b2);
          tmem_wait_ld();
          if (f < D) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              *reinterpret_cast<uint4 *>(snap + sw128(f, q4)) = pack8(a + 8 * q4);
              *reinterpret_cast<uint4 *>(snap + sw128(f, 4 + q4)) = pack8(b2 + 8 * q4);
            }
          }
        }
        snap_z();
      }
    }
  }

  // ---- the state leaving the kernel: the increment (internal order), or
  //      the final state in the library's order ----
  if (ok && nchunks > 0 && (AGG || state_out)) {
    float *dst_agg = agg + ((size_t)bh * G_total + g) * kInc;
    for (int mt = half; mt < NT; mt += 2) {
      const int f = 128 * mt + r;
      uint32_t a[32], b2[32];
      tmem_ld32(tbase + lane_off + SH::ColS + 64 * mt, a);
      tmem_ld32(tbase + lane_off + SH::ColS + 64 * mt + 32, b2);
      tmem_wait_ld();
      if (f >= D) continue;
      float *row;
      float sc = 1.f;
      if (AGG) {
        row = dst_agg + (size_t)f * kVDV;
      } else {
        bool diag;
        const int lr = var_abi_row<V>(f, diag);
        sc = diag ? 1.f : 0.5f;
        row = S_out ? S_out + ((size_t)bh * D + lr) * kVDV : nullptr;
      }
      if (row) {
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
    if (half && quarter == 0) {
      uint32_t zr[32];
      tmem_ld32(tbase + lane_off + SH::ColZ, zr);
      tmem_wait_ld();
      if (AGG) {
        float *row = dst_agg + (size_t)D * kVDV + r * kVDK;
#pragma unroll
        for (int c = 0; c < 32; ++c) row[c] = __uint_as_float(zr[c]);
      } else {
        float other[32];
#pragma unroll
        for (int c = 0; c < 32; ++c)
          other[c] = __shfl_xor_sync(0xffffffffu, __uint_as_float(zr[c ^ 16]), 16);
        if (z_out) {
          // library z of pair (i, j) of a half: Mg2 Z_aa or Z_bb, Sg2 their sum
          const int hr = r / kVH, i = r % kVH;
          if (V == kMg2) {
#pragma unroll
            for (int j = 0; j < kVH; ++j)
              if (j >= i)
                z_out[(size_t)bh * D + hr * 136 + psd16_row(i, j)] =
                    __uint_as_float(hr ? zr[kVH + j] : zr[j]);
          } else if (hr == 0) {
#pragma unroll
            for (int j = 0; j < kVH; ++j)
              if (j >= i) z_out[(size_t)bh * D + psd16_row(i, j)] = __uint_as_float(zr[j]) + other[j];
          }
        }
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) flag_status(status, kStatusDeviceTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, kVTmemCols);
}

template <int V>
cudaError_t launch_var(const ChunkedLaunch &a, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, int G, int seg_len) {
  cudaError_t e;
  if (G > 1) {
    auto kinc = var_tc_kernel<V, true>;
    e = cudaFuncSetAttribute(kinc, cudaFuncAttributeMaxDynamicSharedMemorySize, VarSmem::Bytes);
    if (e != cudaSuccess) return e;
    ProfileScope prof("tc_variant_increment", a.stream);
    kinc<<<(unsigned)(a.BH * (G - 1)), kVThreads, VarSmem::Bytes, a.stream>>>(
        tq, tk, tv, a.agg, nullptr, nullptr, nullptr, nullptr, nullptr, a.status, a.T, G - 1, G,
        seg_len);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  auto kern = var_tc_kernel<V, false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, VarSmem::Bytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_variant_pass", a.stream);
  kern<<<(unsigned)(a.BH * G), kVThreads, VarSmem::Bytes, a.stream>>>(
      tq, tk, tv, a.agg, static_cast<__nv_bfloat16 *>(a.o), a.S0, a.z0, a.S_out, a.z_out, a.status,
      a.T, G, G, seg_len);
  return cudaGetLastError();
}

}  // namespace

bool var_tc_supported(const ChunkedLaunch &a, int d_k, int d_v, int C, int feature) {
  if ((feature != kMg2 && feature != kSg2) || d_k != kVDK || d_v != kVDV || (C != 64 && C != kVC) ||
      a.T <= 0 || a.state_only)
    return false;
  for (const void *p : {a.q, a.k, a.v, (const void *)a.o})
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return false;
  for (const void *p : {(const void *)a.S_out, (const void *)a.S0})
    if (p && reinterpret_cast<uintptr_t>(p) % 16 != 0) return false;
  return true;
}

void var_tc_layout(long long BH, int T, int sms, bool sequential, int *G, int *seg_len) {
  const int g_req = (sequential || BH >= sms) ? 1 : (int)(sms / BH);
  tile_segments(T, kVC, g_req, G, seg_len);
}

cudaError_t var_tc(const ChunkedLaunch &a, int feature) {
  int G, seg_len;
  var_tc_layout(a.BH, a.T, a.sms, a.sequential, &G, &seg_len);
  CUtensorMap tq, tk, tv;
  if (!make_tma_3d_bf16(&tq, a.q, kVDK, a.T, a.BH, kVC) ||
      !make_tma_3d_bf16(&tk, a.k, kVDK, a.T, a.BH, kVC) ||
      !make_tma_3d_bf16(&tv, a.v, kVDV, a.T, a.BH, kVC))
    return cudaErrorInvalidValue;
  return feature == kMg2 ? launch_var<kMg2>(a, tq, tk, tv, G, seg_len)
                         : launch_var<kSg2>(a, tq, tk, tv, G, seg_len);
}

}  // namespace kata
