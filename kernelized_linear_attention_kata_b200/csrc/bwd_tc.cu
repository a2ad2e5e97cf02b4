// Tensor-core (tcgen05 / TMEM / TMA) gradient of the chunked PSD forward,
// bf16 inputs, d_k = 32, d_v = 64, fp32 accumulation.
//
// The chain rule of y_t = sum_(s<=t) w_ts v_s / sum_(s<=t) w_ts with
// w_ts = (q_t . k_s)^2 (KATA explainer section 2.3: the exact chunked form;
// arXiv abstract: the models are trained with these kernels): with
// d_t = sum_(s<=t) w_ts, n_t = sum_(s<=t) w_ts v_s, g_t = dout_t / d_t and
// c_t = -(dout_t . n_t) / d_t^2,
//   e_ts = g_t . v_s + c_t                       (dL/dw_ts, s <= t)
//   dq_t = sum_(s<=t) e_ts 2 (q_t . k_s) k_s.
// Inside a chunk of 128 tokens this is a dense block; the earlier chunks
// enter through the prefix state (S, Z) of the forward:
//   dout_t . n_t (carried) = phi_q(q_t) . (S dout_t),  d_t (carried) = q_t^T Z q_t,
//   dq_t (carried)         = J(q_t)^T (S dout_t) / d_t + 2 c_t Z q_t,
// J the Jacobian of the query feature. Per chunk (bf16 operands, fp32
// accumulators in tensor memory):
//   A  = Q K^T, D' = dout V^T                  the intra-chunk blocks, in two
//                                              halves of 64 keys
//   X  = dout S^T                              64 features at a time; the
//                                              CUDA cores contract X with the
//                                              query features and their
//                                              Jacobian
//   U  = Q Z
//   M  = 2 A (D' / d_t + c_t), masked to s <= t, then dq += M K
//   S += phi(K)^T V,  Z += K^T K               the forward's update.
// The kernel writes dq and, per token, d_t and c_t for the suffix pass.
//
// Parallel carry: the forward's segment increments (one launch of the
// forward's increment kernel) give segment g of a head the sum of segments
// 0 .. g-1 as its carry-in; each CTA then walks its segment's chunks.
//
// The kernel is synchronous: 256 threads (8 warps, two per TMEM lane
// quarter; "half" h = warp / 4 splits each phase's columns). Threads 0 and
// 32 issue a round of MMAs, each accumulator's chain from one of them (one
// thread issues an N <= 64 MMA only every 75-100 cycles, so two issue about
// twice as fast), and commit them to one barrier that every thread waits
// on. The state, the feature order and its doubled off-diagonal rows are
// the forward's (psd_tc_common.cuh).
//
// Tensor memory (512 columns, fp32):
//   [  0, 320)  S, five 128-feature tiles of 64 columns (tile 4: 16 rows used)
//   [320, 352)  Z (lanes 0..31)
//   [352, 384)  U = Q Z_c, then the dq accumulator
//   [384, 512)  work: A | D' (64 keys each), or two 64-feature X blocks, or
//               M (bf16) in the A columns
#include "common.cuh"
#include "launch.h"
#include "profile.h"
#include "tc_common.cuh"
#include "tma_host.h"
#include "psd_tc_common.cuh"

namespace kata {
namespace {

using namespace tc;
using namespace psd;

template <int N> using IC = std::integral_constant<int, N>;

constexpr int kBThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColZ = 320, kColDq = 352, kColA = 384, kColB = 448;

// Shared memory (byte offsets from a 1024-aligned base).
struct DqSmem {
  static constexpr int Q = 0;                      // [128][32] bf16, 64-byte swizzle
  static constexpr int K = 8192;                   // [128][32] bf16, 64-byte swizzle
  static constexpr int V = 16384;                  // [128][64] bf16, 128-byte swizzle
  static constexpr int dO = 32768;                 // [128][64] bf16, 128-byte swizzle
  static constexpr int Snap = 49152;               // S_c bf16 [528][64], 128-byte rows
  static constexpr int ZSnap = Snap + kD * 128;    // Z_c bf16 [32][32], 64-byte rows
  static constexpr int Key = ZSnap + 2048;         // two key-feature tiles of 32 KB
  static constexpr int Xch = Key + 2 * 32768;      // [128][36] fp32: half 1's partial sums
  static constexpr int Ubuf = Xch + 128 * 36 * 4;  // [128][32] fp32: u = Z_c q
  static constexpr int InvD = Ubuf + 128 * 32 * 4; // [128] fp32: 1 / d_t
  static constexpr int Cc = InvD + 512;            // [128] fp32: c_t
  static constexpr int Bars = Cc + 512;
  static constexpr int Bytes = Bars + 64 + 1024;   // barriers + alignment slack
  static_assert(Snap % 1024 == 0 && ZSnap % 1024 == 0 && Key % 1024 == 0, "swizzle atoms");
  static_assert(Bytes <= 232448, "shared memory budget");
};
enum { kBarLoadQ = 0, kBarLoadKV, kBarMma, kNumBars };

// One thread's q (or k) row as 32 fp32 values from a 64-byte-swizzled tile.
__device__ __forceinline__ void row_f32(const uint8_t *tile, int row, float (&x)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4 *>(tile + sw64(row, c));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&w[j]);
      x[8 * c + 2 * j] = __low2float(b);
      x[8 * c + 2 * j + 1] = __high2float(b);
    }
  }
}

template <int N>
__device__ __forceinline__ void rot(float (&R)[32]) {
  float t[32];
#pragma unroll
  for (int l = 0; l < 32; ++l) t[l] = R[(l + N) & 31];
#pragma unroll
  for (int l = 0; l < 32; ++l) R[l] = t[l];
}

// Contraction of one offset d of the feature order (features (l, (l+d) mod 32)
// for l < nl) with its X values: x[l] = X_(d,l) (the state's doubled rows make
// X_f = m_f (S dout)_f). qR = q rotated by d, g2R accumulates the Jacobian's
// second term in the same rotated frame; both are rotated by one afterwards.
// DN adds the contraction with the features themselves (dout . n).
template <int NL, bool DN = true>
__device__ __forceinline__ void contract_offset(const uint32_t *x, const float (&q)[32],
                                                float (&qR)[32], float (&h)[32], float (&g2R)[32],
                                                float &dn) {
#pragma unroll
  for (int l = 0; l < NL; ++l) {
    const float xv = __uint_as_float(x[l]);
    if constexpr (DN) dn = fmaf(q[l] * qR[l], xv, dn);
    h[l] = fmaf(qR[l], xv, h[l]);
    g2R[l] = fmaf(q[l], xv, g2R[l]);
  }
  rot<1>(qR);
  rot<1>(g2R);
}

__global__ void __launch_bounds__(kBThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                 const float *__restrict__ aggS, __nv_bfloat16 *__restrict__ dq,
                 float *__restrict__ den_out, float *__restrict__ c_out,
                 unsigned *__restrict__ status, int T, int G, int seg_len) {
  using L = DqSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::Bars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::Bars + 8 * kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::Bars + 8 * kNumBars + 4);
  float *xch = reinterpret_cast<float *>(smem + L::Xch);
  float *ubuf = reinterpret_cast<float *>(smem + L::Ubuf);
  float *invd_s = reinterpret_cast<float *>(smem + L::InvD);
  float *c_s = reinterpret_cast<float *>(smem + L::Cc);
  uint8_t *snap = smem + L::Snap;
  uint8_t *zsnap = smem + L::ZSnap;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int quarter = warp & 3, half = warp >> 2;
  const int r = quarter * 32 + lane;                  // TMEM lane: token / feature row
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  const int g = blockIdx.x % G, bh = blockIdx.x / G;
  const int t0 = g * seg_len, t1 = min(T, t0 + seg_len);
  const int nchunks = (t1 - t0 + kC - 1) / kC;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kBarLoadQ], 1);
    mbar_init(&bars[kBarLoadKV], 1);
    mbar_init(&bars[kBarMma], 2);                 // one commit per issuing thread
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  auto load_q = [&](int i) {        // Q and dout of chunk i
    mbar_arrive_expect_tx(&bars[kBarLoadQ], 8192 + 16384);
    tma_load_3d(smem + L::Q, &tmq, &bars[kBarLoadQ], 0, t0 + i * kC, bh);
    tma_load_3d(smem + L::dO, &tmo, &bars[kBarLoadQ], 0, t0 + i * kC, bh);
  };
  auto load_kv = [&](int i) {       // K and V of chunk i
    mbar_arrive_expect_tx(&bars[kBarLoadKV], 8192 + 16384);
    tma_load_3d(smem + L::K, &tmk, &bars[kBarLoadKV], 0, t0 + i * kC, bh);
    tma_load_3d(smem + L::V, &tmv, &bars[kBarLoadKV], 0, t0 + i * kC, bh);
  };
  if (threadIdx.x == 0 && nchunks > 0) {
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    tma_prefetch_desc(&tmo);
    load_q(0);
    load_kv(0);
  }

  // One synchronous round: every thread's operand writes (shared memory,
  // tensor memory) and tensor-memory reads are complete, threads 0 and 32
  // issue the MMAs (issue(0), issue(1): every accumulator's MMAs from one of
  // them) and commit them, every thread waits. The result is uniform over
  // the CTA, so a timeout ends every thread's loop at the same point.
  uint32_t mph = 0;
  // round_with also runs CUDA-core work while the MMAs are in flight: work
  // that neither reads nor writes what they touch.
  auto round_with = [&](auto issue, auto work) -> bool {
    tmem_wait_ld();
    tmem_wait_st();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 || threadIdx.x == 32) {
      tc_fence_after();
      issue(threadIdx.x >> 5);
      mma_commit(&bars[kBarMma]);
    }
    work();
    const bool ok = mbar_wait(&bars[kBarMma], mph, abort_flag);
    mph ^= 1;
    tc_fence_after();
    return __syncthreads_and(ok);
  };
  auto round = [&](auto issue) -> bool { return round_with(issue, [] {}); };
  auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
    return __syncthreads_and(mbar_wait(bar, parity, abort_flag));
  };

  // Descriptors (start-address field advanced by bytes / 16 for sub-tiles).
  auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
  const uint64_t d_q = smem_desc(smem_u32(smem + L::Q), 16, 512, kSw64);          // K-major
  const uint64_t d_k = smem_desc(smem_u32(smem + L::K), 16, 512, kSw64);          // K-major
  const uint64_t d_k_mn = smem_desc(smem_u32(smem + L::K), 8192, 512, kSw64);     // MN-major
  const uint64_t d_v = smem_desc(smem_u32(smem + L::V), 16, 1024, kSw128);        // K-major
  const uint64_t d_v_mn = smem_desc(smem_u32(smem + L::V), 16384, 1024, kSw128);  // MN-major
  const uint64_t d_o = smem_desc(smem_u32(smem + L::dO), 16, 1024, kSw128);       // K-major
  const uint64_t d_snap = smem_desc(smem_u32(snap), 16, 1024, kSw128);            // K-major
  const uint64_t d_z = smem_desc(smem_u32(zsnap), 16, 512, kSw64);
  const uint64_t d_key = smem_desc(smem_u32(smem + L::Key), 16384, 1024, kSw128); // MN-major
  constexpr uint32_t id_n64 = idesc_bf16(128, 64, false, false);
  constexpr uint32_t id_n32 = idesc_bf16(128, 32, false, false);
  constexpr uint32_t id_n16 = idesc_bf16(128, 16, false, false);
  constexpr uint32_t id_mk = idesc_bf16(128, 32, false, true);      // M (TMEM) x K_b (MN-major)
  constexpr uint32_t id_up = idesc_bf16(128, 64, true, true);
  constexpr uint32_t id_z = idesc_bf16(128, 32, true, true);

  // A = Q K_b^T and D' = dout V_b^T for keys 64 b .. 64 b + 63
  auto issue_intra = [&](int b, int who) {
    if (who == 0) {
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
        mma_ss(tbase + kColA, adv(d_q, 32 * kk), adv(d_k, 4096 * b + 32 * kk), id_n64, kk);
    } else {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tbase + kColB, adv(d_o, 32 * kk), adv(d_v, 8192 * b + 32 * kk), id_n64, kk);
    }
  };

  // ---- carry-in: S, Z = the increments of segments 0 .. g-1 ----
  {
    const float *seg0 = aggS + (size_t)bh * G * kAggFloats;
    // half 0: tiles 0, 1 and 4; half 1: tiles 2, 3 and Z
    for (int m = half ? 2 : 0; m < (half ? 4 : 2) + (half ? 0 : 1); ++m) {
      const int mt = (!half && m == 2) ? 4 : m;
      const int f = 128 * mt + r;
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        float acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = 0.f;
        if (f < kD) {
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
        tmem_st16(tbase + lane_off + kColS + 64 * mt + 16 * q4, bits);
        if (f < kD) {
          *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4)) = pack8(bits);
          *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4 + 1)) = pack8(bits + 8);
        }
      }
    }
    if (half) {
      float acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = 0.f;
      if (r < kDK) {
        for (int gp = 0; gp < g; ++gp) {
          const float4 *src =
              reinterpret_cast<const float4 *>(seg0 + (size_t)gp * kAggFloats + kD * kDV + r * kDK);
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
      tmem_st32(tbase + lane_off + kColZ, bits);
      if (quarter == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(zsnap + sw64(r, c)) = pack8(bits + 8 * c);
      }
    }
  }

  bool ok = true;
  for (int i = 0; ok && i < nchunks; ++i) {
    const int c0 = t0 + i * kC;
    const bool valid = c0 + r < T;
    if (!(ok = wait_all(&bars[kBarLoadQ], i & 1) && wait_all(&bars[kBarLoadKV], i & 1))) break;
    float q[32];
    row_f32(smem + L::Q, r, q);

    // ---- intra-chunk row sums: l = sum_s w_ts, dn = sum_s w_ts (dout_t . v_s) ----
    float l_part = 0.f, dn_part = 0.f, den_inter = 0.f;
    for (int b = 0; ok && b < 2; ++b) {
      ok = round([&](int who) {
        if (b == 0 && who == 0) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(tbase + kColDq, adv(d_q, 32 * kk), adv(d_z, 32 * kk), id_n32, kk);
        }
        issue_intra(b, who);
      });
      if (!ok) break;
      uint32_t a[32], dp[32];
      tmem_ld32(tbase + lane_off + kColA + 32 * half, a);
      tmem_ld32(tbase + lane_off + kColB + 32 * half, dp);
      tmem_wait_ld();
      const int s0 = 64 * b + 32 * half;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float av = __uint_as_float(a[j]);
        const float w = s0 + j <= r ? av * av : 0.f;
        l_part += w;
        dn_part = fmaf(w, __uint_as_float(dp[j]), dn_part);
      }
      if (b == 0 && half == 0) {
        // u = Z_c q: the carried denominator q^T Z_c q, and 2 c_t u for dq
        uint32_t u[32];
        tmem_ld32(tbase + lane_off + kColDq, u);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) den_inter = fmaf(q[j], __uint_as_float(u[j]), den_inter);
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4 *>(ubuf + r * 32 + j) =
              make_float4(__uint_as_float(u[j]), __uint_as_float(u[j + 1]),
                          __uint_as_float(u[j + 2]), __uint_as_float(u[j + 3]));
      }
    }
    if (!ok) break;

    // ---- carried part: X = dout S_c^T, 64 features a round and half ----
    // half 0 takes features 0 .. 255 (offsets d = 0 .. 7), half 1 features
    // 256 .. 527 (d = 8 .. 15 and the 16 pairs (l, l + 16)).
    float h[32], g2R[32], qR[32];
#pragma unroll
    for (int l = 0; l < 32; ++l) {
      h[l] = 0.f;
      g2R[l] = 0.f;
      qR[l] = q[l];
    }
    if (half) rot<8>(qR);
    float dn_car = 0.f;
    // four rounds; the last also takes the 16 features of tile 4 (half 1's)
    // into the dq columns, free between the read of U and the first dq MMA
    for (int j = 0; ok && j < 4; ++j) {
      ok = round([&](int who) {
        if (who == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tbase + kColA, adv(d_o, 32 * kk), adv(d_snap, 64 * j * 128 + 32 * kk), id_n64, kk);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tbase + kColB, adv(d_o, 32 * kk), adv(d_snap, (256 + 64 * j) * 128 + 32 * kk),
                   id_n64, kk);
          if (j == 3) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tbase + kColDq, adv(d_o, 32 * kk), adv(d_snap, 512 * 128 + 32 * kk), id_n16, kk);
          }
        }
      });
      if (!ok) break;
      uint32_t x[32];
      tmem_ld32(tbase + lane_off + kColA + 64 * half, x);
      tmem_wait_ld();
      contract_offset<32>(x, q, qR, h, g2R, dn_car);
      tmem_ld32(tbase + lane_off + kColA + 64 * half + 32, x);
      tmem_wait_ld();
      contract_offset<32>(x, q, qR, h, g2R, dn_car);
      if (j == 3 && half) {
        uint32_t x16[16];
        tmem_ld16(tbase + lane_off + kColDq, x16);
        tmem_wait_ld();
        contract_offset<16>(x16, q, qR, h, g2R, dn_car);
      }
    }
    if (!ok) break;
    // back to the unrotated frame: half 0 ended at offset 8, half 1 at 17
    if (half) {
      rot<15>(g2R);
    } else {
      rot<24>(g2R);
    }
#pragma unroll
    for (int l = 0; l < 32; ++l) h[l] += g2R[l];

    // ---- combine the halves (d_t, c_t, the carried dq) while the intra
    //      blocks of keys 0..63 are recomputed; then M = 2 A (D' / d_t + c_t)
    //      masked, dq += M K_b ----
    if (half) {
      float *row = xch + r * 36;
      row[32] = l_part;
      row[33] = dn_part + dn_car;
#pragma unroll
      for (int l = 0; l < 32; l += 4)
        *reinterpret_cast<float4 *>(row + l) = make_float4(h[l], h[l + 1], h[l + 2], h[l + 3]);
    }
    float dqc[32];
    auto combine = [&] {        // half 1's partial sums are in xch (the round's barrier)
      if (!half) {
        const float *row = xch + r * 36;
        const float l_all = l_part + row[32];
        const float dn_all = dn_part + dn_car + row[33];
        const float d = l_all + den_inter;
        if (valid && !(d > 0.f)) flag_status(status, kStatusNonPositiveNormaliser);
        const float inv = valid ? 1.f / d : 0.f;
        const float ct = valid ? -dn_all * inv * inv : 0.f;
        invd_s[r] = inv;
        c_s[r] = ct;
        if (valid) {
          den_out[(size_t)bh * T + c0 + r] = d;
          c_out[(size_t)bh * T + c0 + r] = ct;
        }
        const float *u = ubuf + r * 32;
#pragma unroll
        for (int l = 0; l < 32; ++l) dqc[l] = inv * (h[l] + row[l]) + 2.f * ct * u[l];
      }
    };
    // The update S += phi(K)^T V, Z += K^T K (the state of the next chunk)
    // rides in the next three rounds, which touch neither S nor Z: update
    // round U (tiles (0, 2) and Z, then (1, 3), then 4) in the combine round,
    // the first dq += M K round and the second intra round. Its key features
    // (two 32 KB tiles, one per half) are written before each of them.
    const bool upd = i + 1 < nchunks;        // the state after the segment is not needed
    auto write_upd = [&](auto uc) {
      constexpr int U = decltype(uc)::value;
      constexpr int M0 = U < 2 ? U : 4, M1 = U < 2 ? 2 + U : -1;   // this round's tiles, per half
      uint32_t XK[16], P[32], R2[32];
      load_pairs(smem + L::K, r, XK, P);
      if (!half) {
#pragma unroll
        for (int l = 0; l < 32; ++l) R2[l] = bmul2(P[(l + 4 * M0) & 31], 0x40004000u);   // x 2.0
        write_tile(smem + L::Key, r, M0 == kTiles - 1, M0 == 0 ? 0x3f003f00u : 0x3f803f80u, P, R2);
      } else if constexpr (M1 >= 0) {
#pragma unroll
        for (int l = 0; l < 32; ++l) R2[l] = bmul2(P[(l + 4 * M1) & 31], 0x40004000u);
        write_tile(smem + L::Key + 32768, r, false, 0x3f803f80u, P, R2);
      }
    };
    auto issue_upd = [&](int u, int who) {
      const int ma = u < 2 ? u : 4, mb = 2 + u;
      if (who == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tbase + kColS + 64 * ma, adv(d_key, 2048 * kk), adv(d_v_mn, 2048 * kk), id_up, 1);
        if (u == 0) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tbase + kColZ, adv(d_k_mn, 1024 * kk), adv(d_k_mn, 1024 * kk), id_z, 1);
        }
      } else if (u < 2) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tbase + kColS + 64 * mb, adv(d_key, 32768 + 2048 * kk), adv(d_v_mn, 2048 * kk),
                 id_up, 1);
      }
    };
    for (int b = 0; ok && b < 2; ++b) {
      if (b == 0) {
        if (upd) write_upd(IC<0>{});
        ok = round_with([&](int who) {
          issue_intra(0, who);
          if (upd) issue_upd(0, who);
        }, combine);
      } else {
        if (upd) write_upd(IC<2>{});
        ok = round([&](int who) {
          issue_intra(1, who);
          if (upd) issue_upd(2, who);
        });
      }
      if (!ok) break;
      if (b == 1 && threadIdx.x == 0 && i + 1 < nchunks) load_q(i + 1);   // Q, dout read
      const float inv_r = invd_s[r], c_r = c_s[r];
      uint32_t a[32], dp[32], m[16];
      tmem_ld32(tbase + lane_off + kColA + 32 * half, a);
      tmem_ld32(tbase + lane_off + kColB + 32 * half, dp);
      tmem_wait_ld();
      const int s0 = 64 * b + 32 * half;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float a0 = __uint_as_float(a[2 * j]), a1 = __uint_as_float(a[2 * j + 1]);
        const float e0 = fmaf(__uint_as_float(dp[2 * j]), inv_r, c_r);
        const float e1 = fmaf(__uint_as_float(dp[2 * j + 1]), inv_r, c_r);
        const float m0 = s0 + 2 * j <= r ? 2.f * a0 * e0 : 0.f;
        const float m1 = s0 + 2 * j + 1 <= r ? 2.f * a1 * e1 : 0.f;
        m[j] = pack_bf16x2(m0, m1);
      }
      if (b == 0 && upd) write_upd(IC<1>{});   // the first update (the last MMA round) read its tiles
      __syncthreads();          // every thread has read A and D' before M overwrites A
      tmem_st16(tbase + lane_off + kColA + 16 * half, m);
      ok = round([&](int who) {
        if (who == 0) {                          // one accumulator: one issuing thread
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tbase + kColDq, tbase + kColA + 8 * kk, adv(d_k_mn, 4096 * b + 1024 * kk), id_mk,
                   (b > 0 || kk > 0) ? 1u : 0u);
        }
        if (b == 0 && upd) issue_upd(1, who);
      });
    }
    if (!ok) break;
    // dq = the intra part (tensor memory) + the carried part (half 0)
    auto write_dq = [&] {
      if (!half) {
        uint32_t acc[32];
        tmem_ld32(tbase + lane_off + kColDq, acc);
        tmem_wait_ld();
        if (valid) {
          uint4 *dst = reinterpret_cast<uint4 *>(dq + ((size_t)bh * T + c0 + r) * kDK);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              w[j] = pack_bf16x2(__uint_as_float(acc[8 * c + 2 * j]) + dqc[8 * c + 2 * j],
                                 __uint_as_float(acc[8 * c + 2 * j + 1]) + dqc[8 * c + 2 * j + 1]);
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    };
    write_dq();
    if (i == nchunks - 1) break;            // the state after the segment is not needed

    if (threadIdx.x == 0) load_kv(i + 1);             // K, V of this chunk no longer read
    // ---- snapshot S_c+1 (half 0: tiles 0, 1, 4; half 1: tiles 2, 3) and Z_c+1 ----
    for (int m = half ? 2 : 0; m < (half ? 4 : 3); ++m) {
      const int mt = (!half && m == 2) ? 4 : m;
      if (mt == 4 && quarter != 0) continue;        // tile 4: rows 512..527 (lanes 0..15)
      const int f = 128 * mt + r;
      uint32_t a[32], b2[32];
      tmem_ld32(tbase + lane_off + kColS + 64 * mt, a);
      tmem_ld32(tbase + lane_off + kColS + 64 * mt + 32, b2);
      tmem_wait_ld();
      if (f < kD) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          *reinterpret_cast<uint4 *>(snap + sw128(f, q4)) = pack8(a + 8 * q4);
          *reinterpret_cast<uint4 *>(snap + sw128(f, 4 + q4)) = pack8(b2 + 8 * q4);
        }
      }
    }
    if (half && quarter == 0) {
      uint32_t zr[32];
      tmem_ld32(tbase + lane_off + kColZ, zr);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(zsnap + sw64(r, c)) = pack8(zr + 8 * c);
    }
  }
  if (*abort_flag && threadIdx.x == 0) flag_status(status, kStatusDeviceTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

// ---------------------------------------------------------------------------
// The suffix pass: dk and dv, chunks in reverse order.
//
// With the suffix state R = sum_(t in later chunks) phi_q(q_t) g_t^T and
// Rq = sum c_t q_t q_t^T (so that r . phi(k) = k^T Rq k):
//   dv_s (carried) = R^T phi(k_s),
//   dk_s (carried) = J(k_s)^T (R v_s) + 2 Rq k_s,
//   dv_s (intra)   = sum_(t>=s) w_ts g_t,
//   dk_s (intra)   = sum_(t>=s) e_ts 2 (q_t . k_s) q_t,
// then R += phi_q(Q_c)^T G_c, Rq += Q_c^T diag(c) Q_c. R is held with the
// off-diagonal rows doubled (R'_f = m_f R_f), as the forward holds S, so that
// plain key products read it out.
//
// Tensor memory (512 columns, fp32):
//   [  0, 320)  R', five 128-feature tiles
//   [320, 352)  Rq (lanes 0..31)
//   [352, 384)  U2 = K Rq, then the dk accumulator
//   [384, 448)  the dv accumulator (first a 64-feature Y block of half 0)
//   [448, 512)  work: a Y block of half 1; K Q^T | V dout^T (32 queries
//               each); W~ | M (bf16)
// The suffix increments (R', Rq of segments 1 .. G-1, the carry-in of the
// earlier segments) come from the forward's increment kernel in its suffix
// form (psd_tc_suffix_increments).
// ---------------------------------------------------------------------------
constexpr uint32_t kColR = 0, kColRq = 320, kColDk = 352, kColDv = 384, kColW = 448;
constexpr int kQSlotsPsd = 9;      // 64-feature slots of the readout (the last holds 16)

struct DkvSmem {
  static constexpr int Q = 0;
  static constexpr int K = 8192;
  static constexpr int V = 16384;
  static constexpr int dO = 32768;
  static constexpr int Snap = 49152;                 // R' bf16 [528][64]
  static constexpr int RqSnap = Snap + kD * 128;     // Rq bf16 [32][32]
  static constexpr int Slots = RqSnap + 2048;        // 2 x 16 KB key-product slots, or
                                                     // 2 x 32 KB query-feature tiles
  static constexpr int CQ = Slots + 2 * 32768;       // [128][32] bf16 c_t q_t, 64-byte swizzle
  static constexpr int Xch = CQ + 8192;              // [128][36] fp32
  static constexpr int Ubuf = Xch + 128 * 36 * 4;    // [128][32] fp32: Rq k
  static constexpr int InvD = Ubuf + 128 * 32 * 4;
  static constexpr int Cc = InvD + 512;
  static constexpr int Bars = Cc + 512;
  static constexpr int Bytes = Bars + 64 + 1024;
  static_assert(Snap % 1024 == 0 && RqSnap % 1024 == 0 && Slots % 1024 == 0 && CQ % 1024 == 0,
                "swizzle atoms");
  // the Rq update's A operand (M = 128 over a 32-row tile) reads three more
  // 8 KB atoms past CQ: they must lie inside the allocation
  static_assert(CQ + 4 * 8192 <= Bars, "padded A rows of the Rq update");
  static_assert(Bytes <= 232448, "shared memory budget");
};

__global__ void __launch_bounds__(kBThreads, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                   float *__restrict__ aggR, const float *__restrict__ den,
                   const float *__restrict__ cvec, __nv_bfloat16 *__restrict__ dk,
                   __nv_bfloat16 *__restrict__ dv, unsigned *__restrict__ status, int T, int G,
                   int seg_len) {
  using L = DkvSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::Bars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::Bars + 8 * kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::Bars + 8 * kNumBars + 4);
  float *xch = reinterpret_cast<float *>(smem + L::Xch);
  float *ubuf = reinterpret_cast<float *>(smem + L::Ubuf);
  float *invd_s = reinterpret_cast<float *>(smem + L::InvD);
  float *c_s = reinterpret_cast<float *>(smem + L::Cc);
  uint8_t *snap = smem + L::Snap;
  uint8_t *rqsnap = smem + L::RqSnap;
  uint8_t *slots = smem + L::Slots;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int quarter = warp & 3, half = warp >> 2;
  const int r = quarter * 32 + lane;
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  const int g = blockIdx.x % G, bh = blockIdx.x / G;
  const int t0 = g * seg_len, t1 = min(T, t0 + seg_len);
  const int nchunks = (t1 - t0 + kC - 1) / kC;
  // the pass walks its chunks backwards
  auto chunk_of = [&](int i) { return nchunks - 1 - i; };

  if (threadIdx.x == 0) {
    mbar_init(&bars[kBarLoadQ], 1);
    mbar_init(&bars[kBarLoadKV], 1);
    mbar_init(&bars[kBarMma], 2);                 // one commit per issuing thread
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  auto load_q = [&](int i) {        // Q and dout of the i-th chunk in walk order
    const int row = t0 + chunk_of(i) * kC;
    mbar_arrive_expect_tx(&bars[kBarLoadQ], 8192 + 16384);
    tma_load_3d(smem + L::Q, &tmq, &bars[kBarLoadQ], 0, row, bh);
    tma_load_3d(smem + L::dO, &tmo, &bars[kBarLoadQ], 0, row, bh);
  };
  auto load_kv = [&](int i) {
    const int row = t0 + chunk_of(i) * kC;
    mbar_arrive_expect_tx(&bars[kBarLoadKV], 8192 + 16384);
    tma_load_3d(smem + L::K, &tmk, &bars[kBarLoadKV], 0, row, bh);
    tma_load_3d(smem + L::V, &tmv, &bars[kBarLoadKV], 0, row, bh);
  };
  if (threadIdx.x == 0 && nchunks > 0) {
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmo);
    load_q(0);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    load_kv(0);
  }

  uint32_t mph = 0;
  // round_with also runs CUDA-core work while the MMAs are in flight: work
  // that neither reads nor writes what they touch.
  auto round_with = [&](auto issue, auto work) -> bool {
    tmem_wait_ld();
    tmem_wait_st();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 || threadIdx.x == 32) {
      tc_fence_after();
      issue(threadIdx.x >> 5);
      mma_commit(&bars[kBarMma]);
    }
    work();
    const bool ok = mbar_wait(&bars[kBarMma], mph, abort_flag);
    mph ^= 1;
    tc_fence_after();
    return __syncthreads_and(ok);
  };
  auto round = [&](auto issue) -> bool { return round_with(issue, [] {}); };
  auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
    return __syncthreads_and(mbar_wait(bar, parity, abort_flag));
  };

  auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
  const uint64_t d_q = smem_desc(smem_u32(smem + L::Q), 16, 512, kSw64);          // K-major
  const uint64_t d_q_mn = smem_desc(smem_u32(smem + L::Q), 8192, 512, kSw64);     // MN-major
  const uint64_t d_k = smem_desc(smem_u32(smem + L::K), 16, 512, kSw64);          // K-major
  const uint64_t d_v = smem_desc(smem_u32(smem + L::V), 16, 1024, kSw128);        // K-major
  const uint64_t d_o = smem_desc(smem_u32(smem + L::dO), 16, 1024, kSw128);       // K-major
  const uint64_t d_o_mn = smem_desc(smem_u32(smem + L::dO), 16384, 1024, kSw128); // MN-major
  const uint64_t d_snap = smem_desc(smem_u32(snap), 16, 1024, kSw128);            // K-major
  const uint64_t d_snap_mn = smem_desc(smem_u32(snap), 16384, 1024, kSw128);      // MN-major
  const uint64_t d_rq = smem_desc(smem_u32(rqsnap), 16, 512, kSw64);
  const uint64_t d_slot = smem_desc(smem_u32(slots), 16, 1024, kSw128);           // K-major
  const uint64_t d_tile = smem_desc(smem_u32(slots), 16384, 1024, kSw128);        // MN-major
  const uint64_t d_cq = smem_desc(smem_u32(smem + L::CQ), 8192, 512, kSw64);      // MN-major
  constexpr uint32_t id_n64 = idesc_bf16(128, 64, false, false);
  constexpr uint32_t id_n32 = idesc_bf16(128, 32, false, false);
  constexpr uint32_t id_n16 = idesc_bf16(128, 16, false, false);
  constexpr uint32_t id_ro = idesc_bf16(128, 64, false, true);     // slot x R' rows (MN-major)
  constexpr uint32_t id_wo = idesc_bf16(128, 64, false, true);     // W~ (TMEM) x dout rows
  constexpr uint32_t id_mq = idesc_bf16(128, 32, false, true);     // M (TMEM) x Q rows
  constexpr uint32_t id_up = idesc_bf16(128, 64, true, true);
  constexpr uint32_t id_rq = idesc_bf16(128, 32, true, true);

  // ---- carry-in: R', Rq = the increments of segments g+1 .. G-1 ----
  {
    const float *seg0 = aggR + (size_t)bh * G * kAggFloats;
    for (int m = half ? 2 : 0; m < (half ? 4 : 3); ++m) {
      const int mt = (!half && m == 2) ? 4 : m;
      const int f = 128 * mt + r;
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        float acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = 0.f;
        if (f < kD) {
          for (int gp = g + 1; gp < G; ++gp) {
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
        tmem_st16(tbase + lane_off + kColR + 64 * mt + 16 * q4, bits);
        if (f < kD) {
          *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4)) = pack8(bits);
          *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4 + 1)) = pack8(bits + 8);
        }
      }
    }
    if (half) {
      float acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = 0.f;
      if (r < kDK) {
        for (int gp = g + 1; gp < G; ++gp) {
          const float4 *src =
              reinterpret_cast<const float4 *>(seg0 + (size_t)gp * kAggFloats + kD * kDV + r * kDK);
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
      tmem_st32(tbase + lane_off + kColRq, bits);
      if (quarter == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(rqsnap + sw64(r, c)) = pack8(bits + 8 * c);
      }
    }
  }

  // d_t and c_t of a chunk (threads 0..127, one token each), loaded a chunk
  // ahead so that the load's latency hides behind the chunk's work
  float pf_den = 1.f, pf_c = 0.f;
  auto fetch_dc = [&](int i) {
    const int t = t0 + chunk_of(i) * kC + (int)threadIdx.x;
    if (threadIdx.x < kC && t < T) {
      pf_den = den[(size_t)bh * T + t];
      pf_c = cvec[(size_t)bh * T + t];
    } else {
      pf_den = 0.f;
      pf_c = 0.f;
    }
  };
  if (nchunks > 0) fetch_dc(0);

  bool ok = true;
  for (int i = 0; ok && i < nchunks; ++i) {
    const int c0 = t0 + chunk_of(i) * kC;
    const bool valid = c0 + r < T;
    // dk = the intra part + the carried part from ubuf (half 0); dv (half 1)
    auto write_outputs = [&] {
      {
        if (!half) {
          uint32_t acc[32];
          tmem_ld32(tbase + lane_off + kColDk, acc);
          tmem_wait_ld();
          const float *u = ubuf + r * 32;
          if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(dk + ((size_t)bh * T + c0 + r) * kDK);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t w[4];
#pragma unroll
              for (int j2 = 0; j2 < 4; ++j2) {
                const int l0 = 8 * c + 2 * j2;
                w[j2] = pack_bf16x2(__uint_as_float(acc[l0]) + u[l0],
                                    __uint_as_float(acc[l0 + 1]) + u[l0 + 1]);
              }
              dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        } else {
          uint32_t acc[32];
#pragma unroll 1
          for (int hv = 0; hv < 2; ++hv) {
            tmem_ld32(tbase + lane_off + kColDv + 32 * hv, acc);
            tmem_wait_ld();
            if (valid) {
              uint4 *dst = reinterpret_cast<uint4 *>(dv + ((size_t)bh * T + c0 + r) * kDV + 32 * hv);
#pragma unroll
              for (int c = 0; c < 4; ++c) dst[c] = pack8(acc + 8 * c);
            }
          }
        }
      }
    };
    if (!(ok = wait_all(&bars[kBarLoadQ], i & 1))) break;
    if (threadIdx.x < kC) {
      invd_s[threadIdx.x] = pf_den != 0.f ? 1.f / pf_den : 0.f;
      c_s[threadIdx.x] = pf_c;
    }
    if (i + 1 < nchunks) fetch_dc(i + 1);
    __syncthreads();
    {
      if (!(ok = wait_all(&bars[kBarLoadKV], i & 1))) break;
      float kf[32];
      row_f32(smem + L::K, r, kf);

      // ---- dk carried: Y = V R'^T (J(k)^T contraction), U2 = K Rq ----
      float h[32], g2R[32], kR[32];
#pragma unroll
      for (int l = 0; l < 32; ++l) {
        h[l] = 0.f;
        g2R[l] = 0.f;
        kR[l] = kf[l];
      }
      if (half) rot<8>(kR);
      float unused = 0.f;
      // four rounds; the last also takes the 16 features of tile 4 (half
      // 1's) into the dk columns, free between the read of U2 and the first
      // dk MMA
      for (int j = 0; ok && j < 4; ++j) {
        ok = round([&](int who) {
          if (j == 0 && who == 0) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_ss(tbase + kColDk, adv(d_k, 32 * kk), adv(d_rq, 32 * kk), id_n32, kk);
          }
          if (who == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tbase + kColDv, adv(d_v, 32 * kk), adv(d_snap, 64 * j * 128 + 32 * kk), id_n64,
                     kk);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tbase + kColW, adv(d_v, 32 * kk), adv(d_snap, (256 + 64 * j) * 128 + 32 * kk),
                     id_n64, kk);
            if (j == 3) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(tbase + kColDk, adv(d_v, 32 * kk), adv(d_snap, 512 * 128 + 32 * kk), id_n16, kk);
            }
          }
        });
        if (!ok) break;
        if (j == 0 && half == 0) {
          uint32_t u[32];
          tmem_ld32(tbase + lane_off + kColDk, u);
          tmem_wait_ld();
#pragma unroll
          for (int l = 0; l < 32; l += 4)
            *reinterpret_cast<float4 *>(ubuf + r * 32 + l) =
                make_float4(__uint_as_float(u[l]), __uint_as_float(u[l + 1]),
                            __uint_as_float(u[l + 2]), __uint_as_float(u[l + 3]));
        }
        {
          uint32_t x[32];
          const uint32_t col = half ? kColW : kColDv;
          tmem_ld32(tbase + lane_off + col, x);
          tmem_wait_ld();
          contract_offset<32, false>(x, kf, kR, h, g2R, unused);
          tmem_ld32(tbase + lane_off + col + 32, x);
          tmem_wait_ld();
          contract_offset<32, false>(x, kf, kR, h, g2R, unused);
        }
        if (j == 3 && half) {
          uint32_t x16[16];
          tmem_ld16(tbase + lane_off + kColDk, x16);
          tmem_wait_ld();
          contract_offset<16, false>(x16, kf, kR, h, g2R, unused);
        }
      }
      if (!ok) break;
      if (half) {
        rot<15>(g2R);
      } else {
        rot<24>(g2R);
      }
#pragma unroll
      for (int l = 0; l < 32; ++l) h[l] += g2R[l];
      if (half) {
        float *row = xch + r * 36;
#pragma unroll
        for (int l = 0; l < 32; l += 4)
          *reinterpret_cast<float4 *>(row + l) = make_float4(h[l], h[l + 1], h[l + 2], h[l + 3]);
      }

      // ---- dv carried (key products x R' rows, 64 features a slot, half 0
      //      slots 0..3, half 1 slots 4..8, one pair a round) interleaved with
      //      the intra-chunk quarters of 32 queries t >= s ----
      {
        uint32_t XK[16], P[32], R[32];
        load_pairs(smem + L::K, r, XK, P);
#pragma unroll
        for (int l = 0; l < 32; ++l) R[l] = P[l];
        if (half) rotate_left(R, 8);
        // slot pair j: half 0 writes slot j (j < 4), half 1 slot 4 + j
        auto write_slot = [&](int j) {
          if (half || j < 4) {
            const int s9 = half ? 4 + j : j;
            uint32_t w[32];
            q_slot_words(P, R, s9 == kQSlotsPsd - 1, w);
            uint8_t *slot = slots + 16384 * half;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              *reinterpret_cast<uint4 *>(slot + sw128(r, cc)) =
                  make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
            rotate_left(R, 2);
          }
        };
        auto issue_slots = [&](int j) {
          const int sa = j, sb = 4 + j;
          const int nk_b = sb == kQSlotsPsd - 1 ? 1 : 4;
          if (j < 4) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tbase + kColDv, adv(d_slot, 32 * kk), adv(d_snap_mn, (64 * sa + 16 * kk) * 128),
                     id_ro, (j > 0 || kk > 0) ? 1u : 0u);
          }
          for (int kk = 0; kk < nk_b; ++kk)
            mma_ss(tbase + kColDv, adv(d_slot, 16384 + 32 * kk),
                   adv(d_snap_mn, (64 * sb + 16 * kk) * 128), id_ro, 1u);
        };
        write_slot(0);
        const uint32_t ws_col = kColW + 8 * half;           // this half's W~ words
        const uint32_t ms_col = kColW + 16 + 8 * half;      // this half's M words
        for (int qt = 0; ok && qt < 4; ++qt) {
          // the first round also folds the carried dk into ubuf: J(k)^T Y of
          // both halves (half 1's from xch) plus 2 Rq k
          ok = round_with([&](int who) {
            if (who == 0) {
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_ss(tbase + kColW, adv(d_k, 32 * kk), adv(d_q, 2048 * qt + 32 * kk), id_n32, kk);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(tbase + kColW + 32, adv(d_v, 32 * kk), adv(d_o, 4096 * qt + 32 * kk), id_n32, kk);
            } else {
              issue_slots(qt);                     // the dv accumulator
            }
          }, [&] {
            if (qt == 0 && !half) {
              const float *row = xch + r * 36;
              float *u = ubuf + r * 32;
#pragma unroll
              for (int l = 0; l < 32; ++l) u[l] = h[l] + row[l] + 2.f * u[l];
            }
          });
          if (!ok) break;
          uint32_t a[16], dp[16], wv[8], mv[8];
          tmem_ld16(tbase + lane_off + kColW + 16 * half, a);
          tmem_ld16(tbase + lane_off + kColW + 32 + 16 * half, dp);
          tmem_wait_ld();
          const int tb = 32 * qt + 16 * half;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float wq[2], mq[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int t = tb + 2 * j + e;
              const float av = __uint_as_float(a[2 * j + e]);
              const float it = invd_s[t], ct = c_s[t];
              const bool keep = t >= r;
              wq[e] = keep ? av * av * it : 0.f;
              mq[e] = keep ? 2.f * av * fmaf(__uint_as_float(dp[2 * j + e]), it, ct) : 0.f;
            }
            wv[j] = pack_bf16x2(wq[0], wq[1]);
            mv[j] = pack_bf16x2(mq[0], mq[1]);
          }
          __syncthreads();        // every thread has read its columns before W~, M overwrite them
          tmem_st8(tbase + lane_off + ws_col, wv);
          tmem_st8(tbase + lane_off + ms_col, mv);
          // the next slot pair is written while this round runs (the last
          // round read the previous pair); the last pair, read by the last
          // round, before it
          if (qt == 3) write_slot(4);
          ok = round_with([&](int who) {
            if (who == 0) {                        // the dv accumulator
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_ts(tbase + kColDv, tbase + kColW + 8 * kk, adv(d_o_mn, 4096 * qt + 2048 * kk),
                       id_wo, 1u);
              if (qt == 3) issue_slots(4);
            } else {                               // the dk accumulator
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_ts(tbase + kColDk, tbase + kColW + 16 + 8 * kk, adv(d_q_mn, 2048 * qt + 1024 * kk),
                       id_mq, (qt > 0 || kk > 0) ? 1u : 0u);
            }
          }, [&] {
            if (qt < 3) write_slot(qt + 1);
          });
        }
      }
      if (!ok) break;
      if (threadIdx.x == 0 && i + 1 < nchunks) load_kv(i + 1);    // K, V no longer read
    }
    if (i == nchunks - 1) {                    // the state before the segment is not needed
      write_outputs();
      break;
    }

    // ---- update: R' += (m p(q) / d)^T dout (tiles (0, 2), (1, 3), (4)), Rq += Q^T diag(c) Q ----
    {
      uint32_t XQ[16], P[32], R2[32];
      load_pairs(smem + L::Q, r, XQ, P);
      const float inv_r = invd_s[r], c_r = c_s[r];
      const uint32_t two_inv = pack_bf16x2(2.f * inv_r, 2.f * inv_r);
#pragma unroll
      for (int l = 0; l < 32; ++l) R2[l] = bmul2(P[l], two_inv);   // x 2 / d_t
      if (half) {
        rotate_left(R2, 8);
      } else {
        // c_t q_t as bf16, the Rq update's A operand
        const uint32_t cc2 = pack_bf16x2(c_r, c_r);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 x = *reinterpret_cast<const uint4 *>(smem + L::Q + sw64(r, c));
          *reinterpret_cast<uint4 *>(smem + L::CQ + sw64(r, c)) =
              make_uint4(bmul2(x.x, cc2), bmul2(x.y, cc2), bmul2(x.z, cc2), bmul2(x.w, cc2));
        }
      }
      for (int u = 0; ok && u < 3; ++u) {
        const int m = half ? (u < 2 ? 2 + u : -1) : (u < 2 ? u : 4);
        if (m >= 0)
          write_tile(slots + 32768 * half, r, m == kTiles - 1, m == 0 ? 0x3f003f00u : 0x3f803f80u,
                     P, R2);
        if (!half && u == 1) {
          rotate_left(R2, 12);
        } else {
          rotate_left(R2, 4);
        }
        auto issue_upd = [&](int who) {
          const int ma = u < 2 ? u : 4, mb = 2 + u;
          if (who == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tbase + kColR + 64 * ma, adv(d_tile, 2048 * kk), adv(d_o_mn, 2048 * kk), id_up, 1);
          }
          if (u < 2 && who == 1) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tbase + kColR + 64 * mb, adv(d_tile, 32768 + 2048 * kk), adv(d_o_mn, 2048 * kk),
                     id_up, 1);
          }
          if (u == 0 && who == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tbase + kColRq, adv(d_cq, 1024 * kk), adv(d_q_mn, 1024 * kk), id_rq, 1);
          }
        };
        // dk and dv leave while the first update round runs (it touches neither)
        ok = u == 0 ? round_with(issue_upd, write_outputs) : round(issue_upd);
      }
      if (!ok) break;
      if (threadIdx.x == 0 && i + 1 < nchunks) load_q(i + 1);     // Q, dout no longer read
    }
    // ---- snapshot R' (half 0: tiles 0, 1, 4; half 1: tiles 2, 3) and Rq ----
    {
    for (int m = half ? 2 : 0; m < (half ? 4 : 3); ++m) {
      const int mt = (!half && m == 2) ? 4 : m;
      if (mt == 4 && quarter != 0) continue;
      const int f = 128 * mt + r;
      uint32_t a[32], b2[32];
      tmem_ld32(tbase + lane_off + kColR + 64 * mt, a);
      tmem_ld32(tbase + lane_off + kColR + 64 * mt + 32, b2);
      tmem_wait_ld();
      if (f < kD) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          *reinterpret_cast<uint4 *>(snap + sw128(f, q4)) = pack8(a + 8 * q4);
          *reinterpret_cast<uint4 *>(snap + sw128(f, 4 + q4)) = pack8(b2 + 8 * q4);
        }
      }
    }
    if (half && quarter == 0) {
      uint32_t zr[32];
      tmem_ld32(tbase + lane_off + kColRq, zr);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(rqsnap + sw64(r, c)) = pack8(zr + 8 * c);
    }
    }
  }

  if (*abort_flag && threadIdx.x == 0) flag_status(status, kStatusDeviceTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

}  // namespace

cudaError_t tc_bwd_dq(const BackwardLaunch &a, float *aggS, int G, int seg_len) {
  CUtensorMap tq, tk, tv, to;
  if (!make_tma_3d_bf16(&tq, a.q, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tk, a.k, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tv, a.v, kDV, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&to, a.dout, kDV, a.T, a.BH, kC))
    return cudaErrorInvalidValue;
  cudaError_t e = psd_tc_increments(a.k, a.v, aggS, a.status, a.BH, a.T, G - 1, G, seg_len, a.stream);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           DqSmem::Bytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_bwd_dq", a.stream);
  bwd_dq_tc_kernel<<<(unsigned)(a.BH * G), kBThreads, DqSmem::Bytes, a.stream>>>(
      tq, tk, tv, to, aggS, static_cast<__nv_bfloat16 *>(a.dq), a.den, a.c, a.status, a.T, G,
      seg_len);
  return cudaGetLastError();
}


cudaError_t tc_bwd_dkdv(const BackwardLaunch &a, float *aggR, int G, int seg_len) {
  CUtensorMap tq, tk, tv, to;
  if (!make_tma_3d_bf16(&tq, a.q, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tk, a.k, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tv, a.v, kDV, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&to, a.dout, kDV, a.T, a.BH, kC))
    return cudaErrorInvalidValue;
  cudaError_t e;
  // the suffix increments of segments 1 .. G-1 run on the forward's
  // warp-specialised increment kernel (K := Q, V := dout, scaled by 1 / d_t,
  // K^T K weighted by c_t)
  if ((e = psd_tc_suffix_increments(a.q, a.dout, a.den, a.c, aggR, a.status, a.BH, a.T, G, seg_len,
                                    a.stream)) != cudaSuccess)
    return e;
  auto kern = bwd_dkdv_tc_kernel;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DkvSmem::Bytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_bwd_dkdv", a.stream);
  kern<<<(unsigned)(a.BH * G), kBThreads, DkvSmem::Bytes, a.stream>>>(
      tq, tk, tv, to, aggR, a.den, a.c, static_cast<__nv_bfloat16 *>(a.dk),
      static_cast<__nv_bfloat16 *>(a.dv), a.status, a.T, G, seg_len);
  return cudaGetLastError();
}

}  // namespace kata
