// Tensor-core (tcgen05 / TMEM / TMA) flash-style quadratic forward,
// bf16 inputs, fp32 accumulation, d_v = 64.
//
// One CTA per (b, h, 128-query block), key blocks 0 .. qb (causal):
//   S_j = Q K_j^T            tcgen05.mma, A = Q, B = K_j from shared memory (TMA)
//   P_j = S_j^2 (or 1 + S_j) masked to key <= query < T, l += rowsum(P_j)
//                            math warps: TMEM -> registers -> bf16 -> TMEM (in place)
//   O  += P_j V_j            tcgen05.mma, A = P_j from TMEM, B = V_j from shared memory
//   y   = O / l              after the last block
// No exponential and no running maximum: the weights are polynomial and
// nonnegative (the flash-attention-style operating point of the KATA
// explainer, section 2.3).
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM
// and issues MMAs (one elected lane), warps 2-5 are the math warps; math
// thread r owns TMEM lane r = query row r of the block.
// Each key block is processed as two 64-key halves with their own barriers:
// S of half 0 in TMEM columns [0, 64), of half 1 in [64, 128), each half's P
// packed as bf16 over its first 32 columns; O in [128, 192). The math warps
// square one half while the tensor pipe runs P V of the other half and Q K^T
// of the next block's same half. 256 columns are allocated, so two CTAs
// share an SM.
#include "common.cuh"
#include "launch.h"
#include "profile.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace kata {
namespace {

using namespace tc;

constexpr int kBlock = 128;       // queries per CTA, keys per block
constexpr int kHalf = 64;         // keys per half block (one S buffer)
constexpr int kDV = 64;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColO = 128;

template <int DK>
struct QuadLayout {
  // K, V ring depth. A block's loads are issued when the block kStages
  // earlier has been consumed; with two stages that left about half a block
  // of math to cover the load latency and the MMA warp waited on it every
  // block. Four stages fit beside a second CTA on the SM for d_k <= 32;
  // at d_k = 64 a third stage would not, so it keeps two CTAs and two stages.
  static constexpr int kStages = DK <= 32 ? 4 : 2;
  static constexpr int kRowBytes = DK * 2;
  static constexpr int kQKBytes = kBlock * kRowBytes;     // one Q or K tile
  static constexpr int kVBytes = kBlock * kDV * 2;        // one V tile (16 KB)
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQKBytes;
  static constexpr int kV = kK + kStages * kQKBytes;
  static constexpr int kBar = kV + kStages * kVBytes;
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_full
  static constexpr int kNumBars = 6 + 2 * kStages;
  static constexpr int kTmemSlot = kBar + 8 * kNumBars;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr uint32_t kSwizzle = DK == 16 ? kSw32 : DK == 32 ? kSw64 : kSw128;
  static_assert(kQKBytes % 1024 == 0, "tiles must keep 1024-byte alignment");
};

template <int DK, int FEAT>
__global__ void __launch_bounds__(kThreads, 2)
quadratic_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, __nv_bfloat16 *__restrict__ o, int T,
                    int nqb) {
  using L = QuadLayout<DK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
  uint64_t *q_full = bars;
  uint64_t *kv_full = bars + 1;
  uint64_t *kv_empty = bars + 1 + L::kStages;
  uint64_t *s_full = bars + 1 + 2 * L::kStages;     // [2]: one per 64-key half
  uint64_t *p_full = s_full + 2;                 // [2]
  uint64_t *o_full = s_full + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlot);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kAbort);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int qb = nqb - 1 - (int)blockIdx.x;      // longest rows first
  const int bh = blockIdx.y;
  const int nkb = qb + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&s_full[h], 1);
      mbar_init(&p_full[h], 128);
    }
    mbar_init(o_full, 1);
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
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      mbar_arrive_expect_tx(q_full, L::kQKBytes);
      tma_load_3d(smem + L::kQ, &tmq, q_full, 0, qb * kBlock, bh);
      for (int j = 0; j < nkb; ++j) {
        const int s = j % L::kStages;
        if (j >= L::kStages && !mbar_wait(&kv_empty[s], ((j / L::kStages) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&kv_full[s], L::kQKBytes + L::kVBytes);
        tma_load_3d(smem + L::kK + s * L::kQKBytes, &tmk, &kv_full[s], 0, j * kBlock, bh);
        tma_load_3d(smem + L::kV + s * L::kVBytes, &tmv, &kv_full[s], 0, j * kBlock, bh);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // Each 128-key block is handled as two 64-key halves with their own
    // barriers, so that the math warps square one half while the tensor pipe
    // runs P V of the other and Q K^T of the next block's same half (issued
    // after that P V, which has then read the half's P: the pipe runs MMAs
    // in order).
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(kBlock, kHalf, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(kBlock, kDV, false, true);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      auto issue_qk = [&](int j, int h) {
        const uint32_t k_addr = smem_u32(smem + L::kK + (j % L::kStages) * L::kQKBytes) +
                                (uint32_t)(h * kHalf * L::kRowBytes);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
          mma_ss(tbase + kColS + kHalf * h, smem_desc(q_addr + kk * 32, 16, 8 * L::kRowBytes, L::kSwizzle),
                 smem_desc(k_addr + kk * 32, 16, 8 * L::kRowBytes, L::kSwizzle), idesc_qk,
                 kk > 0 ? 1u : 0u);
        mma_commit(&s_full[h]);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag) && mbar_wait(&kv_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(0, 1);
      }
      for (int j = 0; ok && j < nkb; ++j) {
        const int s = j % L::kStages;
        const uint32_t v_addr = smem_u32(smem + L::kV + s * L::kVBytes);
        for (int h = 0; ok && h < 2; ++h) {
          if (!(ok = mbar_wait(&p_full[h], j & 1, abort_flag))) break;
          tc_fence_after();
          // O += P_h V_h (P_h: 64 keys as 32 packed columns of tensor memory)
#pragma unroll
          for (int kk = 0; kk < kHalf / 16; ++kk)
            mma_ts(tbase + kColO, tbase + kColS + kHalf * h + 8 * kk,
                   smem_desc(v_addr + (4 * h + kk) * 2048, 16384, 1024, kSw128), idesc_pv,
                   (j > 0 || h > 0 || kk > 0) ? 1u : 0u);
          if (h == 1) mma_commit(&kv_empty[s]);        // K_j, V_j no longer read
          if (j + 1 < nkb) {
            if (h == 0) {
              if (!(ok = mbar_wait(&kv_full[(j + 1) % L::kStages], ((j + 1) / L::kStages) & 1, abort_flag)))
                break;
              tc_fence_after();
            }
            issue_qk(j + 1, h);
          }
        }
      }
      mma_commit(o_full);
    }
  } else {
    // ---------------- math warps ----------------
    const int quarter = warp % 4;
    const int row = quarter * 32 + lane;
    const int t = qb * kBlock + row;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    // row sum of the weights in four packed partial sums (no long add chain)
    float2 lsum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
    bool ok = true;
    for (int j = 0; ok && j < nkb; ++j) {
      // key blocks below the diagonal block lie entirely before every query
      // of this block (and before T): no mask there
      const bool diag = j == nkb - 1;
      for (int h = 0; h < 2; ++h) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[h], j & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int key0 = j * kBlock + kHalf * h;
#pragma unroll 1
        for (int c = 0; c < kHalf / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tbase + lane_off + kColS + kHalf * h + 32 * c, r);
          tmem_wait_ld();
          uint32_t p[16];
          if (!diag) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 x = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
              const float2 w = FEAT == kPSD ? __fmul2_rn(x, x) : __fadd2_rn(make_float2(1.f, 1.f), x);
              lsum[i & 3] = __fadd2_rn(lsum[i & 3], w);
              p[i] = pack_bf16x2(w.x, w.y);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int k0 = key0 + 32 * c + 2 * i;
              const float2 x = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
              float2 w = FEAT == kPSD ? __fmul2_rn(x, x) : __fadd2_rn(make_float2(1.f, 1.f), x);
              if (k0 > t || k0 >= T) w.x = 0.f;
              if (k0 + 1 > t || k0 + 1 >= T) w.y = 0.f;
              lsum[i & 3] = __fadd2_rn(lsum[i & 3], w);
              p[i] = pack_bf16x2(w.x, w.y);
            }
          }
          tmem_st16(tbase + lane_off + kColS + kHalf * h + 16 * c, p);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[h]);
      }
    }
    const float2 l01 = __fadd2_rn(lsum[0], lsum[1]), l23 = __fadd2_rn(lsum[2], lsum[3]);
    const float l = (l01.x + l01.y) + (l23.x + l23.y);
    // warp-uniform: the TMEM loads below are warp-collective
    const bool have_o = __all_sync(0xffffffffu, ok && mbar_wait(o_full, 0, abort_flag));
    if (have_o) tc_fence_after();
    uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)bh * T + t) * kDV);
#pragma unroll
    for (int h = 0; h < kDV / 32; ++h) {
      uint32_t r[32];
      if (have_o) {
        tmem_ld32(tbase + lane_off + kColO + 32 * h, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0x7fc00000u;   // NaN rows after a device timeout
      }
      const float inv = have_o ? 1.f / l : 1.f;
      if (t < T) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * q4 + 0]) * inv, __uint_as_float(r[8 * q4 + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(r[8 * q4 + 2]) * inv, __uint_as_float(r[8 * q4 + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(r[8 * q4 + 4]) * inv, __uint_as_float(r[8 * q4 + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(r[8 * q4 + 6]) * inv, __uint_as_float(r[8 * q4 + 7]) * inv);
          dst[4 * h + q4] = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

template <int DK, int FEAT>
cudaError_t launch(const QuadraticLaunch &a) {
  using L = QuadLayout<DK>;
  CUtensorMap tq, tk, tv;
  if (!make_tma_3d_bf16(&tq, a.q, DK, a.T, a.BH, kBlock) ||
      !make_tma_3d_bf16(&tk, a.k, DK, a.T, a.BH, kBlock) ||
      !make_tma_3d_bf16(&tv, a.v, kDV, a.T, a.BH, kBlock))
    return cudaErrorInvalidValue;              // accepted shape: a failure, not a fallback
  // 1 KB alignment slack; at least 100 KB so that at most two CTAs (two
  // 256-column TMEM allocations) share an SM.
  const int smem = L::kBytes + 1024 < 100 * 1024 ? 100 * 1024 : L::kBytes + 1024;
  auto kern = quadratic_tc_kernel<DK, FEAT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int nqb = (a.T + kBlock - 1) / kBlock;
  ProfileScope prof("tc_quadratic", a.stream);
  kern<<<dim3(nqb, (unsigned)a.BH), kThreads, smem, a.stream>>>(
      tq, tk, tv, static_cast<__nv_bfloat16 *>(a.o), a.T, nqb);
  return cudaGetLastError();
}

}  // namespace

// Tensor-core quadratic forward for bf16, d_v = 64, d_k in {16, 32, 64}.
// Returns cudaErrorNotSupported, having launched nothing, when the shape or
// alignment is not handled here (the caller then uses the CUDA-core kernel);
// for a shape it accepts it either launches or returns an error.
cudaError_t tc_quadratic(const QuadraticLaunch &a, int d_k, int d_v, int feature) {
  if (d_v != kDV || a.BH > 65535 || a.T <= 0) return cudaErrorNotSupported;
  for (const void *p : {a.q, a.k, a.v, (const void *)a.o})
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return cudaErrorNotSupported;
  if (feature == kPSD) {
    if (d_k == 16) return launch<16, kPSD>(a);
    if (d_k == 32) return launch<32, kPSD>(a);
  } else if (feature == kFirstOrder) {
    if (d_k == 16) return launch<16, kFirstOrder>(a);
    if (d_k == 32) return launch<32, kFirstOrder>(a);
    if (d_k == 64) return launch<64, kFirstOrder>(a);
  }
  return cudaErrorNotSupported;                  // other features: the CUDA-core kernel
}

}  // namespace kata
