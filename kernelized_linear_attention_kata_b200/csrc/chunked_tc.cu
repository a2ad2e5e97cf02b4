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
// Warp roles (384 threads): warp 0 TMA producer; warp 1 TMEM allocation and
// the query-side MMAs (Q K^T, P V, U, the even readout slots into O); warp 11
// the odd readout slots; warp 10 the state-side MMAs (the update of S and Z).
// Each test of a barrier by an issuing thread stalls its MMA stream, so
// three issuing threads share the work and cover one another's waits; warps 2-5, the query side: the
// intra-chunk P, the query features into tensor memory, the epilogue (y
// staged in shared memory, written by one TMA store per chunk); warps 6-9,
// the key side: the key features into the shared-memory ring, the bf16
// snapshot of the state after each update, the carry-in and the state
// written out. Math thread r owns TMEM lane r (quarter = warp mod 4):
// token r of the chunk for the token-major tiles, feature row r of each
// 128-feature state tile.
// The increment kernel (AGG) has no query side: warps 2-5 write the key
// features of tiles 1 and 3 and warps 6-9 those of tiles 0, 2 and 4, and
// the two update issuers (warp 1: Z and tiles 1, 3; warp 10: tiles 0, 2, 4)
// each consume one set, so that both sets and both issuers work at once.
//
// Tensor memory (512 columns, fp32):
//   [  0, 320)  S, five 128-feature tiles of 64 columns (tile 4: 16 rows used)
//   [320, 352)  Z (lanes 0..31)
//   [352, 384)  U = Q_c Z_c (den of the inter-chunk part: q^T Z_c q = q . u);
//               once read, query-feature slot 0 (64 bf16 features per token)
//   [384, 512)  Q_c K_c^T; then P (bf16, in place, [384, 448)) and O ([448, 512));
//               once P V is done, [384, 416) and [416, 448) are query slots 1, 2
// The readout takes its A operand (the query features) from tensor memory,
// so the only shared-memory operands of the hot loop are the key features
// and the state snapshot.
// Shared memory (206 KB): the Q tile (single buffer), two TMA stages of K and
// V, the bf16 snapshots of S_c (the readout's B operand) and Z_c, the output
// stage and a ring of two 128-feature key slots (the update's A operand).
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

constexpr int kThreads = 384;      // 12 warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColZ = 320, kColX = 384, kColO = 448;
constexpr uint32_t kColU = 352;    // U = Q Z_c, then query ring entry 3
// Query ring: entry 0 is a shared-memory slot (SS readout MMAs), entries 1
// and 2 are P's columns once P V is done, entry 3 is U's columns once U is
// read. Readout slot s9 goes to entry s9 mod 4 (entry 0 takes three slots of
// a chunk, the others two), so warp 1 (even slots) consumes entries 0 and 2
// and warp 11 (odd slots) entries 1 and 3.
constexpr int kRing = 4;
__host__ __device__ constexpr int ring_entry(int s9) { return s9 % kRing; }
__host__ __device__ constexpr int ring_uses(int e) { return e == 0 ? 3 : 2; }
__host__ __device__ constexpr uint32_t ring_col(int e) { return e == 3 ? kColU : kColU + 32u * e; }

// Shared memory layout (bytes from a 1024-aligned base). Key features travel
// through a ring with one producer set and one consumer warp (an mbarrier
// parity wait is only unambiguous for a single consumer in order): 32 KB
// slots of 128 token rows x 128 key features, as two 64-feature groups 16 KB
// apart (update A operand, MN-major), five uses per chunk, one per state tile.
//   forward pass:  Q 8 KB | K 2 x 8 KB | V 2 x 16 KB | S_c bf16 66 KB |
//                  Z_c bf16 2 KB | y stage 16 KB | query slot 16 KB | key ring 2 x 32 KB
//   increments:    K 2 x 8 KB | V 2 x 16 KB | key ring 5 x 32 KB
// The query features (readout A operand, 64 features a slot, nine slots a
// chunk) travel through a ring of one shared-memory slot (128 token rows x
// 64 features, K-major) and three tensor-memory slots.
constexpr int kKSlotBytes = 32768;
constexpr int kQSlots = 9;          // 64-feature readout slots per chunk
template <bool AGG, bool SFX = false>
struct Layout {
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = AGG ? 0 : 8192;
  static constexpr int kOffCQ = kOffK + 16384;        // suffix increments: c_t q_t, two stages
  static constexpr int kOffV = kOffCQ + (SFX ? 16384 : 0);
  static constexpr int kOffSnap = kOffV + 32768;      // [528][64] bf16, 128 B rows (pass only)
  static constexpr int kOffZSnap = kOffSnap + (AGG ? 0 : kD * 128);   // [32][32] bf16, 64 B rows
  static constexpr int kOffStage = kOffZSnap + (AGG ? 0 : 2048);      // y: [128][64] bf16, 128 B rows
  static constexpr int kOffQSlot = kOffStage + (AGG ? 0 : 16384);    // query slot (ring entry 0)
  static constexpr int kOffKRing = kOffQSlot + (AGG ? 0 : 16384);
  static constexpr int kKRingSlots = AGG ? 5 : 2;
  static constexpr int kOffBars = kOffKRing + kKRingSlots * kKSlotBytes;
  static constexpr int kSmemBytes = kOffBars + 1024 + 1024;   // barriers + alignment slack
  static_assert(kOffV % 1024 == 0 && kOffSnap % 1024 == 0 && kOffZSnap % 1024 == 0 &&
                    kOffStage % 1024 == 0 && kOffQSlot % 1024 == 0 && kOffKRing % 1024 == 0,
                "swizzle atoms need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};
enum {
  kBarQFull = 0, kBarQEmpty, kBarKvFull, kBarKvEmpty = kBarKvFull + 2, kBarSFull = kBarKvEmpty + 2,
  kBarPFull, kBarPVDone, kBarUDone, kBarOFull, kBarXFree, kBarUpdFull, kBarZDone, kBarZSnap,
  kBarStageFull, kBarStageFree, kBarTileDone,
  kBarTileSnap = kBarTileDone + 5, kBarRingFull = kBarTileSnap + 5, kBarRingEmpty = kBarRingFull + kRing,
  kBarKRingFull = kBarRingEmpty + kRing, kBarKRingEmpty = kBarKRingFull + 5, kNumBars = kBarKRingEmpty + 5
};
constexpr int kBarBytes = 8 * kNumBars;
static_assert(kBarBytes + 8 <= 1024, "barrier area");

// 2 / d_t of token t as a bf16 pair (0 past T or for d_t = 0): the suffix
// increments' scale of the query features.
__device__ __forceinline__ uint32_t suffix_scale(const float *den, int bh, int T, int t) {
  const float d = t < T ? den[(size_t)bh * T + t] : 0.f;
  const float s = d != 0.f ? 2.f / d : 0.f;
  return tc::pack_bf16x2(s, s);
}

// SFX (with AGG): the backward's suffix increments of segments g_off ..
// g_off + G_grid - 1, with K := Q, V := dout, the key features scaled by
// 2 / d_t instead of 2 and K^T K weighted by c_t: R' = sum m_f phi(q_t)
// dout_t^T / d_t, Rq = Q^T diag(c) Q (tok_den, tok_c: [BH][T]).
template <bool AGG, bool SFX = false>
__global__ void __launch_bounds__(kThreads, 1)
chunked_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                  float *__restrict__ agg, const float *__restrict__ S0, const float *__restrict__ z0,
                  float *__restrict__ S_out, float *__restrict__ z_out,
                  unsigned *__restrict__ status, int T, int G_grid, int G_total, int seg_len,
                  const float *__restrict__ tok_den, const float *__restrict__ tok_c, int g_off) {
  static_assert(AGG || !SFX, "the suffix form is an increment kernel");
  using L = Layout<AGG, SFX>;
  constexpr int NK = L::kKRingSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffBars + kBarBytes);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffBars + kBarBytes + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int g = blockIdx.x % G_grid + g_off;
  const int bh = blockIdx.x / G_grid;
  const int t0 = g * seg_len;
  const int t1 = min(T, t0 + seg_len);
  const int nchunks = (t1 - t0 + kC - 1) / kC;

  if (threadIdx.x == 0) {
    // arrival counts: 1 for a TMA transaction or an MMA commit,
    // kSetArrivals for the threads of a math set
    constexpr uint32_t A = kSetArrivals;
    mbar_init(&bars[kBarQFull], 1);
    mbar_init(&bars[kBarQEmpty], 1 + A);            // Q K^T commit + query side
    for (int st = 0; st < 2; ++st) {
      mbar_init(&bars[kBarKvFull + st], 1);
      // two MMA warps + key side (+ the second feature set of the increment kernel)
      mbar_init(&bars[kBarKvEmpty + st], AGG ? 2 + 2 * A : 2 + A);
    }
    mbar_init(&bars[kBarSFull], 1);
    mbar_init(&bars[kBarPFull], A);
    mbar_init(&bars[kBarPVDone], 1);
    mbar_init(&bars[kBarUDone], 1);
    mbar_init(&bars[kBarStageFull], A);
    mbar_init(&bars[kBarStageFree], 1);
    mbar_init(&bars[kBarOFull], 2);                 // both readout issuers
    mbar_init(&bars[kBarXFree], A);
    mbar_init(&bars[kBarUpdFull], AGG ? 2 : 1);
    // done-barriers of the snapshots: one commit from each issuing warp (the
    // readout / U that read the old snapshot, the update that wrote the new state)
    mbar_init(&bars[kBarZDone], 2);
    mbar_init(&bars[kBarZSnap], A);
    for (int m = 0; m < 5; ++m) {
      mbar_init(&bars[kBarTileDone + m], 3);       // both readout issuers + the update
      mbar_init(&bars[kBarTileSnap + m], A);
    }
    for (int k = 0; k < kRing; ++k) {
      mbar_init(&bars[kBarRingFull + k], A);
      mbar_init(&bars[kBarRingEmpty + k], 1);
    }
    for (int k = 0; k < NK; ++k) {
      mbar_init(&bars[kBarKRingFull + k], A);
      mbar_init(&bars[kBarKRingEmpty + k], 1);
    }
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
  uint8_t *kring = smem + L::kOffKRing;

  // Producer side of a ring (one math warp set): use u of a ring with n
  // slots may be written once its previous occupant (use u - n) is consumed.
  auto ring_acquire = [&](uint64_t *empty, int n, int u) -> bool {
    return u < n || warp_wait(&empty[u % n], ((u / n) - 1) & 1, abort_flag);
  };
  auto ring_publish = [&](uint64_t *full, int n, int u) {
    fence_async_smem();
    warp_arrive(&full[u % n]);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      if (!AGG) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmo);
      }
      for (int i = 0; i < nchunks; ++i) {
        const int st = i & 1;
        const int row = t0 + i * kC;
        if (!AGG) {
          if (i >= 1 && !mbar_wait(&bars[kBarQEmpty], (i - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(&bars[kBarQFull], 8192);
          tma_load_3d(smem + L::kOffQ, &tmq, &bars[kBarQFull], 0, row, bh);
        }
        if (i >= 2 && !mbar_wait(&bars[kBarKvEmpty + st], ((i >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&bars[kBarKvFull + st], 8192 + 16384);
        tma_load_3d(smem + L::kOffK + 8192 * st, &tmk, &bars[kBarKvFull + st], 0, row, bh);
        tma_load_3d(smem + L::kOffV + 16384 * st, &tmv, &bars[kBarKvFull + st], 0, row, bh);
      }
    }
  } else if (warp == 1 || warp == 10 || warp == 11) {
    // ------------------------------------------------------------ MMA issue
    // Two issuing warps with independent accumulators, so that one's waits
    // are covered by the other's MMAs: warp 1 issues the query side (Q K^T,
    // P V, the readout into O); warp 10 issues the state side (the update
    // of S and Z).
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t id_pv = idesc_bf16(128, kDV, false, true);
      constexpr uint32_t id_u = idesc_bf16(128, 32, false, false);
      constexpr uint32_t id_ro = idesc_bf16(128, kDV, false, true);
      constexpr uint32_t id_up = idesc_bf16(128, kDV, true, true);
      constexpr uint32_t id_z = idesc_bf16(128, 32, true, true);
      const uint32_t qa = smem_u32(smem + L::kOffQ);
      const uint32_t kring_a = smem_u32(kring);
      // Descriptors are built once; operands at other offsets of the same
      // layout differ only in the start-address field (bytes / 16).
      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
      const uint64_t d_q = smem_desc(qa, 16, 512, kSw64);                       // Q, K-major
      const uint64_t d_z = smem_desc(smem_u32(smem + L::kOffZSnap), 16, 512, kSw64);
      const uint64_t d_snap = smem_desc(smem_u32(smem + L::kOffSnap), 16384, 1024, kSw128);
      const uint64_t d_kring = smem_desc(kring_a, 16384, 1024, kSw128);         // update A
      const uint64_t d_k_k = smem_desc(smem_u32(smem + L::kOffK), 16, 512, kSw64);     // K, K-major
      const uint64_t d_k_mn = smem_desc(smem_u32(smem + L::kOffK), 8192, 512, kSw64);  // K, MN-major
      // c_t q_t (suffix increments), MN-major: the weighted K^T K's A operand
      const uint64_t d_cq_mn = smem_desc(smem_u32(smem + L::kOffCQ), 8192, 512, kSw64);
      const uint64_t d_v = smem_desc(smem_u32(smem + L::kOffV), 16384, 1024, kSw128);  // V, MN-major
      // Key-ring slots are shared memory written by threads (ordered for the
      // tensor core by their proxy fence and the mbarrier), so their waits
      // need no tcgen05 fence; hand-offs of tensor memory do.
      // Two barriers tested back to back so that their latencies overlap.
      auto wait2 = [&](uint64_t *b1, uint32_t p1, uint64_t *b2, uint32_t p2) -> bool {
        const bool a = mbar_test_wait(b1, p1), b = mbar_test_wait(b2, p2);
        if (a && b) return true;
        return (a || mbar_wait(b1, p1, abort_flag)) && (b || mbar_wait(b2, p2, abort_flag));
      };
      bool ok = true;
      // O += phi_q(Q) S_c over the readout slots s9 = first, first + 2, ...
      // (64 features each; slot s9 in ring entry ring_entry(s9), A from the
      // shared-memory slot or tensor memory, B = rows 64 s9 .. 64 s9 + 63 of
      // the snapshot). Each issuer releases snapshot tile s9 / 2 after its own
      // slot of that tile.
      const uint64_t d_qslot = smem_desc(smem_u32(smem + L::kOffQSlot), 16, 1024, kSw128);
      auto readout = [&](int i, int first) -> bool {
        for (int s9 = first; s9 < kQSlots; s9 += 2) {
          const int b = ring_entry(s9), k = ring_uses(b) * i + s9 / kRing;
          if (!mbar_wait(&bars[kBarRingFull + b], k & 1, abort_flag)) return false;
          tc_fence_after();
          const int nk = s9 == kQSlots - 1 ? 1 : 4;
          if (b == 0) {
            for (int kk = 0; kk < nk; ++kk)
              mma_ss(tbase + kColO, adv(d_qslot, 32 * kk), adv(d_snap, (64 * s9 + 16 * kk) * 128), id_ro, 1);
          } else {
            const uint32_t a_col = tbase + ring_col(b);
            for (int kk = 0; kk < nk; ++kk)
              mma_ts(tbase + kColO, a_col + 8 * kk, adv(d_snap, (64 * s9 + 16 * kk) * 128), id_ro, 1);
          }
          mma_commit(&bars[kBarRingEmpty + b]);
          mma_commit(&bars[kBarTileDone + (s9 >> 1)]);
        }
        if (first == 1) mma_commit(&bars[kBarTileDone + (kTiles - 1)]);   // tile 4 has no odd slot
        return true;
      };

      if (warp == 11 && !AGG) {
        // ---------------- odd readout slots; the output store ----------------
        const uint8_t *stage = smem + L::kOffStage;
        for (int i = 0; ok && i < nchunks; ++i) {
          if (!(ok = readout(i, 1))) break;
          mma_commit(&bars[kBarOFull]);
          // y of chunk i, staged by the query side, leaves by one TMA store
          if (!(ok = mbar_wait(&bars[kBarStageFull], i & 1, abort_flag))) break;
          tma_store_3d(&tmo, stage, 0, t0 + i * kC, bh);
          bulk_commit_group();
          bulk_wait_read_all();
          mbar_arrive(&bars[kBarStageFree]);
        }
        bulk_wait_all();                                 // stores complete before the CTA exits
      } else if (warp == 1 && !AGG) {
        // ---------------- query-side MMAs ----------------
        // Every test of a barrier by an issuing thread drains its MMAs from
        // the tensor pipe, so the issuing threads wait on as few barriers as
        // possible: the math warps wait on the others first and fold them
        // into their own arrivals (XFree implies Q_i+1 and K_i+1, V_i+1 in
        // shared memory; PFull implies the Z_c snapshot; a ring slot implies
        // the snapshot tile it is read against).
        auto issue_qk = [&](int i) -> bool {
          const int st = i & 1;
          if (i == 0) {
            if (!wait2(&bars[kBarKvFull + st], (i >> 1) & 1, &bars[kBarQFull], i & 1)) return false;
          } else if (!mbar_wait(&bars[kBarXFree], (i - 1) & 1, abort_flag)) {
            return false;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(tbase + kColX, adv(d_q, 32 * kk), adv(d_k_k, 8192 * st + 32 * kk), id_qk, kk);
          mma_commit(&bars[kBarSFull]);
          return true;
        };
        if (nchunks > 0) ok = issue_qk(0);
        for (int i = 0; ok && i < nchunks; ++i) {
          const int st = i & 1;
          if (!(ok = mbar_wait(&bars[kBarPFull], i & 1, abort_flag))) break;
          tc_fence_after();
          // O = P V (P from tensor memory)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tbase + kColO, tbase + kColX + 8 * kk, adv(d_v, 16384 * st + 2048 * kk), id_pv, kk);
          mma_commit(&bars[kBarPVDone]);                 // P's columns become query slots 1, 2
          // U = Q Z_c into query slot 0
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(tbase + kColU, adv(d_q, 32 * kk), adv(d_z, 32 * kk), id_u, kk);
          mma_commit(&bars[kBarUDone]);
          mma_commit(&bars[kBarQEmpty]);                 // Q tile no longer read by the tensor core
          mma_commit(&bars[kBarZDone]);                  // Z_c snapshot no longer read
          // O += phi_q(Q) S_c over the even readout slots (warp 11 issues
          // the odd ones)
          if (!(ok = readout(i, 0))) break;
          mma_commit(&bars[kBarOFull]);
          mma_commit(&bars[kBarKvEmpty + st]);          // this warp's reads of K_i, V_i are done
          if (i + 1 < nchunks && !(ok = issue_qk(i + 1))) break;
        }
      } else if (warp == 10 || (AGG && warp == 1)) {
        // ---------------- state-side MMAs ----------------
        // In the increment kernel (no readout) warps 10 and 1 split the
        // tiles (warp 10: tiles 0, 2, 4; warp 1: Z and tiles 1, 3), as the
        // two feature sets split their production.
        // The key side writes the key features of chunk i after its snapshots
        // of S_i and Z_i (and after K_i, V_i arrived), so a full key-ring slot
        // also says that the state it updates has been read.
        for (int i = 0; ok && i < nchunks; ++i) {
          const int st = i & 1;
          for (int m = 0; m < kTiles && ok; ++m) {
            if (AGG && (m & 1) != (warp == 1 ? 1 : 0)) continue;
            const int u = i * kTiles + m, b = u % NK;
            if (!(ok = mbar_wait(&bars[kBarKRingFull + b], (u / NK) & 1, abort_flag))) break;
            tc_fence_after();
            if (m == (AGG ? 1 : 0)) {
              // Z += K^T K (A rows 32..127 alias other shared memory; unused lanes)
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_ss(tbase + kColZ, adv(SFX ? d_cq_mn : d_k_mn, 8192 * st + 1024 * kk),
                       adv(d_k_mn, 8192 * st + 1024 * kk), id_z, 1);
              if (!AGG) mma_commit(&bars[kBarZDone]);
            }
            // S tile m += phi(K)^T V
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tbase + kColS + 64 * m, adv(d_kring, b * kKSlotBytes + 2048 * kk),
                     adv(d_v, 16384 * st + 2048 * kk), id_up, 1);
            mma_commit(&bars[kBarKRingEmpty + b]);
            if (!AGG) mma_commit(&bars[kBarTileDone + m]);
          }
          if (!ok) break;
          mma_commit(&bars[kBarKvEmpty + st]);
          if (i == nchunks - 1) mma_commit(&bars[kBarUpdFull]);
        }
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------ query side (warps 2..5)
    if (!AGG) {
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;                  // TMEM lane = token of the chunk
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      uint8_t *stage = smem + L::kOffStage;
      uint8_t *qslot = smem + L::kOffQSlot;
      for (int i = 0; i < nchunks; ++i) {
        const int c0 = t0 + i * kC;
        if (!warp_wait(&bars[kBarQFull], i & 1, abort_flag)) break;
        if (!warp_wait(&bars[kBarSFull], i & 1, abort_flag)) break;
        tc_fence_after();
        // ---- intra-chunk block: P = (Q K^T)^2 masked (key s <= min(r, T-1-c0)) ----
        // 32 keys at a time; P (bf16) overwrites the columns already read.
        // Per warp, a block of keys is entirely valid, entirely masked (no
        // load, zeros) or straddles the diagonal (masked per element).
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
            tmem_ld32(tbase + lane_off + kColX + 32 * c, x);
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
          tmem_st16(tbase + lane_off + kColX + 16 * c, p);
        }
        const float2 l01 = __fadd2_rn(lsum[0], lsum[1]), l23 = __fadd2_rn(lsum[2], lsum[3]);
        const float2 lt = __fadd2_rn(l01, l23);
        const float l_intra = lt.x + lt.y;
        tmem_wait_st();
        tc_fence_before();
        // PFull also hands over the Z_c snapshot (read by U after P V)
        if (!warp_wait(&bars[kBarZSnap], i & 1, abort_flag)) break;
        warp_arrive(&bars[kBarPFull]);

        // ---- phi_q(Q_c) into the tensor-memory ring, 64 features a slot ----
        uint32_t XQ[16], P[32];
        load_pairs(smem + L::kOffQ, r, XQ, P);
        warp_arrive(&bars[kBarQEmpty]);               // Q rows read
        bool ok = true;
        float den_inter = 0.f;
        uint32_t R[32];
#pragma unroll
        for (int l = 0; l < 32; ++l) R[l] = P[l];
        // Entry ring_entry(s9) may be written once its previous use has been
        // read. The first use of a chunk of a tensor-memory entry instead
        // waits for what last used the columns in this chunk (P V for entries
        // 1 and 2, U for entry 3), which also implies every use of the
        // previous chunk is complete; entry 3 first hands its U to the
        // denominator.
        auto wait_entry = [&](int s9) -> bool {
          const int b = ring_entry(s9), j = s9 / kRing, k = ring_uses(b) * i + j;
          if (j == 0 && b == 1) return warp_wait(&bars[kBarPVDone], i & 1, abort_flag);
          if (j == 0 && b == 2) return true;             // P V already waited for (entry 1 first)
          if (j == 0 && b == 3) {
            if (!warp_wait(&bars[kBarUDone], i & 1, abort_flag)) return false;
            tc_fence_after();
            uint32_t uu[32];
            tmem_ld32(tbase + lane_off + kColU, uu);
            tmem_wait_ld();
#pragma unroll
            for (int w = 0; w < 16; ++w) {
              const __nv_bfloat162 qq = *reinterpret_cast<const __nv_bfloat162 *>(&XQ[w]);
              den_inter = fmaf(__low2float(qq), __uint_as_float(uu[2 * w]), den_inter);
              den_inter = fmaf(__high2float(qq), __uint_as_float(uu[2 * w + 1]), den_inter);
            }
            return true;
          }
          return k == 0 || warp_wait(&bars[kBarRingEmpty + b], (k - 1) & 1, abort_flag);
        };
        // Query features of slot s9 (R rotated to its offsets) into its entry.
        auto produce = [&](int s9) {
          const int b = ring_entry(s9);
          tc_fence_after();
          uint32_t w[32];
          q_slot_words(P, R, s9 == kQSlots - 1, w);
          if (b == 0) {
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              *reinterpret_cast<uint4 *>(qslot + sw128(r, cc)) =
                  make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
            fence_async_smem();
          } else {
            tmem_st32(tbase + lane_off + ring_col(b), w);
            tmem_wait_st();
            tc_fence_before();
          }
          warp_arrive(&bars[kBarRingFull + b]);
        };
        // Slots go in pairs (2 p, 2 p + 1): one for each readout issuer, both
        // read against snapshot tile p. The pair's waits come first, so the
        // two issuers receive their slots together.
#pragma unroll 1
        for (int s9 = 0; s9 < kQSlots; s9 += 2) {
          const bool pair = s9 + 1 < kQSlots;
          if (ok) ok = wait_entry(s9);
          if (ok && pair) ok = wait_entry(s9 + 1);
          if (ok) ok = warp_wait(&bars[kBarTileSnap + (s9 >> 1)], i & 1, abort_flag);
          if (ok) produce(s9);
          rotate_left(R, 2);
          if (ok && pair) produce(s9 + 1);
          if (pair) rotate_left(R, 2);
        }
        if (!ok) break;

        // ---- epilogue: y = O / (l_intra + q^T Z_c q) ----
        if (!warp_wait(&bars[kBarOFull], i & 1, abort_flag)) break;
        tc_fence_after();
        uint32_t oo[32], oo2[32];
        tmem_ld32(tbase + lane_off + kColO, oo);
        tmem_ld32(tbase + lane_off + kColO + 32, oo2);
        tmem_wait_ld();
        tc_fence_before();
        // XFree also hands over Q_c+1 and K_c+1, V_c+1 (read by its Q K^T)
        if (i + 1 < nchunks &&
            !(warp_wait(&bars[kBarQFull], (i + 1) & 1, abort_flag) &&
              warp_wait(&bars[kBarKvFull + ((i + 1) & 1)], ((i + 1) >> 1) & 1, abort_flag)))
          break;
        warp_arrive(&bars[kBarXFree]);
        const float den = l_intra + den_inter;
        const int t = c0 + r;
        if (!(den > 0.f) && t < T) flag_status(status, kStatusNonPositiveNormaliser);
        const float inv = 1.f / den;                  // rows past T are not stored
        const float2 inv2 = make_float2(inv, inv);
        // the stage is free once the previous chunk's store has read it
        if (i > 0 && !warp_wait(&bars[kBarStageFree], (i - 1) & 1, abort_flag)) break;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          *reinterpret_cast<uint4 *>(stage + sw128(r, q4)) = pack8_scaled(oo + 8 * q4, inv2);
          *reinterpret_cast<uint4 *>(stage + sw128(r, 4 + q4)) = pack8_scaled(oo2 + 8 * q4, inv2);
        }
        fence_async_smem();
        warp_arrive(&bars[kBarStageFull]);          // warp 11 stores the tile
      }
    } else {
      // ---- increment kernel: the key features of tiles 1 and 3, so that
      //      two feature sets (and both issuing warps) work at once ----
      const int r = (warp & 3) * 32 + lane;               // token of the chunk
      // the key side zeroes the accumulators first (its Z-snapshot arrival)
      bool ok = warp_wait(&bars[kBarZSnap], 0, abort_flag);
      for (int i = 0; ok && i < nchunks; ++i) {
        const int st = i & 1;
        if (!(ok = warp_wait(&bars[kBarKvFull + st], (i >> 1) & 1, abort_flag))) break;
        uint32_t XK[16], P[32], R2[32];
        load_pairs(smem + L::kOffK + 8192 * st, r, XK, P);
        const uint32_t sc2 = SFX ? suffix_scale(tok_den, bh, T, t0 + i * kC + r) : 0x40004000u;
        if constexpr (SFX) {
          // c_t q_t for the weighted K^T K (read by warp 1 after this set's tile 1)
          const int t = t0 + i * kC + r;
          const float c = t < T ? tok_c[(size_t)bh * T + t] : 0.f;
          const uint32_t cc2 = tc::pack_bf16x2(c, c);
          uint8_t *cq = smem + L::kOffCQ + 8192 * st;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4 *>(cq + sw64(r, c4)) =
                make_uint4(bmul2(XK[4 * c4], cc2), bmul2(XK[4 * c4 + 1], cc2), bmul2(XK[4 * c4 + 2], cc2),
                           bmul2(XK[4 * c4 + 3], cc2));
        }
        warp_arrive(&bars[kBarKvEmpty + st]);           // K rows read
#pragma unroll
        for (int l = 0; l < 32; ++l) R2[l] = bmul2(P[(l + 4) & 31], sc2);   // x 2 (or 2 / d_t), rotated by 4
#pragma unroll 1
        for (int m = 1; m < kTiles; m += 2) {
          const int u = i * kTiles + m;
          if (!(ok = ring_acquire(&bars[kBarKRingEmpty], NK, u))) break;
          write_tile(kring + (u % NK) * kKSlotBytes, r, false, 0x3f803f80u, P, R2);
          ring_publish(&bars[kBarKRingFull], NK, u);
          rotate_left(R2, 8);
        }
      }
    }
  } else if (warp < 10) {
    // -------------------------------------------------- key side (warps 6..9)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                    // TMEM lane: token / feature row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t *snap = smem + L::kOffSnap;
    uint8_t *zsnap = smem + L::kOffZSnap;
    bool ok = true;

    // ---- carry-in: the initial state (library layout, if any; features
    //      doubled off the diagonal as inside the kernel) plus the increments
    //      of segments 0 .. g-1 ----
    {
      const float *seg0 = agg + (size_t)bh * G_total * kAggFloats;
#pragma unroll 1
      for (int m = 0; m < kTiles; ++m) {
        const int f = 128 * m + r;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {              // 16 columns at a time
          float acc[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[c] = 0.f;
          if (!AGG && f < kD && S0) {
            const float *s0 = S0 + ((size_t)bh * kD + abi_row(f)) * kDV + 16 * q4;
            const float mf = f < kDK ? 1.f : 2.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[c] = mf * s0[c];
          }
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
            *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4)) = pack8(bits);
            *reinterpret_cast<uint4 *>(snap + sw128(f, 2 * q4 + 1)) = pack8(bits + 8);
          }
        }
      }
      // Z rows live in lanes 0..31 (quarter 0); the other lanes hold zeros
      {
        float acc[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) acc[c] = 0.f;
        if (!AGG && r < kDK && z0) {
          // Z_rc = z_(min, max) (the library's packed row of the pair)
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int i = r < c ? r : c, j = r < c ? c : r;
            acc[c] = z0[(size_t)bh * kD + i * kDK - i * (i - 1) / 2 + (j - i)];
          }
        }
        if (!AGG && r < kDK) {
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
        if (!AGG && quarter == 0) {
#pragma unroll
          for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(zsnap + sw64(r, c)) = pack8(bits + 8 * c);
        }
      }
      fence_async_smem();
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(&bars[kBarZSnap]);
      if (!AGG)
        for (int m = 0; m < kTiles; ++m) warp_arrive(&bars[kBarTileSnap + m]);
    }

    for (int i = 0; i < nchunks; ++i) {
      const int st = i & 1;
      if (!(ok = warp_wait(&bars[kBarKvFull + st], (i >> 1) & 1, abort_flag))) break;
      // ---- phi(K_c) into the ring, one slot per state tile ----
      {
        uint32_t XK[16], P[32], R2[32];
        load_pairs(smem + L::kOffK + 8192 * st, r, XK, P);
        warp_arrive(&bars[kBarKvEmpty + st]);         // K rows read
        const uint32_t sc2 = SFX ? suffix_scale(tok_den, bh, T, t0 + i * kC + r) : 0x40004000u;
#pragma unroll
        for (int l = 0; l < 32; ++l) R2[l] = bmul2(P[l], sc2);   // x 2.0 (suffix: x 2 / d_t)
#pragma unroll 1
        for (int m = 0; m < kTiles; ++m) {
          const int u = i * kTiles + m;
          const bool mine = !AGG || (m & 1) == 0;        // increments: tiles 1, 3 go to warps 2..5
          if (ok && mine) ok = ring_acquire(&bars[kBarKRingEmpty], NK, u);
          if (ok && mine) {
            write_tile(kring + (u % NK) * kKSlotBytes, r, m == kTiles - 1,
                       m == 0 ? 0x3f003f00u : 0x3f803f80u, P, R2);     // x 1/2 on the diagonal
            ring_publish(&bars[kBarKRingFull], NK, u);
          }
          rotate_left(R2, 4);
        }
        if (!ok) break;
      }
      const bool last = i == nchunks - 1;
      if (last) {
        // the state after the last chunk is read below
        if (!(ok = warp_wait(&bars[kBarUpdFull], 0, abort_flag))) break;
        tc_fence_after();
        continue;
      }
      if (AGG) continue;
      // ---- snapshot Z_c+1, then S_c+1 tile by tile as the update finishes ----
      if (!(ok = warp_wait(&bars[kBarZDone], i & 1, abort_flag))) break;
      tc_fence_after();
      if (quarter == 0) {
        uint32_t zr[32];
        tmem_ld32(tbase + lane_off + kColZ, zr);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4 *>(zsnap + sw64(r, c)) = pack8(zr + 8 * c);
      }
      fence_async_smem();
      tc_fence_before();
      warp_arrive(&bars[kBarZSnap]);
      for (int m = 0; m < kTiles && ok; ++m) {
        if (!(ok = warp_wait(&bars[kBarTileDone + m], i & 1, abort_flag))) break;
        tc_fence_after();
        if (m < 4 || quarter == 0) {                       // tile 4: rows 512..527 (lanes 0..15)
          const int f = 128 * m + r;
          uint32_t a[32], b2[32];
          tmem_ld32(tbase + lane_off + kColS + 64 * m, a);
          tmem_ld32(tbase + lane_off + kColS + 64 * m + 32, b2);
          tmem_wait_ld();
          if (f < kD) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              *reinterpret_cast<uint4 *>(snap + sw128(f, q4)) = pack8(a + 8 * q4);
              *reinterpret_cast<uint4 *>(snap + sw128(f, 4 + q4)) = pack8(b2 + 8 * q4);
            }
          }
        }
        fence_async_smem();
        tc_fence_before();
        warp_arrive(&bars[kBarTileSnap + m]);
      }
      if (!ok) break;
    }

    // ---- state leaving the kernel ----
    const bool write_agg = AGG;
    const bool write_out = !AGG && g == G_total - 1 && (S_out || z_out);
    if (ok && nchunks > 0 && (write_agg || write_out)) {
      float *dst_agg = agg + ((size_t)bh * G_total + g) * kAggFloats;
#pragma unroll 1
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
            // increments stay in the internal scaling; S_out is S itself
            const float sc = (write_agg || f < kDK) ? 1.f : 0.5f;
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
  // one wave of CTAs: G segments of whole 128-token chunks per head; each
  // segment's increment is one piece
  const int g_req = (sequential || BH >= sms) ? 1 : (int)(sms / BH);
  tile_segments(T, kC, g_req, G, seg_len);
  *P = 1;
}

namespace {
// Launches the increment kernel over segments 0 .. G_inc - 1 (grid of BH x
// G_inc CTAs; agg strided by G_total increments per head).
cudaError_t launch_increments(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                              const CUtensorMap &to, float *agg, unsigned *status, long long BH,
                              int T, int G_inc, int G_total, int seg_len, cudaStream_t stream) {
  auto kagg = chunked_tc_kernel<true>;
  cudaError_t e = cudaFuncSetAttribute(kagg, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Layout<true>::kSmemBytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_segment_increment", stream);
  kagg<<<(unsigned)(BH * G_inc), kThreads, Layout<true>::kSmemBytes, stream>>>(
      tq, tk, tv, to, agg, nullptr, nullptr, nullptr, nullptr, status, T, G_inc, G_total, seg_len,
      nullptr, nullptr, 0);
  return cudaGetLastError();
}
}  // namespace

cudaError_t psd_tc_increments(const void *k, const void *v, float *agg, unsigned *status,
                              long long BH, int T, int G_inc, int G_total, int seg_len,
                              cudaStream_t stream) {
  if (G_inc <= 0) return cudaSuccess;
  CUtensorMap tk, tv;
  if (!make_tma_3d_bf16(&tk, k, kDK, T, BH, kC) || !make_tma_3d_bf16(&tv, v, kDV, T, BH, kC))
    return cudaErrorInvalidValue;
  return launch_increments(tk, tk, tv, tv, agg, status, BH, T, G_inc, G_total, seg_len, stream);
}

cudaError_t psd_tc_suffix_increments(const void *q, const void *dout, const float *den,
                                     const float *c, float *aggR, unsigned *status, long long BH,
                                     int T, int G, int seg_len, cudaStream_t stream) {
  if (G <= 1) return cudaSuccess;
  CUtensorMap tq, to;
  if (!make_tma_3d_bf16(&tq, q, kDK, T, BH, kC) || !make_tma_3d_bf16(&to, dout, kDV, T, BH, kC))
    return cudaErrorInvalidValue;
  auto ksfx = chunked_tc_kernel<true, true>;
  cudaError_t e = cudaFuncSetAttribute(ksfx, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Layout<true, true>::kSmemBytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_bwd_suffix_increment", stream);
  // segments 1 .. G-1 (the suffix carry of the earlier ones)
  ksfx<<<(unsigned)(BH * (G - 1)), kThreads, Layout<true, true>::kSmemBytes, stream>>>(
      tq, tq, to, to, aggR, nullptr, nullptr, nullptr, nullptr, status, T, G - 1, G, seg_len, den, c,
      1);
  return cudaGetLastError();
}

cudaError_t tc_chunked(const ChunkedLaunch &a) {
  int G, seg_len, P;
  tc_chunked_layout(a.BH, a.T, a.sms, a.sequential, &G, &seg_len, &P);
  // the state-only call reads neither q nor o: their maps are built on k, v
  // and never used by the increment kernel
  CUtensorMap tq, tk, tv, to;
  if (!make_tma_3d_bf16(&tq, a.state_only ? a.k : a.q, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tk, a.k, kDK, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&tv, a.v, kDV, a.T, a.BH, kC) ||
      !make_tma_3d_bf16(&to, a.state_only ? a.v : a.o, kDV, a.T, a.BH, kC))
    return cudaErrorInvalidValue;              // accepted shape: a failure, not a fallback
  cudaError_t e;
  // increments of segments 0 .. G-2 (all G for the state-only call)
  const int G_inc = a.state_only ? G : G - 1;
  if (G_inc > 0 &&
      (e = launch_increments(tq, tk, tv, to, a.agg, a.status, a.BH, a.T, G_inc, G, seg_len,
                             a.stream)) != cudaSuccess)
    return e;
  if (a.state_only)
    return state_reduce(kAggPsdTc, a.agg, a.BH, G, kD, kDK, kDV, a.S_out, a.z_out, 0.f, a.stream);
  auto kpass = chunked_tc_kernel<false>;
  e = cudaFuncSetAttribute(kpass, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Layout<false>::kSmemBytes);
  if (e != cudaSuccess) return e;
  ProfileScope prof("tc_segment_pass", a.stream);
  kpass<<<(unsigned)(a.BH * G), kThreads, Layout<false>::kSmemBytes, a.stream>>>(
      tq, tk, tv, to, a.agg, a.S0, a.z0, a.S_out, a.z_out, a.status, a.T, G, G, seg_len, nullptr,
      nullptr, 0);
  return cudaGetLastError();
}

}  // namespace kata
