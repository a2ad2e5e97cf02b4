// Building blocks shared by the PSD tensor-core kernels (bf16, d_k = 32,
// d_v = 64): the packed feature order, the shared-memory swizzles of the
// TMA tiles, the bf16 feature products and the layout of a segment
// increment.
//
// Feature order inside the kernels ("diagonal offset"): feature f = 32 d + l
// (d = 0..15, l = 0..31) is the pair (l, (l + d) mod 32); f = 512 + l
// (l < 16) is (l, l + 16). Every unordered pair i <= j appears once. State
// tile m (128 features, one TMEM accumulator of 128 lanes) holds offsets
// d = 4 m .. 4 m + 3 (lane 32 (d - 4 m) + l); tile 4 holds the 16 pairs
// (l, l + 16) in lanes 0..15.
//
// A segment increment (what a segment of chunks adds to the state) is
// [528][64] fp32 in this order with the off-diagonal rows doubled (m_f S_f,
// m_f = 2 off the diagonal), then the 32 x 32 matrix sum k k^T.
#pragma once

#include "tc_common.cuh"

namespace kata {
namespace psd {

constexpr int kC = 128;            // tokens per chunk (the MMA's M)
constexpr int kDK = 32;
constexpr int kDV = 64;
constexpr int kD = 528;
constexpr int kTiles = 5;          // 128-feature state tiles: ceil(528 / 128)
constexpr int kAggFloats = kD * kDV + kDK * kDK;      // one segment increment

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

// The feature loops below are rolled (one body for every slot or tile, to
// keep the code small); register indices stay static by walking a rotated
// copy R of the pair array: R[l] = P[(l + d0) mod 32] for the slot's or
// tile's first offset d0, rotated further after each use.
__device__ __forceinline__ void rotate_left(uint32_t (&R)[32], int by) {
  uint32_t t[32];
#pragma unroll
  for (int l = 0; l < 32; ++l) t[l] = R[(l + by) & 31];
#pragma unroll
  for (int l = 0; l < 32; ++l) R[l] = t[l];
}

// Query features of readout slot s (features 64 s .. 64 s + 63: offsets
// d = 2 s, 2 s + 1; slot 8 holds only (16, l < 16)) for one token row, as 32
// bf16 pairs, word c holding features 2c (low half) and 2c + 1 (the K order
// of a tensor-memory A operand): word j = (2 s, 2 j), word 16 + j =
// (2 s + 1, 2 j). R = P rotated by 2 s. The off-diagonal multiplicity 2 of
// the query feature is carried by the state instead (see write_tile).
__device__ __forceinline__ void q_slot_words(const uint32_t (&P)[32], const uint32_t (&R)[32],
                                             bool partial, uint32_t (&w)[32]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    w[j] = bmul2(P[2 * j], R[2 * j]);
    w[16 + j] = bmul2(P[2 * j], R[2 * j + 1]);
  }
  if (partial) {
#pragma unroll
    for (int j = 8; j < 32; ++j) w[j] = 0u;
  }
}

// Key features of state tile m (128 m .. 128 m + 127: offsets d = 4 m ..
// 4 m + 3 in two 64-feature groups 16 KB apart; tile 4 holds only
// (16, l < 16)) for one token row, with the off-diagonal features doubled:
// R2 = 2 P rotated by 4 m, and the diagonal (tile 0, first offset) scaled
// back by dscale = 1/2. The state accumulated inside the kernel is therefore
// S'_f = m_f S_f (m_f = 1 on the diagonal, 2 off it), so that the readout's
// plain query products give phi_q(q) . S; the scaling by 2 is exact and is
// undone where the state leaves the kernel.
__device__ __forceinline__ void write_tile(uint8_t *slot, int row, bool partial, uint32_t dscale,
                                           const uint32_t (&P)[32], const uint32_t (&R2)[32]) {
#pragma unroll
  for (int g2 = 0; g2 < 2; ++g2) {
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      if (partial && (g2 != 0 || cc >= 2)) continue;
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int l = 8 * (cc & 3) + 2 * k;
        w[k] = bmul2(P[l], R2[(l + 2 * g2 + (cc >> 2)) & 31]);
        if (g2 == 0 && cc < 4) w[k] = bmul2(w[k], dscale);
      }
      *reinterpret_cast<uint4 *>(slot + g2 * 16384 + sw128(row, cc)) = make_uint4(w[0], w[1], w[2], w[3]);
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

// Eight fp32 values times inv, rounded to bf16.
__device__ __forceinline__ uint4 pack8_scaled(const uint32_t *a, float2 inv2) {
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 v = __fmul2_rn(make_float2(__uint_as_float(a[2 * j]), __uint_as_float(a[2 * j + 1])), inv2);
    w[j] = tc::pack_bf16x2(v.x, v.y);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 pack8(const uint32_t *a) {
  return make_uint4(tc::pack_bf16x2(__uint_as_float(a[0]), __uint_as_float(a[1])),
                    tc::pack_bf16x2(__uint_as_float(a[2]), __uint_as_float(a[3])),
                    tc::pack_bf16x2(__uint_as_float(a[4]), __uint_as_float(a[5])),
                    tc::pack_bf16x2(__uint_as_float(a[6]), __uint_as_float(a[7])));
}

// Math-set synchronisation: every thread of the set waits and arrives
// (counted per thread), so no lane depends on another lane's wait.
constexpr uint32_t kSetArrivals = 128;
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, abort_flag));
}
__device__ __forceinline__ void warp_arrive(uint64_t *bar) { tc::mbar_arrive(bar); }


}  // namespace psd
}  // namespace kata
