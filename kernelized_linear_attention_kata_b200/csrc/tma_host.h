// Host-side creation of TMA tensor maps for [BH][T][d] bf16 tensors, through
// the driver entry point obtained from the runtime (no link against libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kata {

// Encodes a 3-D tiled map over a contiguous bf16 tensor [BH][T][d] with a
// box of (d, rows, 1) and the swizzle matching a d * 2-byte row (32, 64 or
// 128 bytes). Rows beyond T of a head read as zeros. Returns false on any
// failure (unsupported row size, misaligned base, driver error).
bool make_tma_3d_bf16(CUtensorMap *map, const void *base, int d, int T, long long BH, int rows);

}  // namespace kata
