// Launchers of the CUDA-core kernels (definitions; instantiated per feature
// and element type in simt_*.cu).
#pragma once

#include "launch.h"
#include "profile.h"
#include "simt_kernels.cuh"

namespace kata {

template <int DK, int DV, int FEAT, typename Tin>
cudaError_t simt_chunked(const ChunkedLaunch &a) {
  constexpr int D = state_dim(DK, FEAT);
  const Tin *q = static_cast<const Tin *>(a.q);
  const Tin *k = static_cast<const Tin *>(a.k);
  const Tin *v = static_cast<const Tin *>(a.v);
  Tin *o = static_cast<Tin *>(a.o);
  if (a.state_only) {
    // every segment's increment, then their sum in the library layout
    ProfileScope prof("simt_segment_increment", a.stream);
    segment_increment_kernel<DK, DV, FEAT, Tin><<<(unsigned)(a.BH * a.G), (D + 31) / 32 * 32, 0,
                                                   a.stream>>>(k, v, a.agg, a.T, a.G, a.G,
                                                               a.seg_len);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return state_reduce(kAggLibrary, a.agg, a.BH, a.G, D, DK, DV, a.S_out, a.z_out, 0.f, a.stream);
  }
  if (a.G > 1) {
    const int threads = (D + 31) / 32 * 32;
    ProfileScope prof("simt_segment_increment", a.stream);
    segment_increment_kernel<DK, DV, FEAT, Tin>
        <<<(unsigned)(a.BH * (a.G - 1)), threads, 0, a.stream>>>(k, v, a.agg, a.T, a.G - 1, a.G,
                                                                  a.seg_len);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t smem = segment_pass_smem<DK, DV, FEAT>(a.C);
  auto kern = segment_pass_kernel<DK, DV, FEAT, Tin>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfileScope prof("simt_segment_pass", a.stream);
  kern<<<(unsigned)(a.BH * a.G), kSegThreads, smem, a.stream>>>(
      q, k, v, o, a.agg, a.S0, a.z0, a.S_out, a.z_out, a.status, a.T, a.C, a.G, a.seg_len);
  return cudaGetLastError();
}

template <int DK, int DV, int FEAT, typename Tin>
cudaError_t simt_quadratic(const QuadraticLaunch &a) {
  dim3 grid((a.T + kQuadBlock - 1) / kQuadBlock, (unsigned)a.BH);
  ProfileScope prof("simt_quadratic", a.stream);
  quadratic_kernel<DK, DV, FEAT, Tin><<<grid, kQuadBlock * (DV / 16), 0, a.stream>>>(
      static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v),
      static_cast<Tin *>(a.o), a.T);
  return cudaGetLastError();
}

template <int DK, int DV, int FEAT, typename Tin>
cudaError_t simt_decode(const DecodeLaunch &a) {
  ProfileScope prof("simt_decode", a.stream);
  decode_kernel<DK, DV, FEAT, Tin><<<(unsigned)a.BH, kDecThreads, 0, a.stream>>>(
      static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v),
      a.S, a.z, static_cast<Tin *>(a.y));
  return cudaGetLastError();
}

#define KATA_INSTANTIATE_SIMT(DK, DV, FEAT, TIN)                                     \
  template cudaError_t simt_chunked<DK, DV, FEAT, TIN>(const ChunkedLaunch &);       \
  template cudaError_t simt_quadratic<DK, DV, FEAT, TIN>(const QuadraticLaunch &);   \
  template cudaError_t simt_decode<DK, DV, FEAT, TIN>(const DecodeLaunch &);

}  // namespace kata
