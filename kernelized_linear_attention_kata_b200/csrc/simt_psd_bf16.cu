// CUDA-core kernels instantiated for feature kPSD, element type __nv_bfloat16.
#include "simt_launch.cuh"
namespace kata {
KATA_INSTANTIATE_SIMT(16, 16, kPSD, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(16, 32, kPSD, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(16, 64, kPSD, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(32, 16, kPSD, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(32, 32, kPSD, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(32, 64, kPSD, __nv_bfloat16)
}  // namespace kata
