// CUDA-core kernels instantiated for feature kFirstOrder, element type __nv_bfloat16.
#include "simt_launch.cuh"
namespace kata {
KATA_INSTANTIATE_SIMT(16, 16, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(16, 32, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(16, 64, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(32, 16, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(32, 32, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(32, 64, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(64, 16, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(64, 32, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_SIMT(64, 64, kFirstOrder, __nv_bfloat16)
}  // namespace kata
