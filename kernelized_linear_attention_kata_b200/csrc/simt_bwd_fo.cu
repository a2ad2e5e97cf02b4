// Backward kernels instantiated for feature kFirstOrder, both element types.
#include "simt_backward.cuh"
namespace kata {
KATA_INSTANTIATE_BACKWARD(16, 16, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(16, 32, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(16, 64, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(32, 16, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(32, 32, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(32, 64, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(64, 16, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(64, 32, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(64, 64, kFirstOrder, float)
KATA_INSTANTIATE_BACKWARD(16, 16, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_BACKWARD(16, 32, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_BACKWARD(16, 64, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_BACKWARD(32, 16, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_BACKWARD(32, 32, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_BACKWARD(32, 64, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_BACKWARD(64, 16, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_BACKWARD(64, 32, kFirstOrder, __nv_bfloat16)
KATA_INSTANTIATE_BACKWARD(64, 64, kFirstOrder, __nv_bfloat16)
}  // namespace kata
