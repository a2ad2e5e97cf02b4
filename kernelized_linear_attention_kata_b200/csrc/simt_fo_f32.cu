// CUDA-core kernels instantiated for feature kFirstOrder, element type float.
#include "simt_launch.cuh"
namespace kata {
KATA_INSTANTIATE_SIMT(16, 16, kFirstOrder, float)
KATA_INSTANTIATE_SIMT(16, 32, kFirstOrder, float)
KATA_INSTANTIATE_SIMT(16, 64, kFirstOrder, float)
KATA_INSTANTIATE_SIMT(32, 16, kFirstOrder, float)
KATA_INSTANTIATE_SIMT(32, 32, kFirstOrder, float)
KATA_INSTANTIATE_SIMT(32, 64, kFirstOrder, float)
KATA_INSTANTIATE_SIMT(64, 16, kFirstOrder, float)
KATA_INSTANTIATE_SIMT(64, 32, kFirstOrder, float)
KATA_INSTANTIATE_SIMT(64, 64, kFirstOrder, float)
}  // namespace kata
