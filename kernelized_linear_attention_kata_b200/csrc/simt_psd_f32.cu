// CUDA-core kernels instantiated for feature kPSD, element type float.
#include "simt_launch.cuh"
namespace kata {
KATA_INSTANTIATE_SIMT(16, 16, kPSD, float)
KATA_INSTANTIATE_SIMT(16, 32, kPSD, float)
KATA_INSTANTIATE_SIMT(16, 64, kPSD, float)
KATA_INSTANTIATE_SIMT(32, 16, kPSD, float)
KATA_INSTANTIATE_SIMT(32, 32, kPSD, float)
KATA_INSTANTIATE_SIMT(32, 64, kPSD, float)
}  // namespace kata
