// CUDA-core kernels instantiated for the two-factor features (KATA-Mg and
// KATA-Sigma-g, g = 2), element type float.
#include "simt_launch.cuh"
namespace kata {
KATA_INSTANTIATE_SIMT(16, 16, kMg2, float)
KATA_INSTANTIATE_SIMT(16, 32, kMg2, float)
KATA_INSTANTIATE_SIMT(16, 64, kMg2, float)
KATA_INSTANTIATE_SIMT(32, 16, kMg2, float)
KATA_INSTANTIATE_SIMT(32, 32, kMg2, float)
KATA_INSTANTIATE_SIMT(32, 64, kMg2, float)
KATA_INSTANTIATE_SIMT(16, 16, kSg2, float)
KATA_INSTANTIATE_SIMT(16, 32, kSg2, float)
KATA_INSTANTIATE_SIMT(16, 64, kSg2, float)
KATA_INSTANTIATE_SIMT(32, 16, kSg2, float)
KATA_INSTANTIATE_SIMT(32, 32, kSg2, float)
KATA_INSTANTIATE_SIMT(32, 64, kSg2, float)
}  // namespace kata
