// kata_fwd_chunked_noalloc: the chunked-state forward for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc or hand this library a workspace: a
// host application whose device memory is owned entirely by another
// runtime's pool, or latency-critical code that must not trigger the
// device-wide synchronisation cudaMalloc / cudaFree can cause. For them the
// scratch that kata_fwd_chunked needs (a status word plus the per-segment
// state increments) lives in one fixed, file-scope device array that every
// GPU loading this library holds until the process exits.
//
// The array's name, used in host code, is only a host-side stand-in for the
// symbol, not a device address; its device address is looked up once per
// device with cudaGetSymbolAddress (with that device current) and passed on
// as the workspace pointer. Every call shares the array: the status word is
// cleared at the start of each call (the increments are fully written before
// they are read), and two calls whose work overlaps on the GPU race on it.
#include "../../include/kata.h"

#include <cuda_runtime.h>

#include <mutex>

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KATA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on `dev` (the current device), looked
// up on the first call for that device.
kata_status_t scratch_for_device(int dev, void **out) {
  if (dev < 0 || dev >= kMaxDevices) return KATA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KATA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KATA_OK;
}

}  // namespace

extern "C" kata_status_t kata_fwd_chunked_noalloc(const void *q, const void *k, const void *v,
                                                  void *o, int B, int H, int T, int d_k, int d_v,
                                                  int C, kata_dtype_t dtype,
                                                  kata_feature_t feature, float *S_out,
                                                  float *z_out, kata_stream_t stream) {
  if (B < 0 || H < 0 || T < 0 || C <= 0) return KATA_ERR_INVALID_ARGUMENT;
  // the plan query tells an unsupported shape (KATA_ERR_UNSUPPORTED) from a
  // device that cannot be queried (KATA_ERR_CUDA)
  kata_plan_t plan;
  const kata_status_t pst = kata_fwd_chunked_plan(B, H, T, d_k, d_v, C, dtype, feature, 0, &plan);
  if (pst != KATA_OK) return pst;
  const size_t need = kata_fwd_chunked_workspace_bytes(B, H, T, d_k, d_v, C, dtype, feature);
  if (need == 0) return KATA_ERR_CUDA;
  if (need > (size_t)KATA_NOALLOC_SCRATCH_BYTES) return KATA_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KATA_ERR_CUDA;
  void *scratch = nullptr;
  const kata_status_t st = scratch_for_device(dev, &scratch);
  if (st != KATA_OK) return st;
  return kata_fwd_chunked(q, k, v, o, B, H, T, d_k, d_v, C, dtype, feature, S_out, z_out, scratch,
                          (size_t)KATA_NOALLOC_SCRATCH_BYTES, stream);
}
