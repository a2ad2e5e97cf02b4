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
// symbol, not a device address; its device address on the current device is
// looked up with cudaGetSymbolAddress on every call and passed on as the
// workspace pointer. Every call shares the array: the status word is
// cleared at the start of each call (the increments are fully written before
// they are read), and two calls whose work overlaps on the GPU race on it.
#include "../../include/kata.h"

#include <cuda_runtime.h>


namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KATA_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device and context.
// It is looked up on every call (a table lookup in the runtime once the
// module is loaded), so that a device reset or a new primary context cannot
// leave a stale address behind.
kata_status_t scratch_address(void **out) {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KATA_ERR_CUDA;
  *out = p;
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
  void *scratch = nullptr;
  const kata_status_t st = scratch_address(&scratch);
  if (st != KATA_OK) return st;
  return kata_fwd_chunked(q, k, v, o, B, H, T, d_k, d_v, C, dtype, feature, S_out, z_out, scratch,
                          (size_t)KATA_NOALLOC_SCRATCH_BYTES, stream);
}
