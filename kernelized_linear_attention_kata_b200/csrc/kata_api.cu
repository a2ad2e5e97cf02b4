// C ABI of the KATA library: argument validation, workspace layout and
// kernel dispatch. Declarations and the full contract are in include/kata.h.
#include "../../include/kata.h"

#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"

using namespace kata;

namespace {

constexpr size_t kHeaderBytes = 256;   // status word + padding
constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool supported(int d_k, int d_v, int C, kata_dtype_t dtype, kata_feature_t feature) {
  if (dtype != KATA_DTYPE_F32 && dtype != KATA_DTYPE_BF16) return false;
  if (feature == KATA_FEATURE_PSD) {
    if (d_k != 16 && d_k != 32) return false;
  } else if (feature == KATA_FEATURE_FIRST_ORDER) {
    if (d_k != 16 && d_k != 32 && d_k != 64) return false;
  } else if (feature == KATA_FEATURE_MULTI_PSD2 || feature == KATA_FEATURE_SUMMED_PSD2) {
    if (d_k != 16 && d_k != 32) return false;
  } else {
    return false;
  }
  if (d_v != 16 && d_v != 32 && d_v != 64) return false;
  if (C != 0 && C != 16 && C != 32 && C != 64 && C != 128) return false;
  return true;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Segment split of the chunked forward: G segments of `chunks_per_seg`
// chunks per (b, h), sized so that B*H*G blocks fill the SMs once.
struct Split {
  int G;
  int seg_len;   // tokens per segment (a multiple of C)
};

Split segment_split(long long BH, int T, int C, int sms, bool sequential) {
  const int n_chunks = T <= 0 ? 0 : (T + C - 1) / C;
  if (sequential || n_chunks <= 1 || BH >= sms) return {1, n_chunks * C};
  long long G = sms / BH;
  if (G < 1) G = 1;
  if (G > n_chunks) G = n_chunks;
  const int per = (int)((n_chunks + G - 1) / G);
  const int Gr = (n_chunks + per - 1) / per;
  return {Gr, per * C};
}

// Floats of one segment increment: the CUDA-core kernels keep [D][d_v + 1]
// (z as the last column), the tensor-core kernel keeps [D][d_v] then the
// d_k x d_k matrix sum k k^T; the workspace holds the larger.
size_t increment_floats(int D, int d_k, int d_v) {
  const size_t simt = (size_t)D * (size_t)(d_v + 1);
  const size_t tc = (size_t)D * (size_t)d_v + (size_t)d_k * (size_t)d_k;
  return simt > tc ? simt : tc;
}

// Increments per head a chunked request keeps in its workspace: one per
// segment, or, on the PSD tensor-core path, one per piece of a segment.
size_t increments_per_head(kata_path_t path, long long BH, int T, int sms, bool sequential,
                           const Split &sp) {
  if (path == KATA_PATH_TENSOR_CORE_PSD && !sequential) {   // the sequential carry needs none
    int G, seg_len, P;
    tc_chunked_layout(BH, T, sms, sequential, &G, &seg_len, &P);
    return (size_t)G * (size_t)P;
  }
  if (path == KATA_PATH_TENSOR_CORE_MULTI_FACTOR) {
    int G, seg_len;
    var_tc_layout(BH, T, sms, sequential, &G, &seg_len);
    return (size_t)G;
  }
  return (size_t)sp.G;
}

size_t workspace_bytes_for(long long BH, int D, int d_k, int d_v, size_t incs_per_head) {
  const size_t agg = (size_t)BH * incs_per_head * increment_floats(D, d_k, d_v) * sizeof(float);
  return kHeaderBytes + align_up(agg, kAlign);
}

// Backward workspace: status header | prefix-state increments | suffix-state
// increments (each [BH][G][D][d_v + 1] fp32) | normalisers d_t [BH][T] fp32 |
// c_t [BH][T] fp32.
struct BwdLayout {
  size_t agg_bytes, den_bytes;
  size_t aggS() const { return kHeaderBytes; }
  size_t aggR() const { return kHeaderBytes + agg_bytes; }
  size_t den() const { return kHeaderBytes + 2 * agg_bytes; }
  size_t c() const { return kHeaderBytes + 2 * agg_bytes + den_bytes; }
  size_t total() const { return kHeaderBytes + 2 * agg_bytes + 2 * den_bytes; }
};

// The tensor-core dq pass (bf16 PSD, d_k = 32, d_v = 64) keeps its prefix
// increments in the forward's tensor-core layout and split; each increment
// region is sized for the larger of the two layouts.
bool bwd_tc_shape(int d_k, int d_v, int C, kata_dtype_t dtype, kata_feature_t feature) {
  return dtype == KATA_DTYPE_BF16 && feature == KATA_FEATURE_PSD && d_k == 32 && d_v == 64 &&
         (C == 64 || C == 128);
}

void bwd_tc_split(long long BH, int T, int sms, int *G, int *seg_len) {
  int P;
  tc_chunked_layout(BH, T, sms, false, G, seg_len, &P);
}

BwdLayout bwd_layout(long long BH, int T, int D, int d_v, const Split &sp, bool tc, int sms) {
  size_t agg = (size_t)BH * (size_t)sp.G * (size_t)D * (size_t)(d_v + 1) * sizeof(float);
  if (tc) {
    int G, seg_len;
    bwd_tc_split(BH, T, sms, &G, &seg_len);
    const size_t tc_agg = (size_t)BH * (size_t)G * tc_chunked_agg_floats() * sizeof(float);
    agg = agg > tc_agg ? agg : tc_agg;
  }
  return {align_up(agg, kAlign), align_up((size_t)BH * (size_t)T * sizeof(float), kAlign)};
}

// Calls F::template run<DK, DV, FEAT>() for the runtime (d_k, d_v, feature).
template <typename F>
kata_status_t dispatch_shape(int d_k, int d_v, kata_feature_t feature, F &f) {
#define KATA_DV_CASES(DK, FEAT)                                         \
  switch (d_v) {                                                        \
    case 16: return f.template operator()<DK, 16, FEAT>();              \
    case 32: return f.template operator()<DK, 32, FEAT>();              \
    case 64: return f.template operator()<DK, 64, FEAT>();              \
    default: return KATA_ERR_UNSUPPORTED;                               \
  }
  if (feature == KATA_FEATURE_PSD) {
    if (d_k == 16) { KATA_DV_CASES(16, kPSD) }
    if (d_k == 32) { KATA_DV_CASES(32, kPSD) }
  } else if (feature == KATA_FEATURE_FIRST_ORDER) {
    if (d_k == 16) { KATA_DV_CASES(16, kFirstOrder) }
    if (d_k == 32) { KATA_DV_CASES(32, kFirstOrder) }
    if (d_k == 64) { KATA_DV_CASES(64, kFirstOrder) }
  } else if constexpr (!F::kBaseFeaturesOnly) {
    if (feature == KATA_FEATURE_MULTI_PSD2) {
      if (d_k == 16) { KATA_DV_CASES(16, kMg2) }
      if (d_k == 32) { KATA_DV_CASES(32, kMg2) }
    } else if (feature == KATA_FEATURE_SUMMED_PSD2) {
      if (d_k == 16) { KATA_DV_CASES(16, kSg2) }
      if (d_k == 32) { KATA_DV_CASES(32, kSg2) }
    }
  }
#undef KATA_DV_CASES
  return KATA_ERR_UNSUPPORTED;
}

// Kernel family of a chunked request: decided from the shape and the
// pointers' alignment only, so that kata_fwd_chunked_plan reports exactly
// what a call runs.
kata_path_t chunked_path(const ChunkedLaunch &a, int d_k, int d_v, int C, kata_dtype_t dtype,
                         int feature) {
  if (a.BH == 0 || a.T == 0) return KATA_PATH_NONE;
  if (dtype == KATA_DTYPE_BF16 && tc_chunked_supported(a, d_k, d_v, C, feature))
    return KATA_PATH_TENSOR_CORE_PSD;
  if (dtype == KATA_DTYPE_BF16 && fo_tc_supported(a, d_k, d_v, C, feature))
    return KATA_PATH_TENSOR_CORE_FIRST_ORDER;
  if (dtype == KATA_DTYPE_BF16 && var_tc_supported(a, d_k, d_v, C, feature))
    return KATA_PATH_TENSOR_CORE_MULTI_FACTOR;
  return KATA_PATH_CUDA_CORE;
}

struct ChunkedRun {
  static constexpr bool kBaseFeaturesOnly = false;
  kata_dtype_t dtype;
  ChunkedLaunch a;
  template <int DK, int DV, int FEAT> kata_status_t operator()() {
    cudaError_t e;
    switch (chunked_path(a, DK, DV, a.C, dtype, FEAT)) {
      case KATA_PATH_TENSOR_CORE_PSD: e = tc_chunked(a); break;
      case KATA_PATH_TENSOR_CORE_FIRST_ORDER: e = fo_tc(a); break;
      case KATA_PATH_TENSOR_CORE_MULTI_FACTOR: e = var_tc(a, FEAT); break;
      default:
        e = dtype == KATA_DTYPE_F32 ? simt_chunked<DK, DV, FEAT, float>(a)
                                    : simt_chunked<DK, DV, FEAT, __nv_bfloat16>(a);
    }
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
  }
};

struct QuadraticRun {
  static constexpr bool kBaseFeaturesOnly = false;
  kata_dtype_t dtype;
  QuadraticLaunch a;
  template <int DK, int DV, int FEAT> kata_status_t operator()() {
    cudaError_t e = cudaErrorNotSupported;
    if (dtype == KATA_DTYPE_BF16) e = tc_quadratic(a, DK, DV, FEAT);
    if (e == cudaErrorNotSupported)
      e = dtype == KATA_DTYPE_F32 ? simt_quadratic<DK, DV, FEAT, float>(a)
                                  : simt_quadratic<DK, DV, FEAT, __nv_bfloat16>(a);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
  }
};

struct BackwardRun {
  static constexpr bool kBaseFeaturesOnly = true;     // the gradient covers PSD and first-order
  kata_dtype_t dtype;
  BackwardLaunch a;
  bool tc;                 // bf16 PSD d_k = 32, d_v = 64: the tensor-core kernels
  int tc_G, tc_seg_len;
  template <int DK, int DV, int FEAT> kata_status_t operator()() {
    cudaError_t e;
    if constexpr (DK == 32 && DV == 64 && FEAT == kPSD) {
      if (tc) {
        e = tc_bwd_dq(a, a.aggS, tc_G, tc_seg_len);
        if (e == cudaSuccess) e = tc_bwd_dkdv(a, a.aggR, tc_G, tc_seg_len);
        return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
      }
    }
    e = dtype == KATA_DTYPE_F32 ? simt_backward<DK, DV, FEAT, float>(a)
                                : simt_backward<DK, DV, FEAT, __nv_bfloat16>(a);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
  }
};

struct DecodeRun {
  static constexpr bool kBaseFeaturesOnly = false;
  kata_dtype_t dtype;
  DecodeLaunch a;
  template <int DK, int DV, int FEAT> kata_status_t operator()() {
    cudaError_t e = dtype == KATA_DTYPE_F32 ? simt_decode<DK, DV, FEAT, float>(a)
                                            : simt_decode<DK, DV, FEAT, __nv_bfloat16>(a);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
  }
};

kata_status_t chunked_common(const void *q, const void *k, const void *v, void *o, int B, int H,
                             int T, int d_k, int d_v, int C, kata_dtype_t dtype,
                             kata_feature_t feature, float *S_out, float *z_out, void *workspace,
                             size_t workspace_bytes, kata_stream_t stream_, bool sequential,
                             const float *S0 = nullptr, const float *z0 = nullptr,
                             bool state_only = false) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B < 0 || H < 0 || T < 0 || C <= 0) return KATA_ERR_INVALID_ARGUMENT;
  if (!supported(d_k, d_v, C, dtype, feature)) return KATA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  const int D = (int)kata_state_dim(d_k, feature);
  if (!workspace) return KATA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return KATA_ERR_WORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return KATA_ERR_CUDA;
  const Split sp = segment_split(BH, T, C, sms, sequential);
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  ChunkedLaunch a{q, k, v, o, BH, T, C, S_out, z_out, reinterpret_cast<unsigned *>(ws),
                  reinterpret_cast<float *>(ws + kHeaderBytes), sp.G, sp.seg_len, stream};
  a.S0 = S0;
  a.z0 = z0;
  a.state_only = state_only;
  a.sms = sms;
  a.sequential = sequential;
  const kata_path_t path = chunked_path(a, d_k, d_v, C, dtype, feature);
  if (workspace_bytes <
      workspace_bytes_for(BH, D, d_k, d_v, increments_per_head(path, BH, T, sms, sequential, sp)))
    return KATA_ERR_WORKSPACE;
  if (BH == 0 || T == 0) {
    // no tokens: the state out is the initial state (zero if none is given)
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), stream) != cudaSuccess) return KATA_ERR_CUDA;
    const size_t sb = (size_t)BH * D * d_v * sizeof(float), zb = (size_t)BH * D * sizeof(float);
    if (S_out && BH > 0 &&
        (S0 ? cudaMemcpyAsync(S_out, S0, sb, cudaMemcpyDeviceToDevice, stream)
            : cudaMemsetAsync(S_out, 0, sb, stream)) != cudaSuccess)
      return KATA_ERR_CUDA;
    if (z_out && BH > 0 &&
        (z0 ? cudaMemcpyAsync(z_out, z0, zb, cudaMemcpyDeviceToDevice, stream)
            : cudaMemsetAsync(z_out, 0, zb, stream)) != cudaSuccess)
      return KATA_ERR_CUDA;
    return KATA_OK;
  }
  if (!k || !v || (!state_only && (!q || !o))) return KATA_ERR_INVALID_ARGUMENT;
  if (cudaMemsetAsync(a.status, 0, sizeof(unsigned), stream) != cudaSuccess) return KATA_ERR_CUDA;
  ChunkedRun run{dtype, a};
  return dispatch_shape(d_k, d_v, feature, run);
}

}  // namespace

extern "C" {

int kata_version(void) { return 100; }

const char *kata_status_string(kata_status_t s) {
  switch (s) {
    case KATA_OK: return "KATA_OK";
    case KATA_ERR_INVALID_ARGUMENT: return "KATA_ERR_INVALID_ARGUMENT";
    case KATA_ERR_UNSUPPORTED: return "KATA_ERR_UNSUPPORTED";
    case KATA_ERR_WORKSPACE: return "KATA_ERR_WORKSPACE";
    case KATA_ERR_CUDA: return "KATA_ERR_CUDA";
    case KATA_ERR_NONPOSITIVE_NORMALISER: return "KATA_ERR_NONPOSITIVE_NORMALISER";
    case KATA_ERR_DEVICE_TIMEOUT: return "KATA_ERR_DEVICE_TIMEOUT";
  }
  return "KATA_ERR_UNKNOWN";
}

size_t kata_state_dim(int d_k, kata_feature_t feature) {
  if (d_k <= 0) return 0;
  if (feature == KATA_FEATURE_PSD) return (size_t)d_k * (d_k + 1) / 2;
  if (feature == KATA_FEATURE_FIRST_ORDER) return (size_t)d_k + 1;
  if (d_k % 2) return 0;
  const size_t h = (size_t)d_k / 2;
  if (feature == KATA_FEATURE_MULTI_PSD2) return h * (h + 1);
  if (feature == KATA_FEATURE_SUMMED_PSD2) return h * (h + 1) / 2;
  return 0;
}

kata_status_t kata_fwd_chunked_plan(int B, int H, int T, int d_k, int d_v, int C,
                                    kata_dtype_t dtype, kata_feature_t feature, int sequential,
                                    kata_plan_t *out) {
  if (B < 0 || H < 0 || T < 0 || C <= 0 || !out) return KATA_ERR_INVALID_ARGUMENT;
  if (!supported(d_k, d_v, C, dtype, feature)) return KATA_ERR_UNSUPPORTED;
  const int sms = device_sm_count();
  if (sms <= 0) return KATA_ERR_CUDA;
  const long long BH = (long long)B * H;
  const Split sp = segment_split(BH, T, C, sms, sequential != 0);
  // 16-byte aligned stand-ins for the caller's buffers (never dereferenced)
  void *aligned = reinterpret_cast<void *>(uintptr_t(256));
  ChunkedLaunch a{aligned, aligned, aligned, aligned, BH, T, C, nullptr, nullptr, nullptr,
                  nullptr, sp.G, sp.seg_len, nullptr};
  kata_plan_t p{};
  p.path = chunked_path(a, d_k, d_v, C, dtype, feature);
  if (p.path == KATA_PATH_TENSOR_CORE_PSD) {
    int P;
    p.chunk_tokens = 128;
    tc_chunked_layout(BH, T, sms, sequential != 0, &p.segments, &p.segment_tokens, &P);
  } else if (p.path == KATA_PATH_TENSOR_CORE_FIRST_ORDER) {
    p.chunk_tokens = 128;
    tile_segments(T, 128, sp.G, &p.segments, &p.segment_tokens);
  } else if (p.path == KATA_PATH_TENSOR_CORE_MULTI_FACTOR) {
    p.chunk_tokens = 128;
    var_tc_layout(BH, T, sms, sequential != 0, &p.segments, &p.segment_tokens);
  } else {
    p.chunk_tokens = C;
    p.segments = sp.G;
    p.segment_tokens = sp.seg_len;
  }
  *out = p;
  return KATA_OK;
}

size_t kata_fwd_chunked_workspace_bytes(int B, int H, int T, int d_k, int d_v, int C,
                                        kata_dtype_t dtype, kata_feature_t feature) {
  if (B < 0 || H < 0 || T < 0 || C <= 0) return 0;
  if (!supported(d_k, d_v, C, dtype, feature)) return 0;
  const int sms = device_sm_count();
  if (sms <= 0) return 0;
  const long long BH = (long long)B * H;
  const Split sp = segment_split(BH, T, C, sms, false);
  // the forward needs at least what the sequential carry needs, so one size
  // serves both entry points; the path is the one 16-byte aligned buffers take
  void *aligned = reinterpret_cast<void *>(uintptr_t(256));
  ChunkedLaunch a{aligned, aligned, aligned, aligned, BH, T, C, nullptr, nullptr, nullptr,
                  nullptr, sp.G, sp.seg_len, nullptr};
  const kata_path_t path = chunked_path(a, d_k, d_v, C, dtype, feature);
  size_t incs = increments_per_head(path, BH, T, sms, false, sp);
  // the variants' state-only call (kata_chunked_state) runs on the CUDA cores
  // with their split: the size covers both
  if (path == KATA_PATH_TENSOR_CORE_MULTI_FACTOR && (size_t)sp.G > incs) incs = (size_t)sp.G;
  return workspace_bytes_for(BH, (int)kata_state_dim(d_k, feature), d_k, d_v, incs);
}

kata_status_t kata_fwd_chunked(const void *q, const void *k, const void *v, void *o, int B, int H,
                               int T, int d_k, int d_v, int C, kata_dtype_t dtype,
                               kata_feature_t feature, float *S_out, float *z_out,
                               void *workspace, size_t workspace_bytes, kata_stream_t stream) {
  return chunked_common(q, k, v, o, B, H, T, d_k, d_v, C, dtype, feature, S_out, z_out, workspace,
                        workspace_bytes, stream, false);
}

kata_status_t kata_fwd_chunked_sequential(const void *q, const void *k, const void *v, void *o,
                                          int B, int H, int T, int d_k, int d_v, int C,
                                          kata_dtype_t dtype, kata_feature_t feature,
                                          float *S_out, float *z_out, void *workspace,
                                          size_t workspace_bytes, kata_stream_t stream) {
  return chunked_common(q, k, v, o, B, H, T, d_k, d_v, C, dtype, feature, S_out, z_out, workspace,
                        workspace_bytes, stream, true);
}

kata_status_t kata_fwd_chunked_from_state(const void *q, const void *k, const void *v, void *o,
                                          int B, int H, int T, int d_k, int d_v, int C,
                                          kata_dtype_t dtype, kata_feature_t feature,
                                          const float *S0, const float *z0, float *S_out,
                                          float *z_out, void *workspace, size_t workspace_bytes,
                                          kata_stream_t stream) {
  return chunked_common(q, k, v, o, B, H, T, d_k, d_v, C, dtype, feature, S_out, z_out, workspace,
                        workspace_bytes, stream, false, S0, z0);
}

kata_status_t kata_chunked_state(const void *k, const void *v, int B, int H, int T, int d_k,
                                 int d_v, int C, kata_dtype_t dtype, kata_feature_t feature,
                                 float *S_out, float *z_out, void *workspace,
                                 size_t workspace_bytes, kata_stream_t stream) {
  return chunked_common(nullptr, k, v, nullptr, B, H, T, d_k, d_v, C, dtype, feature, S_out, z_out,
                        workspace, workspace_bytes, stream, false, nullptr, nullptr, true);
}

kata_status_t kata_fwd_quadratic(const void *q, const void *k, const void *v, void *o, int B,
                                 int H, int T, int d_k, int d_v, kata_dtype_t dtype,
                                 kata_feature_t feature, kata_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B < 0 || H < 0 || T < 0) return KATA_ERR_INVALID_ARGUMENT;
  if (!supported(d_k, d_v, 0, dtype, feature)) return KATA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH == 0 || T == 0) return KATA_OK;
  if (!q || !k || !v || !o) return KATA_ERR_INVALID_ARGUMENT;
  if (BH > 65535) return KATA_ERR_UNSUPPORTED;
  QuadraticRun run{dtype, QuadraticLaunch{q, k, v, o, BH, T, stream}};
  return dispatch_shape(d_k, d_v, feature, run);
}

kata_status_t kata_decode_step(const void *q, const void *k, const void *v, float *S, float *z,
                               void *y, int B, int H, int d_k, int d_v, kata_dtype_t dtype,
                               kata_feature_t feature, kata_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B < 0 || H < 0) return KATA_ERR_INVALID_ARGUMENT;
  if (!supported(d_k, d_v, 0, dtype, feature)) return KATA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH == 0) return KATA_OK;
  if (!q || !k || !v || !S || !z || !y) return KATA_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(S) % 16 != 0) return KATA_ERR_INVALID_ARGUMENT;
  if (BH > 0x7fffffffLL) return KATA_ERR_UNSUPPORTED;
  DecodeRun run{dtype, DecodeLaunch{q, k, v, S, z, y, BH, stream}};
  return dispatch_shape(d_k, d_v, feature, run);
}

size_t kata_bwd_chunked_workspace_bytes(int B, int H, int T, int d_k, int d_v, int C,
                                        kata_dtype_t dtype, kata_feature_t feature) {
  if (B < 0 || H < 0 || T < 0 || C <= 0) return 0;
  if (feature != KATA_FEATURE_PSD && feature != KATA_FEATURE_FIRST_ORDER) return 0;
  if (!supported(d_k, d_v, C, dtype, feature)) return 0;
  const int sms = device_sm_count();
  if (sms <= 0) return 0;
  const long long BH = (long long)B * H;
  const Split sp = segment_split(BH, T, C, sms, false);
  return bwd_layout(BH, T, (int)kata_state_dim(d_k, feature), d_v, sp,
                    bwd_tc_shape(d_k, d_v, C, dtype, feature), sms)
      .total();
}

kata_status_t kata_bwd_chunked(const void *q, const void *k, const void *v,
                               const void *dout, void *dq, void *dk, void *dv, int B, int H,
                               int T, int d_k, int d_v, int C, kata_dtype_t dtype,
                               kata_feature_t feature, void *workspace, size_t workspace_bytes,
                               kata_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B < 0 || H < 0 || T < 0 || C <= 0) return KATA_ERR_INVALID_ARGUMENT;
  if (!supported(d_k, d_v, C, dtype, feature)) return KATA_ERR_UNSUPPORTED;
  if (feature != KATA_FEATURE_PSD && feature != KATA_FEATURE_FIRST_ORDER) return KATA_ERR_UNSUPPORTED;
  if (!workspace) return KATA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return KATA_ERR_WORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return KATA_ERR_CUDA;
  const long long BH = (long long)B * H;
  const Split sp = segment_split(BH, T, C, sms, false);
  const bool tc_shape = bwd_tc_shape(d_k, d_v, C, dtype, feature);
  const BwdLayout lay = bwd_layout(BH, T, (int)kata_state_dim(d_k, feature), d_v, sp, tc_shape, sms);
  if (workspace_bytes < lay.total()) return KATA_ERR_WORKSPACE;
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  if (cudaMemsetAsync(ws, 0, sizeof(unsigned), stream) != cudaSuccess) return KATA_ERR_CUDA;
  if (BH == 0 || T == 0) return KATA_OK;
  if (!q || !k || !v || !dout || !dq || !dk || !dv) return KATA_ERR_INVALID_ARGUMENT;
  if (BH * (long long)sp.G > 0x7fffffffLL) return KATA_ERR_UNSUPPORTED;
  // the tensor-core pass reads its operands by TMA and writes dq rows as
  // 16-byte vectors: 16-byte aligned pointers
  bool tc = tc_shape;
  for (const void *p : {q, k, v, dout, (const void *)dq})
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) tc = false;
  int tc_G = 1, tc_seg_len = T;
  if (tc) bwd_tc_split(BH, T, sms, &tc_G, &tc_seg_len);
  BackwardRun run{dtype,
                  BackwardLaunch{q, k, v, dout, dq, dk, dv, BH, T,
                                 reinterpret_cast<unsigned *>(ws),
                                 reinterpret_cast<float *>(ws + lay.aggS()),
                                 reinterpret_cast<float *>(ws + lay.aggR()),
                                 reinterpret_cast<float *>(ws + lay.den()),
                                 reinterpret_cast<float *>(ws + lay.c()), sp.G, sp.seg_len, stream},
                  tc, tc_G, tc_seg_len};
  return dispatch_shape(d_k, d_v, feature, run);
}

kata_status_t kata_fwd_delta(const void *q, const void *k, const void *v, const float *beta,
                             void *o, int B, int H, int T, int d_k, int d_v, kata_dtype_t dtype,
                             kata_feature_t feature, const float *S0, float *S_out,
                             void *workspace, size_t workspace_bytes, kata_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B < 0 || H < 0 || T < 0) return KATA_ERR_INVALID_ARGUMENT;
  if (feature != KATA_FEATURE_PSD || !supported(d_k, d_v, 0, dtype, feature)) return KATA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < kHeaderBytes) return KATA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return KATA_ERR_WORKSPACE;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffLL) return KATA_ERR_UNSUPPORTED;
  unsigned *status = reinterpret_cast<unsigned *>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), stream) != cudaSuccess) return KATA_ERR_CUDA;
  const int D = (int)kata_state_dim(d_k, feature);
  if (BH == 0 || T == 0) {
    const size_t sb = (size_t)BH * D * (d_v + 1) * sizeof(float);
    if (S_out && BH > 0 &&
        (S0 ? cudaMemcpyAsync(S_out, S0, sb, cudaMemcpyDeviceToDevice, stream)
            : cudaMemsetAsync(S_out, 0, sb, stream)) != cudaSuccess)
      return KATA_ERR_CUDA;
    return KATA_OK;
  }
  if (!q || !k || !v || !beta || !o) return KATA_ERR_INVALID_ARGUMENT;
  const DeltaLaunch a{q, k, v, beta, o, S0, S_out, status, BH, T, stream};
  cudaError_t e = cudaErrorNotSupported;
#define KATA_DELTA_CASE(DK, DV)                                                      \
  if (d_k == DK && d_v == DV)                                                        \
    e = dtype == KATA_DTYPE_F32 ? simt_delta<DK, DV, float>(a)                       \
                                : simt_delta<DK, DV, __nv_bfloat16>(a);
  KATA_DELTA_CASE(16, 16) KATA_DELTA_CASE(16, 32) KATA_DELTA_CASE(16, 64)
  KATA_DELTA_CASE(32, 16) KATA_DELTA_CASE(32, 32) KATA_DELTA_CASE(32, 64)
#undef KATA_DELTA_CASE
  if (e == cudaErrorNotSupported) return KATA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

kata_status_t kata_selftest_device_timeout(void *workspace, size_t workspace_bytes,
                                           kata_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!workspace || workspace_bytes < kHeaderBytes) return KATA_ERR_WORKSPACE;
  unsigned *status = reinterpret_cast<unsigned *>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), stream) != cudaSuccess) return KATA_ERR_CUDA;
  return selftest_wait_timeout(status, stream) == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

kata_status_t kata_workspace_status(const void *workspace, kata_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!workspace) return KATA_ERR_WORKSPACE;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return KATA_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KATA_ERR_CUDA;
  if (word & kStatusDeviceTimeout) return KATA_ERR_DEVICE_TIMEOUT;
  if (word & kStatusNonPositiveNormaliser) return KATA_ERR_NONPOSITIVE_NORMALISER;
  return KATA_OK;
}

}  // extern "C"
