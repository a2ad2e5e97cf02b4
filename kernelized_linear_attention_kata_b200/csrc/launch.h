// Host-side launch descriptors shared by the C ABI and the kernel files.
// Each kernel family is instantiated in its own translation unit (one per
// feature x element type) so that nvcc builds them in parallel.
#pragma once

#include <cuda_bf16.h>
#include <cuda.h>
#include <cuda_runtime.h>

namespace kata {

struct ChunkedLaunch {
  const void *q, *k, *v;
  void *o;
  long long BH;
  int T, C;
  float *S_out, *z_out;
  unsigned *status;    // device status word
  float *agg;          // per-segment increments [BH][G][D][d_v + 1]
  int G, seg_len;      // segments per head, tokens per segment
  cudaStream_t stream;
  // initial state (library layout, nullable): the state of the tokens before
  // this sequence, added to every segment's carry-in
  const float *S0 = nullptr, *z0 = nullptr;
  // only the state after the T tokens (S_out, z_out); q and o are not read
  bool state_only = false;
  int sms = 0;             // SMs of the device (the tensor-core kernels size their grids by it)
  bool sequential = false; // one segment per head (the sequential carry)
};

// Sum of the G segment increments of each head, written as the state in the
// library layout ([BH][D][d_v] and [BH][D]). The increments are in the layout
// of the kernel that wrote them: kAggLibrary [D][d_v + 1] (z last, CUDA-core
// kernels), kAggPsdTc (528 x 64 in the PSD tensor-core kernel's feature order
// and scaling, then the 32 x 32 matrix sum k k^T), kAggFoTc (65 x 65: [K|1]^T
// [V|1], minus `count_pad` padded rows from the count).
enum AggLayout : int { kAggLibrary = 0, kAggPsdTc = 1, kAggFoTc = 2 };
cudaError_t state_reduce(AggLayout layout, const float *agg, long long BH, int G, int D, int d_k,
                         int d_v, float *S_out, float *z_out, float count_pad, cudaStream_t stream);

struct QuadraticLaunch {
  const void *q, *k, *v;
  void *o;
  long long BH;
  int T;
  cudaStream_t stream;
};

// DeltaKATA forward (simt_delta.cu): q, k, v, o as the chunked forward; beta
// [BH][T] fp32 write strengths; S0 / S_out nullable [BH][D][d_v + 1] fp32
// (the state augmented with its normaliser column, library row order).
struct DeltaLaunch {
  const void *q, *k, *v;
  const float *beta;
  void *o;
  const float *S0;
  float *S_out;
  unsigned *status;
  long long BH;
  int T;
  cudaStream_t stream;
};
template <int DK, int DV, typename Tin> cudaError_t simt_delta(const DeltaLaunch &a);

struct DecodeLaunch {
  const void *q, *k, *v;
  float *S, *z;
  void *y;
  long long BH;
  cudaStream_t stream;
};

// Gradient of the chunked forward: q, k, v, dout in; dq, dk, dv out (all in
// the element type). Workspace regions: segment increments of the prefix
// state (aggS) and of the suffix state (aggR), each [BH][G][D][d_v + 1], and
// per token the normaliser d_t and c_t = -(dout_t . y_t) / d_t, [BH][T] each.
struct BackwardLaunch {
  const void *q, *k, *v, *dout;
  void *dq, *dk, *dv;
  long long BH;
  int T;
  unsigned *status;
  float *aggS, *aggR, *den, *c;
  int G, seg_len;
  cudaStream_t stream;
};

// Segments of whole `tile`-token tiles for the tensor-core kernels, no more
// of them than the caller sized the workspace for (G_req).
inline void tile_segments(int T, int tile, int G_req, int *G, int *seg_len) {
  const int ntiles = (T + tile - 1) / tile;
  int g = G_req < 1 ? 1 : G_req;
  if (g > ntiles) g = ntiles;
  if (g < 1) g = 1;
  const int per = (ntiles + g - 1) / g;
  *G = per > 0 ? (ntiles + per - 1) / per : 1;
  *seg_len = per * tile;
}

// Tensor-core kernels (bf16 only). The chunked kernels' *_supported
// predicates decide, from the shape and the pointers' alignment alone,
// whether a request runs on them; tc_quadratic returns cudaErrorNotSupported,
// having launched nothing, for the shapes it does not take. Once a kernel
// has accepted a request it either launches or fails: no fallback.
cudaError_t tc_quadratic(const QuadraticLaunch &a, int d_k, int d_v, int feature);
bool tc_chunked_supported(const ChunkedLaunch &a, int d_k, int d_v, int C, int feature);
cudaError_t tc_chunked(const ChunkedLaunch &a);
size_t tc_chunked_agg_floats();   // floats of one segment increment
// Tensor-core chunked forward of the two-factor variants (kMg2, kSg2; bf16,
// d_k = 32, d_v = 64, C in {64, 128}; not the state-only call): G segments
// of seg_len tokens (whole 128-token chunks), one increment per segment.
bool var_tc_supported(const ChunkedLaunch &a, int d_k, int d_v, int C, int feature);
void var_tc_layout(long long BH, int T, int sms, bool sequential, int *G, int *seg_len);
cudaError_t var_tc(const ChunkedLaunch &a, int feature);
// Tensor-core gradient with respect to q of the PSD chunked forward (bf16,
// d_k = 32, d_v = 64): the forward's increments of segments 0 .. G-2 into
// aggS (PSD tensor-core layout, G per head), then dq and, per token, d_t and
// c_t (a.den, a.c) for the suffix pass; G segments of seg_len tokens.
cudaError_t tc_bwd_dq(const BackwardLaunch &a, float *aggS, int G, int seg_len);
// Tensor-core gradients with respect to k and v (same shapes), from a.den and
// a.c of the dq pass: the suffix increments of segments 1 .. G-1 into aggR
// (same layout), then each segment's chunks in reverse order.
cudaError_t tc_bwd_dkdv(const BackwardLaunch &a, float *aggR, int G, int seg_len);
// Segment increments of the PSD tensor-core layout (d_k = 32, d_v = 64 bf16):
// segments 0 .. G_inc - 1 of G_total (seg_len tokens each, whole 128-token
// chunks) into agg[bh][g], G_total increments per head.
cudaError_t psd_tc_increments(const void *k, const void *v, float *agg, unsigned *status,
                              long long BH, int T, int G_inc, int G_total, int seg_len,
                              cudaStream_t stream);
// The backward's suffix increments on the same kernel: segments 1 .. G-1,
// R' = sum m_f phi(q_t) dout_t^T / d_t and Rq = Q^T diag(c) Q into aggR[bh][g]
// (the increment layout), from d_t and c_t ([BH][T] fp32).
cudaError_t psd_tc_suffix_increments(const void *q, const void *dout, const float *den,
                                     const float *c, float *aggR, unsigned *status, long long BH,
                                     int T, int G, int seg_len, cudaStream_t stream);
// The PSD tensor-core forward's split: G segments of seg_len tokens per head,
// each segment's increment computed as P pieces (G * P increments per head in
// the workspace).
void tc_chunked_layout(long long BH, int T, int sms, bool sequential, int *G, int *seg_len, int *P);

bool fo_tc_supported(const ChunkedLaunch &a, int d_k, int d_v, int C, int feature);
cudaError_t fo_tc(const ChunkedLaunch &a);
// One block that waits on a barrier nothing completes, until the bounded
// wait's limit; leaves kStatusDeviceTimeout in *status (selftest.cu).
cudaError_t selftest_wait_timeout(unsigned *status, cudaStream_t stream);
size_t fo_tc_agg_floats();        // floats of one segment increment

template <int DK, int DV, int FEAT, typename Tin> cudaError_t simt_chunked(const ChunkedLaunch &a);
template <int DK, int DV, int FEAT, typename Tin> cudaError_t simt_quadratic(const QuadraticLaunch &a);
template <int DK, int DV, int FEAT, typename Tin> cudaError_t simt_decode(const DecodeLaunch &a);
template <int DK, int DV, int FEAT, typename Tin> cudaError_t simt_backward(const BackwardLaunch &a);
template <int DK, int DV, int FEAT, typename Tin>
cudaError_t simt_backward_dkdv(const BackwardLaunch &a);

}  // namespace kata
