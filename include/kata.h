/*
 * kata.h -- C ABI of the KATA causal linear-attention library (CUDA, sm_100a).
 *
 * The method (Kernelized Linear Attention, "Kernelized Linear Attention:
 * Breaking the Capacity Wall with Symmetric Cones", arXiv 2607.17419v1):
 *
 *   y_t = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts,
 *   w_ts = <phi(q_t), phi(k_s)>.
 *
 * Normalised linear attention as an RNN with a fixed-size state ("線形注意"
 * wiki page, definition); the rank-one PSD feature psi(u) = u u^T, whose
 * weight is <q_t, k_s>^2 >= 0 (gist.science explainer, technical summary
 * 2.2); the normaliser read as a convex output gate (same explainer, 2.1);
 * the exact O(T) chunked-state form with an associative scan across chunks
 * (same explainer, 2.3, and the arXiv abstract).
 *
 * Conventions common to every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    allocates no device memory; scratch is the caller's workspace.
 *  - Layouts: q, k are [B, H, T, d_k]; v, o are [B, H, T, d_v]; row-major and
 *    contiguous, element type `dtype` (o has the same type as q). States are
 *    always fp32.
 *  - Causal mask includes the diagonal (s <= t): y_1 = v_1.
 *  - No temperature or 1/sqrt(d) scale is applied: pass q, k as they should
 *    enter the inner product.
 *  - Packed state layout, shape [B, H, D, d_v] for S and [B, H, D] for z:
 *      PSD         : D = d_k (d_k + 1) / 2, row r <-> pair (i, j), i <= j,
 *                    rows ordered row-major over i then j;
 *                    S[r] = sum_s k_si k_sj v_s, z[r] = sum_s k_si k_sj
 *                    (no factor 2: the readout applies the multiplicity 2
 *                    of the off-diagonal pairs on the query side).
 *      FIRST_ORDER : D = d_k + 1, row 0 is the constant feature 1, row 1 + i
 *                    is k_i; weight 1 + <q_t, k_s>.
 *      MULTI_PSD2  : D = 2 h (h + 1) / 2 with h = d_k / 2: the packed rows
 *                    (i <= j, row-major) of slice 1, then those of slice 2;
 *                    S[r] = sum_s k_si k_sj v_s with (i, j) in one slice.
 *      SUMMED_PSD2 : D = h (h + 1) / 2, row r <-> (i, j), i <= j < h;
 *                    S[r] = sum_s (k_si k_sj + k_s(h+i) k_s(h+j)) v_s.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream). Argument errors are detected on the host and returned
 *    before anything is launched. KATA_ERR_CUDA reports a launch error
 *    (cudaGetLastError) and leaves outputs undefined.
 *  - A row whose normaliser is not positive (for instance a query orthogonal
 *    to every key it sees) yields a non-finite output. kata_fwd_chunked also
 *    records this in its workspace; see kata_workspace_status.
 *  - B, H or T equal to 0 is a valid empty problem: nothing is launched for
 *    the outputs (S_out / z_out, when given, are zero-filled).
 *  - Reproducibility: the states are bitwise reproducible. The bf16
 *    tensor-core chunked forward for PSD (d_k = 32, d_v = 64) accumulates its
 *    readout from two MMA-issuing threads into one fp32 accumulator, in an
 *    order that varies from run to run, so its outputs can differ between
 *    runs in the last bf16 bit.
 *
 * Supported shapes (anything else returns KATA_ERR_UNSUPPORTED):
 *    PSD          d_k in {16, 32}
 *    FIRST_ORDER  d_k in {16, 32, 64}
 *    MULTI_PSD2, SUMMED_PSD2  d_k in {16, 32} (forward forms and the decode
 *                 step; kata_bwd_chunked takes PSD and FIRST_ORDER only)
 *    d_v in {16, 32, 64};  C in {16, 32, 64, 128};  T >= 0;
 *    T need not be a multiple of C (the last chunk is shorter).
 */
#ifndef KATA_H
#define KATA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KATA_API __attribute__((visibility("default")))
#else
#define KATA_API
#endif

/* cudaStream_t without including the CUDA headers. */
typedef struct CUstream_st *kata_stream_t;

typedef enum {
    KATA_OK = 0,
    KATA_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, ...       */
    KATA_ERR_UNSUPPORTED = 2,      /* shape / dtype / feature not built      */
    KATA_ERR_WORKSPACE = 3,        /* workspace missing, too small, unaligned */
    KATA_ERR_CUDA = 4,             /* a CUDA call or launch failed           */
    KATA_ERR_NONPOSITIVE_NORMALISER = 5, /* device: some row had den <= 0    */
    KATA_ERR_DEVICE_TIMEOUT = 6    /* device: a bounded wait inside a kernel
                                      gave up (a library defect); outputs of
                                      that call are undefined               */
} kata_status_t;

typedef enum { KATA_DTYPE_F32 = 0, KATA_DTYPE_BF16 = 1 } kata_dtype_t;

/*
 * Feature maps. The two-factor variants are the KATA-Mg and KATA-Sigma-g of
 * the explainer (section 2.3, g = 2), which names them without a
 * construction; the library reads the factors of a head vector x in R^d_k
 * as its two halves x_1, x_2 in R^(d_k / 2):
 *   KATA_FEATURE_MULTI_PSD2   phi(x) = [x_1 x_1^T, x_2 x_2^T] (KATA-Mg, g = 2),
 *                             weight <q_1,k_1>^2 + <q_2,k_2>^2;
 *   KATA_FEATURE_SUMMED_PSD2  Psi(x) = x_1 x_1^T + x_2 x_2^T (KATA-Sigma-g,
 *                             g = 2), weight sum_{a,b} <q_a,k_b>^2.
 */
typedef enum {
    KATA_FEATURE_PSD = 0,
    KATA_FEATURE_FIRST_ORDER = 1,
    KATA_FEATURE_MULTI_PSD2 = 2,
    KATA_FEATURE_SUMMED_PSD2 = 3
} kata_feature_t;

/* Kernel family a chunked-forward request runs on. */
typedef enum {
    KATA_PATH_NONE = 0,             /* empty problem: nothing is launched      */
    KATA_PATH_TENSOR_CORE_PSD = 1,  /* tcgen05/TMEM kernels, bf16 PSD,
                                       d_k = 32, d_v = 64, C in {64, 128}     */
    KATA_PATH_TENSOR_CORE_FIRST_ORDER = 2, /* tcgen05/TMEM kernels, bf16
                                       first-order, d_k = d_v = 64,
                                       C in {64, 128}                          */
    KATA_PATH_CUDA_CORE = 3,        /* fp32 FFMA kernels: the fp32 path and
                                       every other supported shape            */
    KATA_PATH_TENSOR_CORE_MULTI_FACTOR = 4 /* tcgen05/TMEM kernels, bf16
                                       MULTI_PSD2 / SUMMED_PSD2, d_k = 32,
                                       d_v = 64, C in {64, 128} (the
                                       state-only call kata_chunked_state
                                       runs them on the CUDA cores)           */
} kata_path_t;

/* How kata_fwd_chunked will run a problem (see kata_fwd_chunked_plan). */
typedef struct {
    kata_path_t path;   /* kernel family                                      */
    int segments;       /* segments per (b, h) of the parallel carry (the
                           scan across chunks): 1 = sequential carry          */
    int segment_tokens; /* tokens per segment (a multiple of the chunk the
                           kernels compute with); segment g starts at token
                           g * segment_tokens                                 */
    int chunk_tokens;   /* chunk the kernels compute with: 128 on the tensor
                           cores for C in {64, 128} (the chunked form is exact
                           for any C, so C only schedules the work), else C   */
} kata_plan_t;

/* Library version, major * 10000 + minor * 100 + patch. */
KATA_API int kata_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
KATA_API const char *kata_status_string(kata_status_t status);

/* D, the number of state rows: d_k (d_k + 1) / 2 for PSD, d_k + 1 for
 * FIRST_ORDER, h (h + 1) for MULTI_PSD2 and h (h + 1) / 2 for SUMMED_PSD2
 * (h = d_k / 2); 0 for an unknown feature, d_k <= 0, or an odd d_k with a
 * two-factor feature. */
KATA_API size_t kata_state_dim(int d_k, kata_feature_t feature);

/*
 * Workspace bytes kata_fwd_chunked needs for this problem on the CURRENT
 * device (the segment split depends on its SM count). Returns 0 for a shape
 * the library does not support. The workspace must be 256-byte aligned and
 * must not be used by two calls that run concurrently.
 */
KATA_API size_t kata_fwd_chunked_workspace_bytes(int B, int H, int T, int d_k, int d_v, int C,
                                        kata_dtype_t dtype, kata_feature_t feature);

/*
 * The plan kata_fwd_chunked (sequential = 0) or kata_fwd_chunked_sequential
 * (sequential = 1) follows for this problem on the CURRENT device, with q, k,
 * v, o (and S_out, when given) 16-byte aligned as every cudaMalloc'd buffer
 * is: which kernel family runs and how the sequence is cut into segments
 * for the parallel carry. Nothing is launched.
 *   out      host pointer, written on KATA_OK.
 * Returns KATA_ERR_UNSUPPORTED for a shape the library does not build,
 * KATA_ERR_INVALID_ARGUMENT for a negative size or a NULL `out`, and
 * KATA_ERR_CUDA when the device cannot be queried. A request the plan sends
 * to the tensor cores never falls back to the CUDA cores: if the
 * tensor-core setup fails, the call returns KATA_ERR_CUDA.
 */
KATA_API kata_status_t kata_fwd_chunked_plan(int B, int H, int T, int d_k, int d_v, int C,
                                             kata_dtype_t dtype, kata_feature_t feature,
                                             int sequential, kata_plan_t *out);

/*
 * Exact O(T) chunked-state causal forward (arXiv abstract: "exact O(T)
 * chunked-state form"; explainer 2.3: chunk parallelism with an associative
 * scan across chunks).
 *
 * For each chunk c of C tokens:
 *   A     = (Q_c K_c^T)^2 masked to s <= t          (PSD; 1 + Q_c K_c^T for
 *                                                   FIRST_ORDER)
 *   Y_c   = (A V_c + phi_q(Q_c) S_c) / (A 1 + phi_q(Q_c) z_c)
 *   S_c+1 = S_c + phi(K_c)^T V_c,  z_c+1 = z_c + phi(K_c)^T 1.
 * The carry S_c is an exclusive scan of the per-chunk increments, computed
 * per segment of chunks so the sequence is processed in parallel.
 *
 *   q, k, v, o         device, layouts above.
 *   S_out, z_out       optional (may be NULL, independently): the final state
 *                      after all T tokens, [B, H, D, d_v] and [B, H, D] fp32.
 *   workspace          device, >= kata_fwd_chunked_workspace_bytes(...),
 *                      256-byte aligned; contents on entry are ignored. On
 *                      return (after the stream has run) it holds the device
 *                      status word read by kata_workspace_status.
 * Returns KATA_OK when the work was launched.
 */
KATA_API kata_status_t kata_fwd_chunked(const void *q, const void *k, const void *v, void *o,
                               int B, int H, int T, int d_k, int d_v, int C,
                               kata_dtype_t dtype, kata_feature_t feature,
                               float *S_out, float *z_out,
                               void *workspace, size_t workspace_bytes,
                               kata_stream_t stream);

/*
 * The same forward with a SEQUENTIAL inter-chunk carry: one thread block per
 * (b, h) walks its chunks in order (recurrence depth N_C = ceil(T/C)). This
 * is the matched sequential linear-attention baseline that the arXiv
 * abstract compares the associative scan against. Same arguments and
 * results as kata_fwd_chunked; needs only the status header of the
 * workspace (kata_fwd_chunked_workspace_bytes is always enough).
 */
KATA_API kata_status_t kata_fwd_chunked_sequential(const void *q, const void *k, const void *v, void *o,
                                          int B, int H, int T, int d_k, int d_v, int C,
                                          kata_dtype_t dtype, kata_feature_t feature,
                                          float *S_out, float *z_out,
                                          void *workspace, size_t workspace_bytes,
                                          kata_stream_t stream);

/*
 * The same forward starting from a given state instead of zero: the carry
 * into every chunk is S0 + (the increments of the earlier chunks), i.e. the
 * sequence continues one whose state after its last token is (S0, z0). This
 * is how a sequence cut into slices (one per GPU) is processed: slice r
 * starts from the sum of the states of slices 0 .. r-1 (the scan across
 * chunks, explainer 2.3, taken one level up).
 *   S0, z0             device fp32 [B, H, D, d_v] and [B, H, D], library
 *                      layout (read only); either may be NULL (zero).
 * Everything else as kata_fwd_chunked; S_out / z_out include S0 / z0, and
 * with T = 0 they are copies of S0 / z0.
 */
KATA_API kata_status_t kata_fwd_chunked_from_state(const void *q, const void *k, const void *v,
                                                   void *o, int B, int H, int T, int d_k, int d_v,
                                                   int C, kata_dtype_t dtype, kata_feature_t feature,
                                                   const float *S0, const float *z0,
                                                   float *S_out, float *z_out,
                                                   void *workspace, size_t workspace_bytes,
                                                   kata_stream_t stream);

/*
 * Only the state after the T tokens: S_out = sum_t phi(k_t) v_t^T and
 * z_out = sum_t phi(k_t) (library layout), without computing outputs. The
 * state is a sum over tokens, so it is computed as per-segment increments
 * reduced per head; a sequence slice's state is what the slices after it
 * need as their starting state. q and o are not inputs. Same workspace as
 * kata_fwd_chunked (kata_fwd_chunked_workspace_bytes is enough).
 */
KATA_API kata_status_t kata_chunked_state(const void *k, const void *v, int B, int H, int T,
                                          int d_k, int d_v, int C, kata_dtype_t dtype,
                                          kata_feature_t feature, float *S_out, float *z_out,
                                          void *workspace, size_t workspace_bytes,
                                          kata_stream_t stream);

/*
 * kata_fwd_chunked without a caller-provided workspace, for callers that
 * cannot allocate device memory (for example a host application whose device
 * memory belongs entirely to another runtime's pool, or latency-critical code
 * that must not cause the device-wide synchronisation of cudaMalloc /
 * cudaFree). The paper has no counterpart: this is a library convenience.
 *
 * Scratch is one fixed device array of KATA_NOALLOC_SCRATCH_BYTES (32 MiB)
 * inside the library, held by every GPU that loads it until the process
 * exits. Same arguments and results as kata_fwd_chunked minus the workspace.
 *  - Returns KATA_ERR_WORKSPACE, before launching anything, when the problem
 *    needs more scratch than the array holds, i.e. when
 *    kata_fwd_chunked_workspace_bytes(...) > KATA_NOALLOC_SCRATCH_BYTES.
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress), so a cudaDeviceReset or a new primary context
 *    leaves no stale address behind. The first call on a device may load the
 *    library's device code: make it before any stream capture.
 *  - All calls share the array, which keeps the last call's contents (each
 *    call clears the status word it needs to start at zero). Calls whose work
 *    overlaps on the GPU (different streams, different host threads) race on
 *    it: serialise them.
 *  - The device status word is not readable from outside; rows with a
 *    non-positive normaliser give non-finite outputs as usual.
 */
#define KATA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
KATA_API kata_status_t kata_fwd_chunked_noalloc(const void *q, const void *k, const void *v,
                                                void *o, int B, int H, int T, int d_k, int d_v,
                                                int C, kata_dtype_t dtype, kata_feature_t feature,
                                                float *S_out, float *z_out, kata_stream_t stream);

/*
 * Flash-attention-style quadratic causal forward (explainer 2.3, operating
 * point 1: O(T^2), no state is materialised). For each query block the key
 * blocks up to the diagonal are visited; P = (Q K^T)^2 (or 1 + Q K^T) masked,
 * O += P V, l += rowsum(P); finally O / l. No exponential and no running
 * maximum are needed because the weights are polynomial and nonnegative.
 * Same tensor layouts; no workspace.
 */
KATA_API kata_status_t kata_fwd_quadratic(const void *q, const void *k, const void *v, void *o,
                                 int B, int H, int T, int d_k, int d_v,
                                 kata_dtype_t dtype, kata_feature_t feature,
                                 kata_stream_t stream);

/*
 * One-token recurrent decode step ("線形注意" definition: constant-time
 * recurrent inference with a fixed-size state), batched over B x H heads:
 *   S += phi(k) v^T,  z += phi(k),  y = phi_q(q)^T S / phi_q(q)^T z
 * (update first, then read, so the current token is included exactly as in
 * the forward).
 *   q, k   device [B, H, d_k], dtype;  v, y device [B, H, d_v], dtype.
 *   S, z   device fp32 [B, H, D, d_v] and [B, H, D], read and written in
 *          place (packed layout above).
 */
KATA_API kata_status_t kata_decode_step(const void *q, const void *k, const void *v,
                               float *S, float *z, void *y,
                               int B, int H, int d_k, int d_v,
                               kata_dtype_t dtype, kata_feature_t feature,
                               kata_stream_t stream);

/*
 * Workspace bytes kata_bwd_chunked needs for this problem on the CURRENT
 * device; 0 for an unsupported shape. Same alignment and exclusivity rules as
 * the forward's workspace.
 */
KATA_API size_t kata_bwd_chunked_workspace_bytes(int B, int H, int T, int d_k, int d_v, int C,
                                                 kata_dtype_t dtype, kata_feature_t feature);

/*
 * Gradient of the causal forward: given dout = dL/dy for the output
 * y of kata_fwd_chunked(q, k, v), writes dq = dL/dq, dk = dL/dk, dv = dL/dv.
 * The pages pre-train language models on these kernels (arXiv abstract;
 * explainer sections 3 and 4) without printing the backward; this is the
 * chain rule of the definition above. With d_t = sum_{s<=t} w_ts,
 *   g_t = dout_t / d_t,   c_t = -(dout_t . y_t) / d_t,
 *   e_ts = g_t . v_s + c_t                        (dL/dw_ts, s <= t)
 *   dv_s = sum_{t>=s} w_ts g_t
 *   dq_t = sum_{s<=t} e_ts dw_ts/dq_t,   dk_s = sum_{t>=s} e_ts dw_ts/dk_s
 * (dw/dq = 2 <q,k> k, dw/dk = 2 <q,k> q for PSD; k and q for FIRST_ORDER),
 * evaluated in the exact chunked form: each sum is a dense block inside a
 * chunk plus a state carried from the other chunks (the forward's prefix
 * state for dq, a suffix state R = sum phi_q(q_t) g_t^T, r = sum phi_q(q_t)
 * c_t carried backwards for dk and dv), both through the segment scan. The
 * forward's output is not an input: d_t and dout_t . y_t are recomputed in
 * fp32 (a stored bf16 y would enter c_t with its rounding, which the
 * cancellation in e_ts amplifies by 1 / d_t).
 *
 *   q, k, v            device, the forward's inputs (layouts above).
 *   dout               device [B, H, T, d_v], dtype.
 *   dq, dk / dv        device [B, H, T, d_k] / [B, H, T, d_v], dtype,
 *                      written (may not alias the inputs).
 *   workspace          device, >= kata_bwd_chunked_workspace_bytes(...),
 *                      256-byte aligned, contents on entry ignored; holds the
 *                      status word afterwards (kata_workspace_status reports
 *                      a non-positive normaliser as for the forward).
 * bf16 PSD with d_k = 32, d_v = 64, C in {64, 128} and 16-byte aligned
 * pointers runs on the tensor cores (bf16 MMA operands: the inputs, the
 * state snapshots and the intra-chunk gradient blocks; fp32 accumulation;
 * the same bf16 tolerance as the forward). Every other case computes in
 * fp32 on the CUDA cores. Returns KATA_OK when the work was launched; B, H
 * or T = 0 launches nothing.
 */
KATA_API kata_status_t kata_bwd_chunked(const void *q, const void *k, const void *v,
                                        const void *dout, void *dq, void *dk, void *dv,
                                        int B, int H, int T, int d_k, int d_v, int C,
                                        kata_dtype_t dtype, kata_feature_t feature,
                                        void *workspace, size_t workspace_bytes,
                                        kata_stream_t stream);

/*
 * DeltaKATA forward: the delta-rule state update that the KATA explainer
 * (section 4, "DeltaKATA") credits with correcting stale bindings at
 * repeated keys. The pages give no rule; the library reads it as the delta
 * rule on the state augmented with its normaliser, S' = [S | z] (D rows,
 * d_v + 1 columns), with a per-token write strength beta_t in (0, 1]:
 *   S'_t = S'_(t-1) + beta_t phi(k_t) ([v_t, 1] - phi_q(k_t)^T S'_(t-1)),
 *   y_t  = (phi_q(q_t)^T S'_t)[:d_v] / (phi_q(q_t)^T S'_t)[d_v]
 * (phi the key-side, phi_q the query-side packed PSD feature; the current
 * token's write is read, as in the additive forward). For a unit key
 * phi_q(k) . phi(k) = |k|^4 = 1, so beta = 1 overwrites the binding stored
 * at a repeated key; keys orthogonal in feature space give the additive
 * state with weights beta. Computed in chunks of 32 tokens (an exact form:
 * a triangular solve per chunk), one thread block per (b, h), fp32 on the
 * CUDA cores for both element types.
 *   q, k, v, o         as kata_fwd_chunked.
 *   beta               device fp32 [B, H, T], entries in (0, 1] (not
 *                      checked on the device; other values give the rule's
 *                      arithmetic without its meaning).
 *   S0                 optional device fp32 [B, H, D, d_v + 1]: the state
 *                      before the first token (library PSD row order, the
 *                      normaliser in column d_v); NULL is zero.
 *   S_out              optional device fp32 [B, H, D, d_v + 1]: the state
 *                      after the last token.
 *   workspace          device, >= 256 bytes, 256-byte aligned: the status
 *                      word (kata_workspace_status reports a non-positive
 *                      normaliser as for the forward).
 * Feature: PSD with d_k in {16, 32}, d_v in {16, 32, 64}; anything else
 * returns KATA_ERR_UNSUPPORTED.
 */
KATA_API kata_status_t kata_fwd_delta(const void *q, const void *k, const void *v,
                                      const float *beta, void *o, int B, int H, int T, int d_k,
                                      int d_v, kata_dtype_t dtype, kata_feature_t feature,
                                      const float *S0, float *S_out, void *workspace,
                                      size_t workspace_bytes, kata_stream_t stream);

/*
 * Synchronises `stream`, then reads the status word a kata_fwd_chunked(...),
 * kata_fwd_chunked_sequential(...), kata_fwd_chunked_from_state(...),
 * kata_chunked_state(...), kata_bwd_chunked(...), kata_fwd_delta(...) or
 * kata_selftest_device_timeout(...) call left in `workspace`: KATA_OK, or
 * KATA_ERR_DEVICE_TIMEOUT if a bounded wait inside a kernel gave up (the
 * kernel returned early, its outputs are undefined, the context is usable),
 * KATA_ERR_NONPOSITIVE_NORMALISER if any row had a normaliser <= 0, or
 * KATA_ERR_CUDA if the synchronisation or the copy failed.
 */
KATA_API kata_status_t kata_workspace_status(const void *workspace, kata_stream_t stream);

/*
 * Self-test of the device-timeout path (failure detection without a fault).
 * Launches one thread block that waits on an mbarrier nothing completes. The
 * bounded wait the tensor-core kernels use gives up after 2 s of GPU time;
 * the block then frees its tensor memory and records a device timeout in the
 * status word, as a forward kernel does when one of its waits runs out. Once
 * the stream has run, kata_workspace_status(workspace) returns
 * KATA_ERR_DEVICE_TIMEOUT, and the CUDA context remains usable.
 *   workspace   device, >= 256 bytes (a status header); the status word is
 *               reset on `stream` before the launch.
 * Returns KATA_OK when launched; KATA_ERR_WORKSPACE for a null or short
 * workspace (checked on the host before anything is launched); KATA_ERR_CUDA
 * if the reset or the launch failed. Needs an sm_100a device.
 */
KATA_API kata_status_t kata_selftest_device_timeout(void *workspace, size_t workspace_bytes,
                                                    kata_stream_t stream);

/*
 * Optional per-kernel device timing (CUDA events), for benchmarks. Not part
 * of the method. kata_profile_enable(1) clears the counters and starts
 * bracketing every kernel the library launches with two events recorded on
 * the launch's stream; kata_profile_enable(0) stops. kata_profile_count and
 * kata_profile_get synchronise on the recorded events, then report, per
 * kernel name (static storage), the number of launches and their summed
 * device time in milliseconds. Use from one host thread.
 */
KATA_API kata_status_t kata_profile_enable(int enable);
KATA_API int kata_profile_count(void);
KATA_API kata_status_t kata_profile_get(int index, const char **name, long long *launches,
                                        double *total_ms);

#ifdef __cplusplus
}
#endif

#endif /* KATA_H */
