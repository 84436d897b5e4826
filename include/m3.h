/*
 * m3.h -- C ABI of the B200 Mamba-3 SSM layer library (libm3.so).
 *
 * The layer is the selective state-space recurrence of "Mamba-3: Improved
 * Sequence Modeling using State Space Principles":
 *   - exponential-trapezoidal discretisation (PaperWeekly page section 2.2,
 *     "generalized trapezoidal rule"; wmrh.cn blog section 2.1):
 *       h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}^T + gamma_t B_t x_t^T,
 *       alpha_t = exp(dt_t A_t), gamma_t = lam_t dt_t,
 *       beta_t = (1 - lam_t) dt_t alpha_t;
 *   - complex-valued transition applied as data-dependent RoPE (section 2.1,
 *     section 2.2; arXiv 2603.15569 abstract): the state rows are pairs
 *     (2k, 2k+1); alpha_t (and the beta_t term) also rotate pair k by the angle
 *     dt_t theta_{t,k}; equivalently B and C are rotated by the cumulative
 *     angles;
 *   - MIMO (section 2.3): B_t x_t^T is the rank-R product B_t (N x R) X_t^T (R x P);
 *   - output y_t = C_t^T h_t (R x P per token and head), the real part of the
 *     complex state read by C (section 2.1).
 *
 * Calls: the chunked prefill scan (m3_scan_fwd; its packed variable-length
 * form m3_scan_fwd_varlen; m3_scan_fwd_noalloc without a workspace argument;
 * m3_scan_state for the final state only), the single-token decode step
 * (m3_decode_step), the backward pass (m3_scan_bwd, m3_scan_bwd_varlen), the
 * B / C projection prep (m3_bc_prep), the block projections around the
 * layer (m3_linear, m3_mimo_up, m3_mimo_down_gate), the pieces of a sequence split across
 * ranks (m3_segment_totals, m3_state_fold), and sizing, planning and status
 * (m3_*_workspace_size, m3_scan_plan, m3_check_shape, m3_stream_status,
 * m3_status_string, m3_version).
 *
 * Conventions for every call:
 *   - Every data pointer is a DEVICE pointer owned by the caller.  The library
 *     never allocates, frees or retains memory; it writes only the outputs
 *     named below (and the caller's workspace).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are detected on the host before any
 *     launch and returned synchronously; nothing is launched then.  Launch
 *     failures return M3_ERR_CUDA.  Faults inside kernels surface through
 *     m3_stream_status().
 *   - All tensors are row-major and contiguous:
 *       x, y              [batch][seqlen][nheads][rank][headdim]   io dtype
 *       B, C              [batch][seqlen][ngroups][rank][dstate]   io dtype
 *       dt, A, lam        [batch][seqlen][nheads]                  fp32
 *       theta             [batch][seqlen][ngroups][dstate/2]       fp32
 *                         ([batch][seqlen][nheads][dstate/2] with M3_FLAG_THETA_PER_HEAD)
 *       h0, final_state   [batch][nheads][dstate][headdim]         fp32
 *       B_prev            [batch][ngroups][rank][dstate]           io dtype
 *       x_prev            [batch][nheads][rank][headdim]           io dtype
 *     Head h reads group g = h / (nheads / ngroups).  theta is an angle RATE:
 *     the step angle of pair k is dt * theta_k.  State pairs are adjacent rows
 *     (2k, 2k+1); the rotation is [[cos, -sin], [sin, cos]].
 *   - io dtype tensors (x, y, B, C, B_prev, x_prev), fp32 state tensors and
 *     theta must be 16-byte aligned; dt, A, lam 4-byte aligned.
 *
 * Supported shapes (anything else returns M3_ERR_UNSUPPORTED):
 *   dstate N in {16, 32, 64, 128, 256}; headdim P in {16, 32, 64, 128};
 *   N * P <= 16384; rank R in {1, 2, 4, 8}; chunk in {16, 32, 64};
 *   batch <= 65535, nheads <= 65535.
 */
#ifndef M3_H_
#define M3_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define M3_API __declspec(dllexport)
#else
#define M3_API __attribute__((visibility("default")))
#endif

/* Same underlying type as cudaStream_t / CUstream. */
struct CUstream_st;
typedef struct CUstream_st* m3_stream_t;

/* Element type of x, y, B, C, B_prev, x_prev. */
typedef enum { M3_F32 = 0, M3_BF16 = 1 } m3_dtype;

typedef enum {
  M3_OK = 0,
  M3_ERR_INVALID_ARGUMENT = -1, /* null required pointer, bad extent, bad dtype */
  M3_ERR_UNSUPPORTED = -2,      /* valid but outside the supported shape set   */
  M3_ERR_ALIGNMENT = -3,        /* a pointer violates its alignment rule       */
  M3_ERR_WORKSPACE = -4,        /* workspace null, misaligned or too small     */
  M3_ERR_CUDA = -5,             /* a CUDA launch or runtime call failed        */
  M3_ERR_TIMEOUT = -6,          /* a bounded device-side wait gave up          */
  M3_ERR_BOUNDS = -7            /* bounds-checked builds only: a kernel formed
                                   an index outside its tensor and skipped the
                                   access (a library defect, never the caller's) */
} m3_status;

/* Flags (m3_shape.flags). */
#define M3_FLAG_SIMT 1u /* force the CUDA-core fp32 scan (no tensor cores) */
/* Diagnostic for the failure path of m3_scan_fwd on the tensor-core path:
 * every CTA first waits, with a 1 ms limit, on an mbarrier that nothing
 * completes, so the call computes nothing and the next m3_stream_status
 * returns M3_ERR_TIMEOUT.  Lets a test check that a bounded device-side wait
 * ends, reports its status and leaves the context usable.  Ignored by the
 * CUDA-core path and by m3_decode_step. */
#define M3_FLAG_TEST_TIMEOUT 2u
/* theta holds one angle-rate vector per head: [b][L][H][N/2] for the scan,
 * [b][H][N/2] for the decode step (default: per group, like B and C). */
#define M3_FLAG_THETA_PER_HEAD 4u
/* m3_scan_bwd, m3_scan_bwd_varlen: dy is fp32 whatever the io dtype (a bf16
 * layer trained with fp32 output gradients keeps them unrounded).  Ignored
 * by every other call. */
#define M3_FLAG_DY_F32 8u

typedef struct {
  int64_t batch;    /* b >= 1                                   */
  int64_t seqlen;   /* L >= 0 (ignored by m3_decode_step)       */
  int64_t nheads;   /* H >= 1                                   */
  int64_t ngroups;  /* G >= 1, H % G == 0 (B, C, theta groups)  */
  int64_t headdim;  /* P                                        */
  int64_t dstate;   /* N (even)                                 */
  int64_t rank;     /* R (1 = SISO)                             */
  int64_t chunk;    /* Q, scan chunk length (ignored by decode) */
  int32_t io_dtype; /* m3_dtype                                 */
  uint32_t flags;   /* M3_FLAG_*; 0 = automatic choice          */
} m3_shape;

/* Library version string (static storage). */
M3_API const char* m3_version(void);

/* Human-readable name of a status code (static storage). */
M3_API const char* m3_status_string(int status);

/* Checks a shape against the rules above without touching the GPU.
 * Returns M3_OK, M3_ERR_INVALID_ARGUMENT or M3_ERR_UNSUPPORTED. */
M3_API int m3_check_shape(const m3_shape* shape);

/* Workspace bytes that m3_scan_fwd needs for `shape` (0 when L == 0).
 * Host-only; writes *bytes.  Returns M3_OK or the m3_check_shape error. */
M3_API int m3_scan_workspace_size(const m3_shape* shape, size_t* bytes);

/* The same query as a single value: the workspace bytes m3_scan_fwd needs for
 * `shape` (0 when L == 0 or when the shape needs none), or SIZE_MAX when the
 * shape fails m3_check_shape (the status itself is not reported; call
 * m3_check_shape for it).  Host-only, never touches the GPU. */
M3_API size_t m3_scan_workspace_bytes(const m3_shape* shape);

/* How m3_scan_fwd will run `shape` (host-only): *tensor_core = 1 for the
 * tcgen05 path (bf16 io, N = 128, P = 64, chunk * rank in {64, 128, 256},
 * M3_FLAG_SIMT clear), 0 for the CUDA-core fp32 path; *segments = the most
 * pieces any (batch, head) sequence is cut into (tensor-core path; 1
 * otherwise; a plan may cut only the sequences that would run in a last,
 * partly empty wave of CTAs);
 * *launches = kernel launches per call (0 when seqlen == 0).  Any output
 * pointer may be NULL.  Returns M3_OK or the m3_check_shape error. */
M3_API int m3_scan_plan(const m3_shape* shape, int* tensor_core, int64_t* segments,
                        int* launches);

/* Chunked prefill scan over a whole sequence batch: the recurrence above for
 * every (batch, head), y_t = C_t^T h_t for every token, and the state after
 * the last token.
 *
 * The scan splits each sequence into chunks of `chunk` tokens (the last chunk
 * may be shorter).  Within a chunk it evaluates the equivalent masked
 * quadratic form (cumulative decay times the width-2 trapezoid convolution,
 * PaperWeekly page section 2.2, Figure 2); across chunks it passes the state.
 *
 *   h0          initial state h_{-1}, or NULL for zero.
 *   B_prev,
 *   x_prev      the token before the sequence (its B and x, not their
 *               product): the left endpoint of the first step.  Both NULL for
 *               none (zero), or both non-NULL.  Together with h0 this continues
 *               a previous scan exactly.
 *   y           output [b][L][H][R][P] in the io dtype (rounded to nearest).
 *   final_state output h_{L-1} [b][H][N][P] fp32, or NULL to skip.  With
 *               L == 0 it receives h0 (or zeros).
 *   workspace   device scratch of at least m3_scan_workspace_size() bytes,
 *               256-byte aligned; its contents on entry do not matter and are
 *               undefined on return.  It must not be shared by scans in flight
 *               at the same time.
 * No input may alias an output.  Returns M3_OK when the work was enqueued. */
M3_API int m3_scan_fwd(const m3_shape* shape, const void* x, const float* dt,
                       const float* A, const float* lam, const float* theta,
                       const void* B, const void* C, const float* h0,
                       const void* B_prev, const void* x_prev, void* y,
                       float* final_state, void* workspace,
                       size_t workspace_bytes, m3_stream_t stream);

/* One decode step for every (batch, head): reads the fp32 state once, applies
 * the decay and rotation to it and to the previous token's left-endpoint
 * term, adds the current token's rank-R update, writes the new state and
 * y_t = C_t^T h_t (PaperWeekly page section 3.3; the step is memory-bound).
 * shape->seqlen and shape->chunk are ignored.
 *
 *   state_in   [b][H][N][P] fp32.
 *   state_out  [b][H][N][P] fp32; may equal state_in (in-place update), but
 *              must not partially overlap it.
 *   x_t        [b][H][R][P] io dtype;  dt_t, A_t, lam_t [b][H] fp32;
 *   theta_t    [b][G][N/2] fp32 ([b][H][N/2] with M3_FLAG_THETA_PER_HEAD);
 *   B_t, C_t [b][G][R][N] io dtype.
 *   B_prev,
 *   x_prev     previous token's B [b][G][R][N] and x [b][H][R][P]; both NULL
 *              for a zero left endpoint.
 *   y_t        [b][H][R][P] io dtype.
 * Returns M3_OK when the work was enqueued. */
M3_API int m3_decode_step(const m3_shape* shape, const float* state_in,
                          float* state_out, const void* x_t, const float* dt_t,
                          const float* A_t, const float* lam_t,
                          const float* theta_t, const void* B_t,
                          const void* C_t, const void* B_prev,
                          const void* x_prev, void* y_t, m3_stream_t stream);

/* Size of the fixed device scratch array used by m3_scan_fwd_noalloc (16 MiB). */
#define M3_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* m3_scan_fwd for callers that cannot allocate device memory: for example a
 * plugin whose host framework owns all device memory and offers it no
 * allocator, or a caller on a path where a cudaMalloc (which may synchronise
 * the device) is not acceptable.  The caller passes inputs and outputs only;
 * the scratch memory that m3_scan_fwd takes as `workspace` comes from a
 * library-owned static device array of M3_NOALLOC_SCRATCH_BYTES, which every
 * GPU that loads the library holds until the process exits.  The paper has no
 * counterpart to this call; it only changes where the scratch lives.
 *
 *   - Arguments, layouts, outputs and errors are those of m3_scan_fwd.
 *   - Shapes whose workspace (m3_scan_workspace_size) exceeds
 *     M3_NOALLOC_SCRATCH_BYTES return M3_ERR_WORKSPACE and launch nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept with the identity of
 *     the device's context and looked up again when that changes (after a
 *     cudaDeviceReset, say), so it never outlives the module it points into.
 *   - Nothing is allocated or freed: no cudaMalloc, cudaFree or allocating
 *     library routine.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents; every scratch element is written before it is read, so
 *     nothing needs clearing.  Calls that overlap on the GPU (unordered
 *     streams or host threads) race on the array: order them on one stream. */
M3_API int m3_scan_fwd_noalloc(const m3_shape* shape, const void* x, const float* dt,
                               const float* A, const float* lam, const float* theta,
                               const void* B, const void* C, const float* h0,
                               const void* B_prev, const void* x_prev, void* y,
                               float* final_state, m3_stream_t stream);

/* ---- backward pass ------------------------------------------------------------
 * Gradients of a scalar loss with respect to every input of m3_scan_fwd,
 * given its gradients dy with respect to y and d_final with respect to the
 * final state.  The recurrence is the one of m3_scan_fwd (PaperWeekly page
 * sections 2.1-2.3); the gradients are those of its token-by-token form,
 * evaluated chunk by chunk: the forward's chunk-start states are recomputed,
 * the adjoint of the state is passed backwards over the chunks, and each
 * chunk's gradients follow from its masked quadratic form.  Computed on CUDA
 * cores in fp32 for both io dtypes; every gradient is written in fp32.
 *
 *   inputs      as m3_scan_fwd (same layouts, dtypes and nullability).
 *   dy          [b][L][H][R][P] io dtype, or fp32 with M3_FLAG_DY_F32 (required
 *               when L > 0).
 *   d_final     [b][H][N][P] fp32, or NULL for zero.
 *   dx          [b][L][H][R][P] fp32;  ddt, dA, dlam [b][L][H] fp32;
 *   dtheta      fp32, theta's layout;  dB, dC [b][L][G][R][N] fp32 (summed
 *               over the heads of a group).  All required when L > 0.
 *   dh0         [b][H][N][P] fp32, or NULL to skip (computed whether or not
 *               h0 was given: the gradient with respect to the initial state).
 *   dB_prev,
 *   dx_prev     [b][G][R][N] and [b][H][R][P] fp32, both NULL or both
 *               non-NULL; zeros when B_prev is NULL.
 *   workspace   at least m3_scan_bwd_workspace_size() bytes, 256-byte aligned.
 * dB, dC and dtheta sum contributions of all heads of a group, and ddt, dlam
 * of a chunk's first token also receive the previous chunk's term; these sums
 * are floating-point atomic adds, so those outputs can differ in the last
 * bits from run to run (dx, dA, dh0 are written once and are reproducible).
 * Returns M3_OK when the work was enqueued, M3_ERR_UNSUPPORTED for shapes
 * whose chunk tiles do not fit one CTA's shared memory.
 *
 * m3_scan_bwd_varlen is the same for a packed variable-length batch, with
 * cu_seqlens / total_tokens / layouts as m3_scan_fwd_varlen: dy and dx
 * [T][H][R][P], ddt, dA, dlam [T][H], dtheta [T][Gt][N/2], dB, dC
 * [T][G][R][N]; d_final, dh0 [S][H][N][P]; dB_prev, dx_prev per sequence.
 * Rows of the token dimension outside every sequence are left undefined
 * in dx and dA (zero in the others).  The workspace size is
 * m3_scan_bwd_workspace_size(shape) with shape->batch = S and
 * shape->seqlen = the longest sequence. */
M3_API int m3_scan_bwd_workspace_size(const m3_shape* shape, size_t* bytes);
M3_API int m3_scan_bwd(const m3_shape* shape, const void* x, const float* dt, const float* A,
                       const float* lam, const float* theta, const void* B, const void* C,
                       const float* h0, const void* B_prev, const void* x_prev, const void* dy,
                       const float* d_final, float* dx, float* ddt, float* dA, float* dlam,
                       float* dtheta, float* dB, float* dC, float* dh0, float* dB_prev,
                       float* dx_prev, void* workspace, size_t workspace_bytes,
                       m3_stream_t stream);
M3_API int m3_scan_bwd_varlen(const m3_shape* shape, const int32_t* cu_seqlens,
                              int64_t total_tokens, const void* x, const float* dt,
                              const float* A, const float* lam, const float* theta,
                              const void* B, const void* C, const float* h0,
                              const void* B_prev, const void* x_prev, const void* dy,
                              const float* d_final, float* dx, float* ddt, float* dA,
                              float* dlam, float* dtheta, float* dB, float* dC, float* dh0,
                              float* dB_prev, float* dx_prev, void* workspace,
                              size_t workspace_bytes, m3_stream_t stream);

/* ---- B / C projection prep ------------------------------------------------------
 * QK-norm and learnable bias after the B and C projections (PaperWeekly page
 * section 2.4, "normalisation and bias"; Figure 4).  For every row of N values
 * (one per token, group and rank):
 *   out[n] = raw[n] / sqrt(mean_m raw[m]^2 + eps) * weight[n] + bias[n],
 * computed in fp32 and rounded to the io dtype (nearest even for bf16).  The
 * outputs are the B and C that m3_scan_fwd and m3_decode_step take.
 *
 *   shape      batch, seqlen (tokens = batch * seqlen; 1 for a decode step),
 *              ngroups, rank, dstate, io_dtype; the other fields are checked
 *              as usual but not used.
 *   B_raw, B   [tokens][G][R][N] io dtype; both NULL to skip B.
 *   C_raw, C   the same for C.
 *   *_weight,
 *   *_bias     [G][R][N] fp32, or NULL for 1 and 0.
 *   eps        >= 0.
 * All pointers are 16-byte aligned device pointers.  An output may be its
 * own input (in place); any other overlap returns M3_ERR_INVALID_ARGUMENT. */
M3_API int m3_bc_prep(const m3_shape* shape, const void* B_raw, const void* C_raw,
                      const float* B_weight, const float* B_bias, const float* C_weight,
                      const float* C_bias, float eps, void* B, void* C, m3_stream_t stream);

/* ---- block projections around the layer ----------------------------------------
 * The dense maps of a Mamba-3 block that feed the layer and read its output
 * (PaperWeekly page section 2.4 and Figure 4: the input projections, the
 * data-dependent RoPE angles theta, the MIMO projection; the output gate).
 * The pages name these steps but print no formula for them; the readings are
 * the plainest ones the rest supports:
 *   - every projection is a linear map of the token's features,
 *     out = A W^T (+ bias), with the angle rates theta one such projection
 *     (no nonlinearity);
 *   - the MIMO up-projection gives each rank r of head h a learned copy of
 *     the head's input, X[r][p] = x[p] w_up[h][r][p], and the down-projection
 *     sums the ranks back, y[p] = sum_r Y[r][p] w_down[h][r][p];
 *   - the output gate multiplies by silu(z) = z / (1 + exp(-z)), z a
 *     projection of the block input (the gate of the Mamba block family).
 *
 * m3_linear: out[M][N] = A[M][K] W[N][K]^T (+ bias[N]) on the tensor cores
 * (tcgen05, bf16 operands, fp32 accumulation).
 *   A          [M][K] bf16 (one token per row); W [N][K] bf16 (a weight in
 *              the [out][in] layout); bias [N] fp32 or NULL.
 *   out        [M][N], out_dtype M3_BF16 (rounded to nearest even) or M3_F32.
 *   M >= 0; N >= 1; K >= 8 with K % 8 == 0; N % 8 == 0 (bf16 out) or
 *   N % 4 == 0 (fp32 out); M, N < 2^31 - 256.
 *   A, W, out 16-byte aligned, bias 4-byte aligned; out must not overlap A,
 *   W or bias.  Errors as elsewhere; a device-side wait that gives up is
 *   reported by m3_stream_status (M3_ERR_TIMEOUT). */
M3_API int m3_linear(int64_t M, int64_t N, int64_t K, const void* A, const void* W,
                     const float* bias, void* out, int32_t out_dtype, m3_stream_t stream);

/* MIMO up-projection: X[t][h][r][p] = x[t][h][p] * w_up[h][r][p].
 *   shape      batch, seqlen (tokens = batch * seqlen), nheads, rank,
 *              headdim, io_dtype; the other fields are checked as usual but
 *              not used.
 *   x          [tokens][H][P] io dtype;  w_up [H][R][P] fp32;
 *   X          [tokens][H][R][P] io dtype (the layer's x).
 *   x, X, w_up 16-byte aligned; P % 8 == 0 for bf16 io. */
M3_API int m3_mimo_up(const m3_shape* shape, const void* x, const float* w_up, void* X,
                      m3_stream_t stream);

/* MIMO down-projection and output gate:
 *   out[t][h][p] = (sum_r Y[t][h][r][p] * w_down[h][r][p]) * silu(z[t][h][p]),
 * fp32 arithmetic, rounded to the io dtype.
 *   Y          [tokens][H][R][P] io dtype (the layer's y);  w_down [H][R][P] fp32;
 *   z          [tokens][H][P] io dtype, or NULL for no gate;
 *   out        [tokens][H][P] io dtype.
 *   Shape, alignment and size rules as m3_mimo_up. */
M3_API int m3_mimo_down_gate(const m3_shape* shape, const void* Y, const float* w_down,
                             const void* z, void* out, m3_stream_t stream);

/* ---- packed variable-length batch -------------------------------------------
 * Several sequences of different lengths in one call, stored back to back
 * along the token dimension (no padding): sequence i is tokens
 * [cu_seqlens[i], cu_seqlens[i+1]).  Each sequence is scanned exactly as
 * m3_scan_fwd scans one batch row, with its own h0 / B_prev / x_prev and
 * final state; no state crosses a sequence boundary.  The pages describe no
 * packed layout (the wmrh blog, section 4.3, only discusses deployment in
 * production): this is the serving layout of independent sequences that the
 * recurrence itself allows.
 *
 *   shape->batch   number of sequences S >= 1.
 *   shape->seqlen  an upper bound on every sequence's length (the longest);
 *                  the workspace and launch grid are sized from it.
 *   cu_seqlens     DEVICE array of S + 1 int32 offsets, cu_seqlens[0] = 0,
 *                  nondecreasing, cu_seqlens[S] <= total_tokens; a sequence
 *                  may be empty (its final state is then h0, or zeros).
 *                  Read by the kernels: a pair that breaks these rules or a
 *                  sequence longer than shape->seqlen is not read from; it
 *                  sets M3_ERR_INVALID_ARGUMENT in the device error word
 *                  (m3_stream_status) and that sequence's outputs are
 *                  undefined.
 *   total_tokens   rows T >= 0 of the token dimension of every packed tensor.
 *   x, y           [T][H][R][P] io dtype;  dt, A, lam [T][H] fp32;
 *   theta          [T][G][N/2] fp32 ([T][H][N/2] with M3_FLAG_THETA_PER_HEAD);
 *   B, C           [T][G][R][N] io dtype.
 *   h0, final_state [S][H][N][P] fp32 (nullable, as in m3_scan_fwd);
 *   B_prev [S][G][R][N], x_prev [S][H][R][P] (both NULL or both non-NULL).
 *   workspace      at least m3_scan_workspace_size(shape) bytes.
 * Alignment, aliasing and errors otherwise as m3_scan_fwd; cu_seqlens must
 * be 4-byte aligned. */
M3_API int m3_scan_fwd_varlen(const m3_shape* shape, const int32_t* cu_seqlens,
                              int64_t total_tokens, const void* x, const float* dt,
                              const float* A, const float* lam, const float* theta,
                              const void* B, const void* C, const float* h0,
                              const void* B_prev, const void* x_prev, void* y,
                              float* final_state, void* workspace,
                              size_t workspace_bytes, m3_stream_t stream);

/* ---- sequence split across ranks (context parallel) -------------------------
 * Over a segment of tokens the recurrence unrolls (PaperWeekly page section
 * 2.2, exponential-trapezoidal step; section 2.1, rotation) to
 *   h_end = exp(Lam_seg) Rot(Phi_seg) h_start + T,
 * Lam_seg = sum_t dt_t A_t, Phi_seg,k = sum_t dt_t theta_{t,k}, and T the
 * segment's end state from a zero start.  A rank holding one segment of every
 * sequence calls m3_scan_state (T), m3_segment_totals (Lam_seg, Phi_seg),
 * exchanges them, folds the earlier segments' summaries into its incoming
 * state with m3_state_fold and calls m3_scan_fwd from that state.  These
 * calls have no counterpart on the pages beyond that identity. */

/* Workspace of m3_scan_state (may differ from m3_scan_fwd's). */
M3_API int m3_scan_state_workspace_size(const m3_shape* shape, size_t* bytes);

/* The state after the last token of every sequence, final_state
 * [b][H][N][P] fp32 (required), from h0 (nullable: zero) and
 * B_prev / x_prev (nullable), without computing y.  Arguments, layouts,
 * alignment and errors as m3_scan_fwd; y is not taken. */
M3_API int m3_scan_state(const m3_shape* shape, const void* x, const float* dt, const float* A,
                         const float* lam, const float* theta, const void* B, const void* C,
                         const float* h0, const void* B_prev, const void* x_prev,
                         float* final_state, void* workspace, size_t workspace_bytes,
                         m3_stream_t stream);

/* Segment totals: lam_tot [b][H] = sum_t dt_t A_t and phi_tot [b][H][N/2] =
 * sum_t dt_t theta_{t,k} over the shape's seqlen tokens, accumulated in fp64
 * and written fp32; phi_tot is reduced to [-pi, pi] first (the angle acts only
 * through its cosine and sine).  dt, A, theta as for m3_scan_fwd (4-byte aligned device
 * pointers); outputs 4-byte aligned device arrays owned by the caller. */
M3_API int m3_segment_totals(const m3_shape* shape, const float* dt, const float* A,
                             const float* theta, float* lam_tot, float* phi_tot,
                             m3_stream_t stream);

/* Fold nseg >= 0 segment summaries in order:
 *   h = h0 (nullable: zero);  for s < nseg: h = Rot(phi_tot[s]) exp(lam_tot[s]) h + T[s];
 *   out = h.
 * T [nseg][b][H][N][P], lam_tot [nseg][b][H], phi_tot [nseg][b][H][N/2], h0
 * and out [b][H][N][P], all fp32 device arrays, 16-byte aligned (T, h0,
 * out) or 4-byte aligned (the totals); out must not overlap the inputs.
 * shape->seqlen and shape->chunk are ignored. */
M3_API int m3_state_fold(const m3_shape* shape, int64_t nseg, const float* h0, const float* T,
                         const float* lam_tot, const float* phi_tot, float* out,
                         m3_stream_t stream);

/* Waits for `stream`, then reports the first error since the previous call:
 * M3_ERR_CUDA for a CUDA fault, M3_ERR_TIMEOUT if a bounded device-side wait
 * gave up, else M3_OK.  Clears the library's device-side error word. */
M3_API int m3_stream_status(m3_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* M3_H_ */
