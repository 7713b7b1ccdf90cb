/*
 * rocs_ikbo.h -- C ABI of the B200 (sm_100a) In-Kernel Broadcast Optimization library.
 *
 * The operations are those of "ROCS: Request-Oriented Compute Sharing for
 * Efficient Large-Scale Recommendation" (arXiv:2607.27744), as described in the
 * paper-archivist reading notes of that paper:
 *
 *   IKBO-LCB  the two-group ROCSified linear compression block, section 3.1.2, Eq. (6)
 *               Y^R   = W_RR . X^R
 *               Y^C_i = W_CR . X^R_{m_i} + W_CC . X^C_i
 *             executed as the section 4.1 decomposition, Eq. (14):
 *               [Y^R ; Z] = [W_RR ; W_CR] . X^R        once per request (batch B_r)
 *               Y^C_i     = Z_{m_i} + W_CC . X^C_i      per candidate, Z added in the
 *                                                       GEMM epilogue (section 4.2.1)
 *             with request and candidate tiles in one persistent kernel that waits on
 *             per-request completion flags (section 4.2.3).
 *   IKBO-DCA  candidate-group cross attention, section 3.2, Eq. (13):
 *               A^C_i = softmax(scale . Q_i K_{m_i}^T) V_{m_i}     (non-causal)
 *             with K/V stored once per request and m_i resolved inside the kernel
 *             (section 4.3.1).
 *   projection  the linear query generation of the chained block (section 3.2, Eq. (12),
 *             read as a plain linear map): Q_i = W_q . vec(Y^C_i).
 *
 * Common conventions
 *   - Every pointer named *_dev or any tensor pointer is a DEVICE pointer of the current
 *     CUDA device; *_host pointers are host memory.  The caller owns every buffer; the
 *     library never allocates, frees or synchronises inside a *_forward call, and all
 *     device work is enqueued on `stream` (asynchronous w.r.t. the host).
 *   - Tensors are dense row-major with the last axis contiguous.  bf16 tensors hold
 *     IEEE bfloat16 bit patterns; accumulation is fp32; outputs are rounded once
 *     (round-to-nearest-even) when stored.
 *   - Candidate -> request association is a CSR offsets array cand_off[R+1]: request r
 *     owns candidates cand_off[r] .. cand_off[r+1]-1 (candidates of a request are stored
 *     contiguously, section 4.2.1).  m_i is derived from it.  Requests may own zero
 *     candidates.  The host copy must equal the device copy.
 *   - Host-side validation errors are returned synchronously and nothing is enqueued.
 *     Device-side errors (a wait that exceeded its time limit, an index out of range)
 *     are recorded in the workspace status word and reported by rocs_read_status().
 *     No entry point calls exit/abort/__trap or lets a C++ exception cross the ABI.
 *   - workspace: caller-allocated device memory of at least the *_workspace_size()
 *     bytes, 256-byte aligned.  One workspace must not be used by two calls that can
 *     run concurrently.  Each *_forward call resets the status word it uses.
 */
#ifndef ROCS_IKBO_H
#define ROCS_IKBO_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ROCS_API __attribute__((visibility("default")))
#else
#define ROCS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* rocs_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  ROCS_OK = 0,
  ROCS_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned pointer */
  ROCS_ERR_BAD_OFFSETS = 2, /* CSR offsets not 0-based / not non-decreasing / wrong total */
  ROCS_ERR_UNSUPPORTED = 3, /* shape outside the supported set (see each entry point) */
  ROCS_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  ROCS_ERR_TIMEOUT = 5,     /* device: a bounded wait expired (reported by rocs_read_status) */
  ROCS_ERR_WORKSPACE = 6,   /* workspace missing or smaller than required */
  ROCS_ERR_DEVICE_INDEX = 7 /* device: an index derived from device offsets fell out of range */
} rocs_status;

typedef enum { ROCS_F32 = 0, ROCS_BF16 = 1 } rocs_dtype;

/* ------------------------------------------------------------------------------------
 * IKBO-LCB  (section 3.1.2 Eq. (6); section 4.1 Eq. (14); sections 4.2.1-4.2.3)
 *
 *   x_req  [R, n_r, d]       request embeddings X^R (natural batch B_r = R)
 *   x_cand [C, n_c, d]       candidate embeddings X^C (natural batch B_c = C)
 *   w_rr   [o_r, n_r]        W_RR ;  w_cr [o_c, n_r] W_CR ;  w_cc [o_c, n_c] W_CC
 *   y_req  [R, o_r, d]       out: Y^R (computed once per request)
 *   y_cand [C, o_c, d]       out: Y^C
 *   C = cand_off_host[R].
 * dtype ROCS_BF16 (tcgen05 tensor-core path): n_r % 64 == 0, n_c in {64, 128},
 *   d in {64, 128}, o_r % 128 == 0, o_c == 128; else ROCS_ERR_UNSUPPORTED.
 * dtype ROCS_F32 (fp32 CUDA-core path, exact fp32 accumulation): any positive sizes
 *   with n_r, n_c <= 1024 and d <= 1024.
 * Row strides are d * sizeof(element) bytes; they must be multiples of 16 bytes
 *   (the alignment contract of section 4.2.4; padding is the caller's), else
 *   ROCS_ERR_UNSUPPORTED.  All tensor pointers must be 16-byte aligned.
 * ---------------------------------------------------------------------------------- */
typedef struct {
  int64_t R;
  int64_t n_r, n_c, d, o_r, o_c;
  int32_t dtype; /* rocs_dtype, for all inputs and outputs */
  const int32_t* cand_off_dev;  /* [R+1] */
  const int32_t* cand_off_host; /* [R+1] */
  const void* x_req;
  const void* x_cand;
  const void* w_rr;
  const void* w_cr;
  const void* w_cc;
  void* y_req;
  void* y_cand;
  void* workspace; /* >= rocs_lcb_workspace_size(args) bytes: status, flags, tile counter, Z fp32 */
  size_t workspace_bytes;
} rocs_lcb_args;

/* Bytes of workspace rocs_lcb_forward needs for these sizes (0 if the sizes are invalid). */
ROCS_API size_t rocs_lcb_workspace_size(const rocs_lcb_args* args);

/* IKBO-LCB forward, on `stream`: a kernel that zeroes the workspace header and the ready flags, then the
 * LCB kernel (bf16, launched as its programmatic dependent) or the two fp32 kernels. */
ROCS_API int rocs_lcb_forward(const rocs_lcb_args* args, rocs_stream_t stream);

/* Explicit-expand baseline (ablation, not the method): materialises X^R per candidate
 * into an expanded [C, n_r, d] tensor inside the workspace, then runs the same LCB
 * kernels with the identity map (every candidate its own request), so Y^R and Z are
 * recomputed per candidate.  y_req receives the request rows of the first candidate of
 * each request; requests without candidates get W_RR . X^R computed on their own.
 * Workspace: rocs_lcb_expand_workspace_size(). */
ROCS_API size_t rocs_lcb_expand_workspace_size(const rocs_lcb_args* args);
ROCS_API int rocs_lcb_forward_expand(const rocs_lcb_args* args, rocs_stream_t stream);

/* Fault-injection hook for testing the bounded waits (not for production use; the paper has
 * no counterpart).  Identical to rocs_lcb_forward with dtype ROCS_BF16, except that the request
 * tile computing Z for request `skip_release_request` (-1: none) never releases its ready flag, so
 * every candidate epilogue of that request waits until `wait_limit_ns` (1e6 .. 1e10) expires.  The
 * kernel then finishes with ROCS_ERR_TIMEOUT in the workspace status word (read it with
 * rocs_read_status): no trap, no hang, and the CUDA context stays usable.  Outputs of the
 * affected request are undefined.  ROCS_ERR_UNSUPPORTED for ROCS_F32. */
ROCS_API int rocs_lcb_forward_fault_injection(const rocs_lcb_args* args, rocs_stream_t stream,
                                              int64_t skip_release_request, int64_t wait_limit_ns);

/* IKBO-LCB without a caller workspace.  The paper has no counterpart: this entry point
 * exists for callers that cannot hand the library device memory -- e.g. a plugin inside a
 * serving process whose device memory is fully reserved by the host framework's own pool
 * with no allocator exposed, or a latency-critical path on which cudaMalloc is not allowed.
 * It computes exactly what rocs_lcb_forward computes, with the same kernel, but keeps its
 * scratch (status word, ready flags, fp32 Z) in a fixed array of
 * ROCS_LCB_NOALLOC_SCRATCH_BYTES bytes of device memory that the library declares; it
 * allocates and frees nothing.  args->workspace and args->workspace_bytes are ignored.
 *   - Sizes whose scratch (rocs_lcb_workspace_size(args)) exceeds the array are rejected
 *     with ROCS_ERR_WORKSPACE (with o_c = d = 128 that is about 127 requests).
 *   - Every GPU that loads the library holds the array until the process exits.
 *   - All calls on a device share the array: calls that can overlap on the GPU race and
 *     must be serialised by the caller.  The array keeps the last call's contents; each
 *     call clears the status word and flags itself.
 *   - The first call on a device looks up the array's device address (once per device);
 *     make that first call before any stream capture starts.  cudaDeviceReset() invalidates
 *     that address: do not use this entry point on a device after resetting it.
 *   - Device-side status (a bounded wait that expired: ROCS_ERR_TIMEOUT; a bad device
 *     offset: ROCS_ERR_DEVICE_INDEX) is kept in the array's own header: read it with
 *     rocs_lcb_noalloc_read_status(), not rocs_read_status().  Host-side validation errors
 *     are returned as for rocs_lcb_forward. */
#define ROCS_LCB_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
ROCS_API int rocs_lcb_forward_noalloc(const rocs_lcb_args* args, rocs_stream_t stream);

/* Device status of the last rocs_lcb_forward_noalloc call on the CURRENT device (the paper
 * has no counterpart).  Synchronises `stream`, then copies the code and detail words from the
 * header of the library's scratch array into *device_code (a rocs_status; required) and
 * *detail (may be NULL); allocates nothing.  Call it on the stream of that call, with the same
 * device current.  Returns ROCS_OK, or ROCS_ERR_INVALID_ARG / ROCS_ERR_CUDA for the read. */
ROCS_API int rocs_lcb_noalloc_read_status(rocs_stream_t stream, int32_t* device_code, int32_t* detail);

/* ------------------------------------------------------------------------------------
 * LCB block: IKBO-LCB with a fused per-group output epilogue
 *   (section 3.1.2 Eq. (4) bias; section 3.1.3 Eq. (7) group-local norm and Eq. (8)
 *    pointwise merge / activation)
 *
 * For every output row y (length d) of group g in {R, C}, in this order:
 *   y = (W X)_row + bias_g[o]                 o = the row's index within the group's o_g rows
 *   y = y + residual_g[row]                    if residual_g != NULL
 *   y = Norm_g(y) * gamma_g + beta_g           LayerNorm (population variance) or RMSNorm over
 *                                              the row's d entries, eps_g inside the square root
 *   y = act_g(y)                               ReLU, SiLU or GELU (erf form)
 * Each group uses only its own parameters and its own rows, so the request outputs stay
 * independent of the candidate inputs (Eq. (1)).  The candidate bias is folded into Z once
 * per request (Eq. (14)); the norm's statistics stay in the thread that owns the row.
 *
 *   bias     [o_g] fp32, or NULL (0)      gamma, beta [d] fp32 16-byte aligned, or NULL (1, 0)
 *   residual bf16, shape of the group's output ([R, o_r, d] or [C, o_c, d]), or NULL;
 *            16-byte aligned (read by TMA)
 *   norm     ROCS_NORM_*;  act ROCS_ACT_*;  eps >= 0 and finite
 * dtype must be ROCS_BF16 (else ROCS_ERR_UNSUPPORTED); sizes, workspace and errors as for
 * rocs_lcb_forward (workspace: rocs_lcb_workspace_size).  A NULL epilogue pointer means no
 * epilogue for that group.  Two kernel launches (the zeroing kernel and the LCB kernel).
 * ---------------------------------------------------------------------------------- */
typedef enum { ROCS_NORM_NONE = 0, ROCS_NORM_LAYER = 1, ROCS_NORM_RMS = 2 } rocs_norm;
typedef enum { ROCS_ACT_NONE = 0, ROCS_ACT_RELU = 1, ROCS_ACT_SILU = 2, ROCS_ACT_GELU = 3 } rocs_act;
typedef struct {
  const float* bias;
  const void* residual;
  const float* gamma;
  const float* beta;
  float eps;
  int32_t norm; /* rocs_norm */
  int32_t act;  /* rocs_act */
} rocs_lcb_epilogue;

ROCS_API int rocs_lcb_block_forward(const rocs_lcb_args* args, const rocs_lcb_epilogue* epi_req,
                                    const rocs_lcb_epilogue* epi_cand, rocs_stream_t stream);

/* Fault-injection hook for the LCB block kernel (not for production use; the paper has no
 * counterpart): rocs_lcb_block_forward whose request tile computing Z for request
 * `skip_release_request` (-1: none) never releases its ready flag, with every device wait limited
 * to `wait_limit_ns` (1e6 .. 1e10).  Same contract as rocs_lcb_forward_fault_injection: the
 * kernel ends with ROCS_ERR_TIMEOUT in the workspace status word, no trap, no hang, and the
 * context stays usable; outputs of the affected request are undefined. */
ROCS_API int rocs_lcb_block_forward_fault_injection(const rocs_lcb_args* args, const rocs_lcb_epilogue* epi_req,
                                                    const rocs_lcb_epilogue* epi_cand, rocs_stream_t stream,
                                                    int64_t skip_release_request, int64_t wait_limit_ns);

/* ------------------------------------------------------------------------------------
 * IKBO masked factorization machine  (section 3.1.4 Eq. (9)-(10); section 4.1; section 4.2.4)
 *
 *   Y^R_r = X^R_r X^R_r^T                           once per request
 *   Y^C_i = [ X^C_i X^R_{m_i}^T , X^C_i X^C_i^T ]    per candidate (n_r + n_c columns)
 *
 *   x_req  [R, n_r, d] bf16        x_cand [C, n_c, d] bf16        C = cand_off_host[R]
 *   y_req  [R, n_r, ld_req] bf16   out: Y^R_r in columns [0, n_r), zeros in [n_r, ld_req)
 *   y_cand [C, n_c, ld_cand] bf16  out: Y^C_i in columns [0, n_r + n_c), zeros beyond
 * The leading dimensions are the alignment transform of section 4.2.4: 0 selects
 * rocs_align_cols(n_r, 2) / rocs_align_cols(n_r + n_c, 2), the smallest row lengths whose byte
 * size is a multiple of 16, so every row moves by TMA even when n_r + n_c alone would not; a
 * consumer of the padded rows gives its weight zero columns at the padded positions (which
 * rocs_pad_cols produces) and computes the same result.
 * Supported: d in {64, 128}; n_c in {32, 64, 128}; n_r even and <= 256; ld_* multiples of 8 and
 * <= 384; else ROCS_ERR_UNSUPPORTED.  Pointers 16-byte aligned.  fp32 accumulation, one bf16
 * rounding per output.  Workspace: rocs_fm_workspace_size() bytes (status + a per-request tile
 * table).  Two launches (tile table, FM kernel) plus one memset on `stream`.
 * ---------------------------------------------------------------------------------- */
typedef struct {
  int64_t R, n_r, n_c, d;
  const int32_t* cand_off_dev;  /* [R+1] */
  const int32_t* cand_off_host; /* [R+1] */
  const void* x_req;
  const void* x_cand;
  void* y_req;
  void* y_cand;
  int64_t ld_req, ld_cand; /* row lengths of y_req / y_cand in elements; 0 = aligned default */
  void* workspace;
  size_t workspace_bytes;
} rocs_fm_args;

ROCS_API size_t rocs_fm_workspace_size(const rocs_fm_args* args);
ROCS_API int rocs_fm_forward(const rocs_fm_args* args, rocs_stream_t stream);

/* Alignment transform helpers (section 4.2.4; no device memory of their own).
 * rocs_align_cols: the smallest n >= cols with n * elem_bytes a multiple of 16 (elem_bytes in
 *   {1, 2, 4, 8}; -1 otherwise).
 * rocs_pad_cols: dst[r, 0:cols] = src[r, 0:cols], dst[r, cols:ld_dst] = 0 for r < rows, with row
 *   strides ld_src / ld_dst in elements (ld_* >= cols).  With ld_dst == cols it removes padding.
 *   Pointers aligned to elem_bytes; src and dst must not overlap.  One launch on `stream`. */
ROCS_API int64_t rocs_align_cols(int64_t cols, int64_t elem_bytes);
ROCS_API int rocs_pad_cols(const void* src, int64_t rows, int64_t cols, int64_t ld_src, void* dst, int64_t ld_dst,
                           int64_t elem_bytes, rocs_stream_t stream);

/* ------------------------------------------------------------------------------------
 * IKBO-DCA  (section 3.2 Eq. (13); section 4.3)
 *
 *   q_ptr  [C*q, H, dh] bf16   query tokens; candidate i owns rows i*q .. i*q+q-1
 *   k_ptr  [T, H, dh]   bf16   request keys, T = seq_off_host[R]; request r owns rows
 *   v_ptr  [T, H, dh]   bf16   seq_off[r] .. seq_off[r+1]-1 (stored once per request)
 *   o_ptr  [C*q, H, dh] bf16   out: attention output
 *   lse_ptr [C*q, H]    fp32   out (optional, may be NULL): natural-log sum-exp of the
 *                              scaled scores; -inf where the request has no keys
 *   scale                      softmax scale (1/sqrt(dh) in the usual setting)
 * A request with keys but no candidates is legal (no work); a request with candidates
 * but no keys gets O = 0 and LSE = -inf.  Every query token attends to all keys of its
 * request (non-causal); query tokens of one candidate do not attend to each other.
 * Supported: dh in {64, 128}, H >= 1, q >= 1, row strides multiples of 16 bytes.
 * kv_ld: row stride of K and V in elements (0 means H*dh, i.e. dense rows); it lets K and V be
 * read in place from a wider projection output.
 * ---------------------------------------------------------------------------------- */
typedef struct {
  int64_t R, q, H, dh;
  float scale;
  const int32_t* cand_off_dev;  /* [R+1] */
  const int32_t* cand_off_host; /* [R+1] */
  const int32_t* seq_off_dev;   /* [R+1] */
  const int32_t* seq_off_host;  /* [R+1] */
  const void* q_ptr;
  const void* k_ptr;
  const void* v_ptr;
  void* o_ptr;
  float* lse_ptr;
  void* workspace; /* >= rocs_dca_workspace_size(args): status, work-unit table, counter */
  size_t workspace_bytes;
  int64_t kv_ld; /* row stride of K and V in elements; 0 = H*dh */
} rocs_dca_args;

/* The size depends on the current device's SM count (the units of the last partial wave are split in
 * two along the keys when every request has the same number of K/V tiles, and each split unit needs a
 * merge area): query it with the device current that rocs_dca_forward will run on.  Returns 0 when
 * the arguments are invalid. */
ROCS_API size_t rocs_dca_workspace_size(const rocs_dca_args* args);

/* IKBO-DCA forward: a scheduling kernel (work-unit table, longest request first) and the
 * persistent attention kernel, both on `stream`. */
ROCS_API int rocs_dca_forward(const rocs_dca_args* args, rocs_stream_t stream);

/* Explicit-expand baseline (ablation): copies each candidate's request K/V into a
 * per-candidate buffer (the materialised broadcast of section 4.3), `chunk` candidates
 * at a time, and runs the same attention kernel with the identity map on each chunk.
 * Workspace: rocs_dca_expand_workspace_size(args, chunk). */
ROCS_API size_t rocs_dca_expand_workspace_size(const rocs_dca_args* args, int64_t chunk);
ROCS_API int rocs_dca_forward_expand(const rocs_dca_args* args, int64_t chunk, rocs_stream_t stream);

/* ------------------------------------------------------------------------------------
 * DCA block: both query groups of section 3.2, Eq. (13), with the K/V projections done once per
 * request (section 4.1: (S_{m_i}) W = (S W)_{m_i}):
 *   [K^C | V^C | K^R | V^R] = S . [W_K^C ; W_V^C ; W_K^R ; W_V^R]^T     (one GEMM at batch B_r)
 *   A^C_i = softmax(scale Q^C_i K^C_{m_i}^T) V^C_{m_i}                   (IKBO-DCA, candidate group)
 *   A^R_r = softmax(scale Q^R_r K^R_r^T) V^R_r                            (request group, q_req tokens)
 *   s_seq [T, d_s] bf16     request sequence representation, T = seq_off_host[R]
 *   w_kv  [4*H*dh, d_s]     the four projection weights stacked in that order
 *   q_c [C*q, H, dh], q_r [R*q_req, H, dh]; o_c / o_r alike; lse_c [C*q, H], lse_r [R*q_req, H]
 *   (lse pointers may be NULL).  Projected K/V are stored bf16 in the workspace.
 * Supported: dh in {64, 128}, d_s % 64 == 0, q >= 1, q_req >= 1.
 * Launches: one projection GEMM, one identity-map fill and two (schedule + attention) pairs.
 * ---------------------------------------------------------------------------------- */
typedef struct {
  int64_t R, q, q_req, H, dh, d_s; /* q: tokens per candidate, q_req: request query tokens */
  float scale;
  const int32_t* cand_off_dev;  /* [R+1] */
  const int32_t* cand_off_host; /* [R+1] */
  const int32_t* seq_off_dev;   /* [R+1] */
  const int32_t* seq_off_host;  /* [R+1] */
  const void* s_seq;
  const void* w_kv;
  const void* q_c;
  const void* q_r;
  void* o_c;
  float* lse_c;
  void* o_r;
  float* lse_r;
  void* workspace; /* >= rocs_dca_block_workspace_size(args) */
  size_t workspace_bytes;
} rocs_dca_block_args;

ROCS_API size_t rocs_dca_block_workspace_size(const rocs_dca_block_args* args);
ROCS_API int rocs_dca_block_forward(const rocs_dca_block_args* args, rocs_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Linear query projection of the chained block (section 3.2, Eq. (12), plain linear
 * map, no bias, no activation):  out[i, :] = W . in[i, :]
 *   in  [M, K] bf16 (for the chained block: Y^C viewed as [C, o_c*d])
 *   w   [N, K] bf16
 *   out [M, N] bf16
 * Supported: K % 64 == 0, N % 256 == 0, M >= 0.
 * ---------------------------------------------------------------------------------- */
typedef struct {
  int64_t M, N, K;
  const void* in;
  const void* w;
  void* out;
  void* workspace; /* >= rocs_proj_workspace_size(args) */
  size_t workspace_bytes;
} rocs_proj_args;

ROCS_API size_t rocs_proj_workspace_size(const rocs_proj_args* args);
ROCS_API int rocs_proj_forward(const rocs_proj_args* args, rocs_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Split chain: the query projection of the chained block distributed over the IKBO
 * decomposition (section 3.2 Eq. (12) with section 4.1 Eq. (14); the projection is a plain
 * linear map):
 *     Q_i = W_q vec(Y^C_i) = W_q vec(Z_{m_i}) + W_q vec(W_CC X^C_i)
 *         = q^R_{m_i} + W_fold vec(X^C_i)
 * with q^R_r = W_q vec(Z_r) computed once per request and W_fold[k, n*d + c] =
 * sum_o W_q[k, o*d + c] W_CC[o, n] prepared once per model.  Y^C is never written; the
 * result equals the chain on the exact (unrounded) LCB output up to bf16 rounding of Z_r and
 * of W_fold.
 *
 * rocs_chain_prepare_weights (once per model):
 *   w_q [n_out, o_c*d], w_rr [o_r, n_r], w_cr [o_c, n_r], w_cc [o_c, n_c]  bf16 in
 *   w_fold [n_out, n_c*d] bf16 out (fp32 accumulation, one rounding)
 *   w_rs   [o_r + o_c, n_r] bf16 out: [W_RR; W_CR] stacked
 *   One launch plus two device-to-device copies on `stream`.
 * rocs_chain_split_forward (per batch):
 *   y_req [R, o_r + o_c, d] bf16 out: rows [0, o_r) = Y^R_r, rows [o_r, o_r + o_c) = Z_r
 *   q     [C, n_out] bf16 out: the candidate queries (input of rocs_dca_forward)
 *   Shapes as rocs_lcb_forward (ROCS_BF16) with o_r + o_c in place of o_r, n_out % 256 == 0,
 *   (n_c*d) % 64 == 0.  Workspace rocs_chain_split_workspace_size(); one status header for all
 *   steps (rocs_read_status).  Four kernel launches plus memsets.
 * ---------------------------------------------------------------------------------- */
typedef struct {
  int64_t n_out, o_r, o_c, n_r, n_c, d;
  const void* w_q;
  const void* w_rr;
  const void* w_cr;
  const void* w_cc;
  void* w_fold;
  void* w_rs;
} rocs_chain_weights_args;

ROCS_API int rocs_chain_prepare_weights(const rocs_chain_weights_args* args, rocs_stream_t stream);

typedef struct {
  int64_t R, n_r, n_c, d, o_r, o_c, n_out;
  const int32_t* cand_off_dev;  /* [R+1] */
  const int32_t* cand_off_host; /* [R+1] */
  const void* x_req;  /* [R, n_r, d] */
  const void* x_cand; /* [C, n_c, d] */
  const void* w_rs;   /* [o_r + o_c, n_r] from rocs_chain_prepare_weights */
  const void* w_q;    /* [n_out, o_c*d] */
  const void* w_fold; /* [n_out, n_c*d] from rocs_chain_prepare_weights */
  void* y_req;        /* [R, o_r + o_c, d] */
  void* q;            /* [C, n_out] */
  void* workspace;
  size_t workspace_bytes;
} rocs_chain_split_args;

ROCS_API size_t rocs_chain_split_workspace_size(const rocs_chain_split_args* args);
ROCS_API int rocs_chain_split_forward(const rocs_chain_split_args* args, rocs_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Host-resident batches (no counterpart in the paper: the serving path of a batch that lives in
 * host memory).  The same operations as rocs_lcb_forward / rocs_dca_forward, but the batch
 * tensors are HOST pointers (pinned memory, so the copies run asynchronously):
 *   LCB: x_req, x_cand in; y_req, y_cand out (host).  Weights w_* and cand_off_dev stay on the
 *        device; cand_off_host as usual.
 *   DCA: q_ptr, k_ptr, v_ptr in; o_ptr, lse_ptr (or NULL) out (host); cand_off_dev, seq_off_dev
 *        on the device; kv_ld must be 0 (or H*dh).
 * The batch is cut into `chunks` groups of whole requests of about equal bytes; chunk c is computed
 * while chunk c+1 is copied in and chunk c-1 copied out, through two device staging slots held in
 * `staging` (>= rocs_*_host_staging_size(args, chunks) bytes, 256-byte aligned, caller-owned; the
 * args' workspace fields are ignored).  Copies and kernels run on three streams the library creates
 * once per device and keeps; `stream` waits for the whole call, so work enqueued on it afterwards
 * (e.g. a host read of the outputs after a synchronize) sees every output.  Device status of all
 * chunks is kept in the first 256 bytes of `staging` (rocs_read_status(staging, ...)).  Errors as
 * for the device entry points; a host error returned after some chunks were enqueued leaves the
 * outputs of those chunks to complete.
 * ---------------------------------------------------------------------------------- */
ROCS_API size_t rocs_lcb_host_staging_size(const rocs_lcb_args* args, int64_t chunks);
ROCS_API int rocs_lcb_forward_host(const rocs_lcb_args* args, int64_t chunks, void* staging, size_t staging_bytes,
                                   rocs_stream_t stream);
ROCS_API size_t rocs_dca_host_staging_size(const rocs_dca_args* args, int64_t chunks);
ROCS_API int rocs_dca_forward_host(const rocs_dca_args* args, int64_t chunks, void* staging, size_t staging_bytes,
                                   rocs_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Status and introspection
 * ---------------------------------------------------------------------------------- */

/* Synchronises `stream`, then reads the device status word of `workspace` (the workspace
 * of the last *_forward call that used it) into *device_code (a rocs_status) and, if
 * `detail` is non-NULL, a code naming where the error was raised.  Returns ROCS_OK or
 * ROCS_ERR_CUDA / ROCS_ERR_INVALID_ARG for the read itself. */
ROCS_API int rocs_read_status(const void* workspace, rocs_stream_t stream, int32_t* device_code, int32_t* detail);

/* Human-readable name of a rocs_status value (static string). */
ROCS_API const char* rocs_status_string(int code);

/* Number of kernel launches the last successful *_forward call on this host thread
 * enqueued (memsets not counted). */
ROCS_API int rocs_last_launch_count(void);

/* Bit k is set once some kernel of this library has had its per-device set-up (the opt-in to
 * large dynamic shared memory, which CUDA applies to the current device only) done on device
 * ordinal k in this process.  The set-up runs on the first launch of each kernel on each device,
 * so a process that drives several GPUs configures every one of them.  Ordinals past 63 are
 * configured on every launch and not recorded.  Host-only; never fails. */
ROCS_API uint64_t rocs_configured_device_mask(void);

#ifdef __cplusplus
}
#endif

#endif /* ROCS_IKBO_H */
