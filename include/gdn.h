/*
 * gdn.h -- C ABI of libgdn.so: the Gated DeltaNet token-mixer recurrence on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (Qwen3.8-Flash-Next summary, picx.dev, "Theoretical
 * foundations", eqs. (1)-(4)), per sequence and head, with a state
 * S in R^{dk x dv}:
 *
 *     St  = alpha_t S_{t-1}            e_t = v_t - St^T k_t
 *     S_t = St + beta_t k_t e_t^T      y_t = scale * S_t^T q_t
 *
 * alpha_t, beta_t are one scalar per (token, head); the pages give their range
 * as (0, 1) (same passage).  When l2norm_qk != 0, q and k are first replaced by
 * x / sqrt(sum(x^2) + 1e-6) (same page, "Methodology", "1. GDN Hybrid Token
 * Mixing": L2 normalisation of queries and keys; the exact formula and epsilon
 * are this library's reading).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers to dense, row-major (C-order)
 *    arrays, last index fastest, each 16-byte aligned.  The caller owns every
 *    buffer; the library allocates nothing and keeps no state between calls.
 *  - Token tensors: q, k [B, T, H, dk]; v, y, dy [B, T, H, dv] in `dtype`
 *    (bf16 or fp32).  alpha, beta, dalpha, dbeta [B, T, H] fp32.  States
 *    s0, s_final, ds_final, ds0 [B, H, dk, dv] fp32 (varlen: [num_seqs, ...]).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous and stream ordered; arguments are validated on the host before
 *    anything is launched, and a rejected call launches nothing.
 *  - Supported sizes: dk == dv, both 64 or 128.  H >= 1, T >= 1, B >= 1.
 *  - Domain: alpha in (0, 1], beta in [0, 1]; not checked on the device.
 *  - Return value: a gdn_status.  Launch failures map to GDN_ERR_CUDA.  Errors
 *    found inside a kernel (a bounded wait that ran out) are recorded in a
 *    device status word read with gdn_read_device_status().  Nothing throws.
 *  - The calls are thread safe: no global mutable host state is touched after
 *    the first call on a device (which caches its properties and the device
 *    addresses of the library's own device arrays).  Those cached addresses do
 *    not survive cudaDeviceReset: do not call the library on a device after a
 *    reset of it in the same process.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,       /* null pointer, bad size, misaligned pointer, bad cu_seqlens */
    GDN_ERR_UNSUPPORTED_SHAPE = 2, /* dk/dv outside the supported set */
    GDN_ERR_WORKSPACE = 3,         /* workspace missing or smaller than gdn_workspace_bytes() */
    GDN_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
    GDN_ERR_TIMEOUT = 5,           /* a device-side bounded wait ran out (device status word) */
    GDN_ERR_UNSUPPORTED_DEVICE = 6 /* the current device is not sm_100 */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_FP32 = 1 } gdn_dtype;

typedef enum {
    GDN_OP_PREFILL = 0,
    GDN_OP_PREFILL_VARLEN = 1,
    GDN_OP_DECODE = 2,
    GDN_OP_BACKWARD = 3,
    GDN_OP_PREFILL_SEGMENTED = 4, /* num_seqs carries the number of segments */
    GDN_OP_QSA_SCORES = 5         /* gdn_qsa_block_scores: only num_seqs matters */
} gdn_op;

/* Static description of a status code.  Never NULL. */
const char* gdn_status_string(int status);

/* Library version string, e.g. "gdn-b200 0.1". */
const char* gdn_version(void);

/*
 * Workspace (device scratch memory, caller-allocated) needed by `op` at the given
 * sizes, in bytes, written to *bytes.  num_seqs is only read for
 * GDN_OP_PREFILL_VARLEN (T is then the packed token count).  A size of 0 means
 * the op needs no workspace and ws may be NULL.
 * Errors: GDN_ERR_INVALID_ARG (bytes NULL, bad sizes, unknown op).
 */
int gdn_workspace_bytes(int op, int B, int T, int H, int dk, int dv, int num_seqs,
                        size_t* bytes);

/*
 * gdn_prefill -- chunked (64-token chunks) forward over B independent sequences
 * of T tokens: writes y and, if s_final is non-NULL, the state after the last
 * token.  s0 == NULL means S_0 = 0.  The computation is exactly eqs. (1)-(4)
 * above, rearranged chunk-wise (WY/UT form), on the tensor cores.  bf16 inputs
 * need the workspace (gdn_workspace_bytes); the fp32 path (a token loop) uses
 * none and accepts ws == NULL.
 *   q, k  [B,T,H,dk]  dtype        v [B,T,H,dv] dtype
 *   alpha, beta [B,T,H] fp32       s0 [B,H,dk,dv] fp32 or NULL
 *   y [B,T,H,dv] dtype (output)    s_final [B,H,dk,dv] fp32 or NULL (output)
 *   ws/ws_bytes: see gdn_workspace_bytes(GDN_OP_PREFILL, ...).
 */
int gdn_prefill(const void* q, const void* k, const void* v, const float* alpha,
                const float* beta, const float* s0, void* y, float* s_final, int B, int T, int H,
                int dk, int dv, int dtype, float scale, int l2norm_qk, void* ws, size_t ws_bytes,
                void* stream);

/*
 * gdn_prefill_varlen -- as gdn_prefill over ONE packed stream of T tokens
 * (tensors laid out with B = 1) holding num_seqs documents: document n covers
 * tokens cu_seqlens[n] .. cu_seqlens[n+1]-1 and starts from s0[n] (zero if s0
 * is NULL); its final state goes to s_final[n].
 *   cu_seqlens: DEVICE int32 [num_seqs+1], cu_seqlens[0] = 0, non-decreasing,
 *   cu_seqlens[num_seqs] = T.  Empty documents are allowed (their s_final is
 *   s0 or 0).  The kernel reads cu_seqlens on the device (no host sync); the
 *   values themselves are not validated on the host.
 */
int gdn_prefill_varlen(const void* q, const void* k, const void* v, const float* alpha,
                       const float* beta, const int32_t* cu_seqlens, int num_seqs,
                       const float* s0, void* y, float* s_final, int T, int H, int dk, int dv,
                       int dtype, float scale, int l2norm_qk, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * gdn_prefill_varlen_prepare / gdn_prefill_varlen_finish -- gdn_prefill_varlen (bf16) in two
 * calls.  The chunked form splits into a part that depends on the chunk alone (decay, norms,
 * the 64x64 triangular inverse and the W / U~ / P operands of every chunk of every document,
 * all computed at once) and a sequential part that walks the chunks from s0 (same page,
 * eqs. (1)-(4), chunk-wise).  prepare runs the first part into the workspace; finish runs the
 * second and writes y and s_final.  The pair computes exactly what one gdn_prefill_varlen call
 * does (which is these two phases back to back); prepare needs no initial state, so it may run
 * before s0 is known.
 *   - finish must get the same q, k, cu_seqlens, num_seqs, T, H, dk, dv and workspace as the
 *     prepare call whose records it reads, be ordered after it (same stream, or an event), and
 *     nothing may write the workspace in between.  scale and l2norm_qk are applied by prepare.
 *   - dtype must be GDN_BF16 (the fp32 path has no split; use gdn_prefill_varlen).
 *   - ws/ws_bytes: gdn_workspace_bytes(GDN_OP_PREFILL_VARLEN, ...).  Errors and validation as
 *     for gdn_prefill_varlen; a non-bf16 dtype is GDN_ERR_INVALID_ARG.
 */
int gdn_prefill_varlen_prepare(const void* q, const void* k, const void* v, const float* alpha,
                               const float* beta, const int32_t* cu_seqlens, int num_seqs, int T,
                               int H, int dk, int dv, int dtype, float scale, int l2norm_qk,
                               void* ws, size_t ws_bytes, void* stream);
int gdn_prefill_varlen_finish(const void* q, const void* k, const int32_t* cu_seqlens,
                              int num_seqs, const float* s0, void* y, float* s_final, int T,
                              int H, int dk, int dv, int dtype, void* ws, size_t ws_bytes,
                              void* stream);
/*
 * gdn_decode_step -- one new token for each of N independent sequences
 * (eqs. (1)-(4) with T = 1).  The state is read once and written once, in place.
 *   q, k [N,H,dk] dtype   v [N,H,dv] dtype   alpha, beta [N,H] fp32
 *   state [N,H,dk,dv] fp32 (input and output)   y [N,H,dv] dtype (output)
 */
int gdn_decode_step(const void* q, const void* k, const void* v, const float* alpha,
                    const float* beta, float* state, void* y, int N, int H, int dk, int dv,
                    int dtype, float scale, int l2norm_qk, void* stream);

/*
 * gdn_backward -- gradients of L(y, s_final) given dy and ds_final (NULL = 0),
 * with respect to the raw q, k (through the normalisation when l2norm_qk), v,
 * alpha (d/d alpha itself), beta and s0 (ds0 may be NULL if not wanted).
 * Dense layout as gdn_prefill.  dq, dk_out, dv_out have q/k/v's dtype; dalpha,
 * dbeta [B,T,H] fp32; ds0 [B,H,dk,dv] fp32.
 *   ws/ws_bytes: see gdn_workspace_bytes(GDN_OP_BACKWARD, ...): per (sequence, 64-token
 *   chunk, head) the chunk's fp32 matrices (W, Ut, P, T, A/beta; 4 * (2*64*dk + 3*64*64)
 *   bytes), 1 KB of scalars, its start state and end-state gradient (2 * 4*dk*dv bytes), its
 *   pseudo-values and their gradient (2 * 4*64*dv bytes), and split bf16 images (hi, lo) of
 *   -W and P (4*64*dk + 4*64*64 bytes).
 * Runs the chunked form: a chunk-parallel pass (the chunk matrices), a forward and a reverse
 * pass over the chunks (states and state gradients), and a chunk-parallel pass for every
 * token's gradients, all in fp32.
 */
int gdn_backward(const void* q, const void* k, const void* v, const float* alpha,
                 const float* beta, const float* s0, const void* dy, const float* ds_final,
                 void* dq, void* dk_out, void* dv_out, float* dalpha, float* dbeta, float* ds0,
                 int B, int T, int H, int dk, int dv, int dtype, float scale, int l2norm_qk,
                 void* ws, size_t ws_bytes, void* stream);

/*
 * gdn_backward_noalloc -- gdn_backward for callers that cannot allocate device memory.
 * (The pages describe no such call; it exists for the library's users.)
 *
 * Some callers may not call cudaMalloc, or any allocator, on the path where they run the
 * backward pass: a plugin inside a host framework whose device memory is owned by that
 * framework's pool, or a server that reserves all of its memory at start-up and forbids later
 * allocations.  This entry point takes no workspace argument: it uses a fixed 32 MiB scratch
 * array compiled into the library, which every GPU that loads the library keeps until the
 * process exits.  It allocates nothing (no cudaMalloc/cudaFree, no allocating library call).
 *   - Arguments, layouts, results and error codes are those of gdn_backward; inputs and
 *     outputs are still the caller's buffers.
 *   - It runs the token-loop form of the backward (one fp32 state checkpoint per 64-token
 *     chunk, each chunk replayed token by token), whose scratch is
 *     (ceil(T/64) + 64) * B*H*dk*dv*4 bytes; sizes where that exceeds
 *     gdn_backward_noalloc_max_workspace() are rejected with GDN_ERR_WORKSPACE before any
 *     launch.  At dk = dv = 128 that is B*H*(ceil(T/64) + 64) <= 512.  Its results agree with
 *     gdn_backward's to rounding (both are fp32).
 *   - The first call on each device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call before any
 *     stream capture.  The address is kept for the life of the process, so the library must
 *     not be used on a device after cudaDeviceReset (or any teardown of its primary context)
 *     has run on it; the device status word behind gdn_read_device_status is kept the same
 *     way.
 *   - All calls share the one array and it keeps the last call's contents; every byte a call
 *     reads from it is written earlier by the same call, so nothing needs clearing.  Calls
 *     whose kernels overlap on the GPU (other streams, other host threads) race on the array:
 *     order them on one stream.
 */
int gdn_backward_noalloc(const void* q, const void* k, const void* v, const float* alpha,
                         const float* beta, const float* s0, const void* dy,
                         const float* ds_final, void* dq, void* dk_out, void* dv_out,
                         float* dalpha, float* dbeta, float* ds0, int B, int T, int H, int dk,
                         int dv, int dtype, float scale, int l2norm_qk, void* stream);

/* Capacity in bytes of the fixed scratch behind gdn_backward_noalloc (32 MiB). */
size_t gdn_backward_noalloc_max_workspace(void);

/*
 * Gated form: the same calls with alpha and beta given by their parameterisation (same page,
 * "Methodology", "1. GDN Hybrid Token Mixing", eqs. (9)-(10)):
 *
 *     beta_t  = sigmoid(b_t)
 *     alpha_t = exp[-exp(A) softplus(a_t + b_alpha)]
 *
 *   a [.., H] fp32: a_t = W_alpha x_t per (token, head), before the bias (in place of alpha);
 *   b [.., H] fp32: b_t = W_beta x_t per (token, head) (in place of beta);
 *   A_log [H], b_alpha [H] fp32: the per-head parameters A and b_alpha (this library's reading:
 *   one each per head, like alpha_t itself).
 * The projections W_alpha x, W_beta x are the caller's (dense products with learned weights).
 * The decay is evaluated in log space, ln alpha = -exp(A) softplus(a + b_alpha), which is what
 * the chunked kernels use, so strong decays never pass through an alpha that underflows.  Every
 * other argument, layout, workspace and error is that of the plain call; A_log and b_alpha must
 * be non-NULL and 16-byte aligned (else GDN_ERR_INVALID_ARG).  a and b may take any finite
 * value; the domain precondition on alpha and beta holds by construction.
 */
int gdn_prefill_gated(const void* q, const void* k, const void* v, const float* a,
                      const float* b, const float* A_log, const float* b_alpha, const float* s0,
                      void* y, float* s_final, int B, int T, int H, int dk, int dv, int dtype,
                      float scale, int l2norm_qk, void* ws, size_t ws_bytes, void* stream);
int gdn_prefill_varlen_gated(const void* q, const void* k, const void* v, const float* a,
                             const float* b, const float* A_log, const float* b_alpha,
                             const int32_t* cu_seqlens, int num_seqs, const float* s0, void* y,
                             float* s_final, int T, int H, int dk, int dv, int dtype, float scale,
                             int l2norm_qk, void* ws, size_t ws_bytes, void* stream);
int gdn_decode_step_gated(const void* q, const void* k, const void* v, const float* a,
                          const float* b, const float* A_log, const float* b_alpha, float* state,
                          void* y, int N, int H, int dk, int dv, int dtype, float scale,
                          int l2norm_qk, void* stream);
/*
 * gdn_backward_gated -- gdn_backward for the gated form: writes da, db [B,T,H] fp32 (gradients
 * with respect to a and b) in place of dalpha, dbeta, and dA_log, db_alpha [H] fp32 (sums over
 * every token of the batch; the call overwrites them).  Workspace: GDN_OP_BACKWARD.  The
 * per-head sums are accumulated with atomic adds, so their last bits may differ between runs.
 */
int gdn_backward_gated(const void* q, const void* k, const void* v, const float* a,
                       const float* b, const float* A_log, const float* b_alpha, const float* s0,
                       const void* dy, const float* ds_final, void* dq, void* dk_out,
                       void* dv_out, float* da, float* db, float* dA_log, float* db_alpha,
                       float* ds0, int B, int T, int H, int dk, int dv, int dtype, float scale,
                       int l2norm_qk, void* ws, size_t ws_bytes, void* stream);

/*
 * gdn_gated_rmsnorm -- the bracket of eq. (11) of the same section,
 *
 *     o = sigmoid(z) * RMSNorm(y),   RMSNorm(y) = (1 + w) * y / sqrt(mean(y^2) + eps),
 *
 * over `rows` independent rows of dv values: one row is one head of one token (y as the
 * recurrence writes it, [B,T,H,dv] being B*T*H rows).  "Zero-centered RMSNorm" is read as the
 * gain (1 + w), so that w = 0 is the identity; no mean is subtracted.  W_z x (= z) and the W_o
 * product after it are the caller's.
 *   y, z, o [rows, dv] in dtype (bf16 or fp32); w [dv] fp32; dv in {64, 128}; eps >= 0
 *   (1e-6 is this library's choice elsewhere); rows >= 0 (0 launches nothing, and y, z, w, o
 *   may then be NULL).
 * Errors: GDN_ERR_INVALID_ARG (null or misaligned pointer, rows < 0, eps < 0 or NaN, bad dtype),
 * GDN_ERR_UNSUPPORTED_SHAPE (dv), GDN_ERR_CUDA.  No workspace.
 */
int gdn_gated_rmsnorm(const void* y, const void* z, const float* w, void* o, int64_t rows,
                      int dv, int dtype, float eps, void* stream);
/*
 * gdn_gated_rmsnorm_backward -- gradients of the above given d_o [rows, dv]: dy, dz [rows, dv]
 * in dtype and dw [dv] fp32 (summed over all rows; the call overwrites it, accumulating with
 * atomic adds, so its last bits may differ between runs).  Same sizes and errors; with rows = 0
 * only dw (zeros) is written and dw alone must be non-NULL.
 */
int gdn_gated_rmsnorm_backward(const void* y, const void* z, const float* w, const void* d_o,
                               void* dy, void* dz, float* dw, int64_t rows, int dv, int dtype,
                               float eps, void* stream);

/*
 * Device status word of the current device: 0 when no kernel has recorded an
 * error, otherwise the first gdn_status a kernel recorded (GDN_ERR_TIMEOUT).
 * Synchronises the current device.  If reset != 0 the word is cleared.
 */
int gdn_read_device_status(int reset, int* device_status);

/*
 * gdn_prefill_segmented -- gdn_prefill of a dense batch with every sequence cut along time into
 * num_segments segments that run side by side.  By eqs. (1)-(3) one token maps the state
 * affinely (S -> alpha (I - beta k k^T) S + beta k v^T), so each segment acts on its start state
 * as S -> M S + N, computable from its own tokens.  The call runs the B * P segments as packed
 * documents: once with v = 0 from S0 = I (giving every M), once from S0 = 0 (every N), scans
 * the maps from s0 for every segment's start state (fp32), and once more from the start states
 * (giving y).  This pays three prefill passes for B * P independent chains instead of B: it is
 * for batches of few, long sequences, where the plain call leaves most SMs idle.
 *   - Arguments and layouts as gdn_prefill; num_segments >= 1.  Segments are whole 64-token
 *     chunks of ceil(ceil(T / 64) / num_segments) chunks each, so fewer may result; with one
 *     segment the call is gdn_prefill.  dk == dv.
 *   - s_final (if non-NULL) is the scan's state after the last segment.
 *   - ws/ws_bytes: gdn_workspace_bytes(GDN_OP_PREFILL_SEGMENTED, B, T, H, dk, dv, num_segments).
 *     It holds the inner packed prefill's workspace (bf16), a zero copy of v, and four fp32
 *     states per (segment, head).
 */
int gdn_prefill_segmented(const void* q, const void* k, const void* v, const float* alpha,
                          const float* beta, const float* s0, void* y, float* s_final, int B,
                          int T, int H, int dk, int dv, int dtype, float scale, int l2norm_qk,
                          int num_segments, void* ws, size_t ws_bytes, void* stream);

/*
 * Short causal convolution ahead of the recurrence (same page, "Methodology", "1. GDN Hybrid
 * Token Mixing": "short causal convolutions").  The page fixes neither the width nor the form;
 * this library's reading is a depthwise causal convolution of each [T, C] input (q, k or v with
 * C = H * d, or a fused [T, 2 H dk + H dv] tensor), W taps per channel and no bias:
 *
 *     y[t, c] = act( sum_{i=0}^{W-1} w[c, i] * x[t - (W - 1) + i, c] ),
 *
 * tap W - 1 weighing the current token; act = identity (activation 0) or SiLU, x sigmoid(x)
 * (activation 1).  Its outputs are the q, k, v the recurrence calls take; the L2 norm of q and
 * k stays fused inside those calls.
 *
 * gdn_short_conv_varlen -- packed documents.
 *   x, y [T, C] in dtype (bf16 or fp32), C a multiple of 8; w [C, W] fp32, 1 <= W <= 8.
 *   cu_seqlens [num_seqs + 1] int32 on the device (monotone, cu[0] = 0, cu[num_seqs] = T;
 *   not checked on the host).  T >= 0, num_seqs >= 1.
 *   conv_state_in [num_seqs, W - 1, C] in dtype (NULL: zero): row j holds the input at
 *   position start - (W - 1) + j of each document, i.e. its W - 1 inputs before its start.
 *   conv_state_out [num_seqs, W - 1, C] (NULL: not written): the last W - 1 inputs of each
 *   document (rows of the initial state where a document is shorter; empty documents keep
 *   theirs).  It must not overlap conv_state_in (equal pointers give GDN_ERR_INVALID_ARG).
 *   Every pointer 16-byte aligned.  One launch; HBM-bound (x read once, y written once).
 * gdn_short_conv_step -- one token per sequence (decode): x, y [N, C]; conv_state
 *   [N, W - 1, C] in dtype, read and then updated in place (shifted by the new token).
 * Errors: GDN_ERR_INVALID_ARG for a null or misaligned pointer, C % 8 != 0, W outside 1..8,
 * an unknown activation or dtype; nothing is launched then.
 */
int gdn_short_conv_varlen(const void* x, const float* w, const int32_t* cu_seqlens,
                          int num_seqs, const void* conv_state_in, void* conv_state_out, void* y,
                          int T, int C, int width, int dtype, int activation, void* stream);
int gdn_short_conv_step(const void* x, const float* w, void* conv_state, void* y, int N, int C,
                        int width, int dtype, int activation, void* stream);

/*
 * QSA block indexer (same page, "Methodology", "2. Qwen Sparse Attention (QSA)", eq. (13); the
 * bud-325 wiki entry, "Key claims": an MQA indexer with 4 query heads and 1 shared key head of
 * dimension 128, a budget of 512 blocks).  Per document (packed by cu_seqlens), keys are cut
 * into blocks of 4 tokens from the document's first token and compressed,
 *     k^_b = g * m / sqrt(mean(m^2) + 1e-6),   m = the mean of the block's 4 key rows;
 * a trailing partial block is never scored.  Query token t at position i of its document scores
 * the blocks complete at or before it (b < floor((i + 1) / 4)) by
 *     I[t, b] = sum_{h<4} ReLU(q[t, h] . k^_b)
 * and selects the budget highest (ties to the lower block index).
 *
 * gdn_qsa_block_scores -- pooled keys and scores.
 *   q [T, 4, 128] bf16, k [T, 128] bf16, g [128] fp32; cu_seqlens [num_seqs + 1] int32 on the
 *   device (monotone, cu[0] = 0, cu[num_seqs] = T), every document at most max_doc_len tokens
 *   (a longer one is recorded as GDN_ERR_INVALID_ARG in the device status word and its scores
 *   are not written).
 *   k_hat [T / 4, 128] bf16 (out): the pooled keys of every document, packed (document n's at
 *   rows block_base[n] .. block_base[n + 1] - 1); block_base [num_seqs + 1] int32 (out).
 *   scores [T, ld] fp32 (out), ld >= floor(max_doc_len / 4) and a multiple of 4: row t holds
 *   I[t, b] for its visible blocks b (document-local indices); the rest of the row is not
 *   written.  ws/ws_bytes: gdn_workspace_bytes(GDN_OP_QSA_SCORES, 1, T, 1, 128, 128, num_seqs).
 *   Launches: a scan of the documents, the pooling, and one tcgen05 product per 32-token query
 *   tile against 128-block key tiles (TMA-fed), ReLU and the head sum in its epilogue.
 * gdn_qsa_select_blocks -- the selection from those scores: sel [T, budget] int32 (out), the
 *   min(budget, visible) selected document-local block indices in increasing order, then -1.
 *   1 <= budget.  One CTA per query token (radix selection over the scores' bit patterns).
 * gdn_qsa_indexer -- both calls, in stream order.
 * Errors: GDN_ERR_INVALID_ARG for a null or misaligned pointer or a bad size; nothing is
 * launched then.
 */
int gdn_qsa_block_scores(const void* q, const void* k, const float* g, const int32_t* cu_seqlens,
                         int num_seqs, int T, int max_doc_len, void* k_hat, int32_t* block_base,
                         float* scores, int ld, void* ws, size_t ws_bytes, void* stream);
int gdn_qsa_select_blocks(const float* scores, int ld, const int32_t* cu_seqlens, int num_seqs,
                          int T, int budget, int32_t* sel, void* stream);
int gdn_qsa_indexer(const void* q, const void* k, const float* g, const int32_t* cu_seqlens,
                    int num_seqs, int T, int max_doc_len, int budget, void* k_hat,
                    int32_t* block_base, float* scores, int ld, int32_t* sel, void* ws,
                    size_t ws_bytes, void* stream);

/*
 * gdn_selftest_wait_timeout -- exercises the failure path of the library's bounded waits.
 * Every wait inside the kernels gives up after a limit, records GDN_ERR_TIMEOUT in the device
 * status word and returns, so that a lost arrival is reported rather than left to hang the GPU.
 * This call launches one small kernel whose wait, on a barrier that nothing arrives on, runs
 * out after about limit_ns nanoseconds (1e3 <= limit_ns <= 1e9, else GDN_ERR_INVALID_ARG).
 * Afterwards gdn_read_device_status() reports GDN_ERR_TIMEOUT (clear it with reset != 0) and
 * the device stays usable.  It touches no caller memory.
 */
int gdn_selftest_wait_timeout(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
