// internal.h -- host-side launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

struct DecodeArgs {
    const void *q, *k, *v;
    const float *alpha, *beta;
    float* state;
    void* y;
    int N, H, dk, dv, dtype;
    float scale;
    int l2norm;
    // Gated form (eqs. (9)-(10)): when A_log != nullptr, alpha and beta hold the logits
    // a = W_alpha x and b = W_beta x, and A_log, b_alpha [H] the per-head parameters.
    const float* A_log;
    const float* b_alpha;
};

// Dense prefill is the varlen case with B documents of T tokens each (cu_seqlens == nullptr).
struct PrefillArgs {
    const void *q, *k, *v;
    const float *alpha, *beta;
    const float* s0;
    void* y;
    float* s_final;
    const int32_t* cu_seqlens;  // device, [num_seqs+1]; nullptr for the dense layout
    int num_seqs;               // documents (dense: B)
    int T;                      // tokens per sequence (dense) or packed total (varlen)
    int H, dk, dv, dtype;
    float scale;
    int l2norm;
    int* status;                // device status word
    void* ws;                   // workspace (bf16 path), see prefill_workspace
    size_t ws_bytes;
    const float* A_log;         // gated form, as in DecodeArgs
    const float* b_alpha;
};

// Workspace of the bf16 prefill: per (chunk record, head) the operand tiles that the prep kernel
// writes and the chain kernel reads, plus the chunk-record base of every packed document.
struct PrefillWorkspace {
    int nrec_chunks;  // chunk records (an upper bound for packed documents)
    size_t off_cb, off_map, off_w, off_p, off_u, off_s, off_x, total;
};
PrefillWorkspace prefill_workspace(int num_seqs, int T, int H, int d, bool varlen);

struct BackwardArgs {
    const void *q, *k, *v;
    const float *alpha, *beta, *s0;
    const void* dy;
    const float* ds_final;
    void *dq, *dk, *dv;
    float *dalpha, *dbeta, *ds0;
    int B, T, H, dkdim, dvdim, dtype;
    float scale;
    int l2norm;
    void* ws;
    size_t ws_bytes;
    int* status;
    // Gated form, as in DecodeArgs; dalpha and dbeta then receive d a and d b, and the
    // per-head gradients are summed into dA_log, db_alpha [H] (cleared by the launcher).
    const float* A_log;
    const float* b_alpha;
    float* dA_log;
    float* db_alpha;
};

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st);
// One phase of the bf16 prefill: 0 = state-independent part (chunk map + prep kernel),
// 1 = sequential part (chain kernel).  launch_prefill runs both.
cudaError_t launch_prefill_phase(const PrefillArgs& a, int phase, cudaStream_t st);
// Token-by-token prefill on CUDA cores (used for fp32 inputs).
cudaError_t launch_prefill_seq(const PrefillArgs& a, cudaStream_t st);
// The token-loop backward (one fp32 checkpoint per chunk, each chunk replayed token by token).
cudaError_t launch_backward_tokenloop(const BackwardArgs& a, cudaStream_t st);

// Workspace of the token-loop backward (chunk-start states), bytes; the fixed-scratch entry point
// runs that path.
size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv);

// The chunked backward (gdn_backward): per-chunk fp32 records (chunk matrices, S^c, dS', U, dU).
size_t backward_chunked_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_backward_chunked(const BackwardArgs& a, cudaStream_t st);

// The bracket of eq. (11), sigma(z) * RMSNorm(y) with the zero-centred gain (1 + w), over rows
// of dv values, and its reverse mode (dw summed over all rows; cleared by the launcher).
struct GatedNormArgs {
    const void *y, *z;
    const float* w;
    const void* d_o;       // backward only
    void* o;               // forward: o; backward: unused
    void *dy, *dz;         // backward only
    float* dw;             // backward only
    long long rows;
    int dv, dtype;
    float eps;
    int* status;           // device status word (bounded waits that give up)
};
cudaError_t launch_gated_norm(const GatedNormArgs& a, cudaStream_t st);
cudaError_t launch_gated_norm_backward(const GatedNormArgs& a, cudaStream_t st);

// A kernel whose bounded wait runs out (nothing arrives on its barrier): it records
// GDN_ERR_TIMEOUT in `status` after about limit_ns and returns.
cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns, cudaStream_t st);

// Segment-parallel prefill of a dense batch (segmented.cu): every sequence cut into P segments
// of L tokens (whole chunks), the segments' affine state maps formed by two prefill passes, a
// scan of the maps from s0, and a third pass from the segments' start states.
struct SegmentedLayout {
    int L, P;  // segment length in tokens; number of non-empty segments
    size_t off_inner, inner_bytes, off_cu, off_vzero, off_eye, off_m, off_n, off_start, total;
};
SegmentedLayout segmented_layout(int B, int T, int H, int D, int P, int dtype);
cudaError_t launch_prefill_segmented(const PrefillArgs& a, int P, cudaStream_t st);

// The short causal convolution (short_conv.cu): depthwise, W taps per channel, over [T, C]
// tensors with per-document conv states of W - 1 rows.  The varlen form reads state_in (nullable)
// and writes state_out (nullable); the step form (one token per sequence, num_seqs sequences)
// updates state_out in place.
struct ShortConvArgs {
    const void* x;
    const float* w;              // [C, W] fp32
    const int32_t* cu_seqlens;   // varlen form: device, [num_seqs + 1]
    int num_seqs;
    const void* state_in;        // [num_seqs, W - 1, C], dtype of x
    void* state_out;
    void* y;
    int T, C, width, dtype;
    bool silu;
};
cudaError_t launch_short_conv(const ShortConvArgs& a, bool step, cudaStream_t st);

// The QSA block indexer (qsa_indexer.cu): pooled key blocks, block scores, top-budget selection.
struct QsaArgs {
    const void* q;               // [T, 4, 128] bf16 indexer queries
    const void* k;               // [T, 128] bf16 indexer keys (one shared head)
    const float* g;              // [128] RMSNorm gain
    const int32_t* cu_seqlens;   // device, [num_seqs + 1]
    int num_seqs, T, max_doc_len;
    void* k_hat;                 // [T / 4, 128] bf16: pooled keys, packed by document
    int32_t* block_base;         // [num_seqs + 1]: first pooled key of every document
    float* scores;               // [T, ld] fp32: row t holds its visible blocks' scores
    int ld;
    int budget;
    int32_t* sel;                // [T, budget]
    int* status;
    void* ws;
    size_t ws_bytes;
};
size_t qsa_workspace_bytes(int num_seqs);
cudaError_t launch_qsa_scores(const QsaArgs& a, cudaStream_t st);
cudaError_t launch_qsa_select(const QsaArgs& a, cudaStream_t st);

// Size of the fixed device scratch array behind gdn_backward_noalloc.
constexpr size_t kBackwardFixedScratchBytes = size_t(32) << 20;
// Device address of that array on the current device (looked up on first use per device).
int backward_fixed_scratch(void** ptr);

}  // namespace gdn
