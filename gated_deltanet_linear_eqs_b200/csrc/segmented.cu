// segmented.cu -- segment-parallel prefill of long sequences.
//
// By eqs. (1)-(3) of the Qwen3.8-Flash-Next summary (picx.dev, "Theoretical foundations") one
// token maps the state affinely, S -> alpha (I - beta kh kh^T) S + beta kh v^T, so a run of tokens
// maps it as S -> M S + N with (M, N) computable from the run's own tokens.  A sequence cut into
// P segments therefore runs as:
//   1. every segment's M: the ordinary prefill of the segment with v = 0 from S0 = I
//      (the state then evolves as the product of the token maps' linear parts);
//   2. every segment's N: the ordinary prefill of the segment from S0 = 0;
//   3. the start state of every segment: S^(0) = s0, S^(p+1) = M_p S^(p) + N_p (seg_scan_kernel);
//   4. every segment's outputs: the ordinary prefill of the segment from its start state.
// Steps 1, 2 and 4 treat the B * P segments as independent documents of one packed varlen call,
// so a batch of few long sequences (few chains) fills the GPU with B * P chains; the price is
// three prefill passes instead of one.  The state after the last segment is the scan's.
#include "common.cuh"
#include "internal.h"

namespace gdn {

namespace {

constexpr int kSegChunk = 64;    // segments start on chunk boundaries of their sequence
constexpr int kScanCols = 32;    // state columns per scan CTA
constexpr int kScanThreads = 256;

__host__ __device__ inline size_t seg_up(size_t x) { return (x + 255) & ~size_t(255); }

// segment boundaries as packed-document offsets, and an identity state per (segment, head)
__global__ void seg_setup_kernel(int32_t* cu, float* eye, int B, int P, int T, int L, int H, int D) {
    const long n_cu = (long)B * P + 1;
    const long n_eye = (long)B * P * H * D * D;
    const long stride = (long)gridDim.x * blockDim.x;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n_cu; i += stride) {
        const long b = i / P, p = i % P;
        cu[i] = (i == n_cu - 1) ? (int32_t)((long)B * T) : (int32_t)(b * T + p * L);
    }
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n_eye; i += stride) {
        const long r = i % ((long)D * D);
        eye[i] = (r / D == r % D) ? 1.f : 0.f;
    }
}

// Start state of every segment and the final state, one CTA per (sequence, head, 32 columns):
// S = s0 (or 0); for p < P: start[b P + p] = S; S = M[b P + p] S + N[b P + p].  fp32 FMA.
template <int D>
__global__ void __launch_bounds__(kScanThreads) seg_scan_kernel(const float* __restrict__ M,
                                                                const float* __restrict__ N,
                                                                const float* __restrict__ s0,
                                                                float* __restrict__ start,
                                                                float* __restrict__ s_final, int P,
                                                                int H) {
    constexpr int NPT = D * kScanCols / kScanThreads;  // outputs per thread (16 or 8)
    constexpr int TPR = kScanCols / NPT;               // threads per state row
    __shared__ float Ss[D][kScanCols];
    constexpr int nsl = D / kScanCols;
    const int jsl = blockIdx.x % nsl, h = (blockIdx.x / nsl) % H, b = blockIdx.x / (nsl * H);
    const int col0 = jsl * kScanCols, tid = threadIdx.x;
    const int m = tid / TPR, n0 = (tid % TPR) * NPT;
    const size_t DD = (size_t)D * D;
    for (int e = tid; e < D * kScanCols; e += kScanThreads) {
        const int mm = e / kScanCols, nn = e % kScanCols;
        Ss[mm][nn] = s0 ? s0[((size_t)b * H + h) * DD + (size_t)mm * D + col0 + nn] : 0.f;
    }
    __syncthreads();
    for (int p = 0; p < P; ++p) {
        const size_t rec = ((size_t)b * P + p) * H + h;
        float acc[NPT];
#pragma unroll
        for (int j = 0; j < NPT; ++j) {
            start[rec * DD + (size_t)m * D + col0 + n0 + j] = Ss[m][n0 + j];
            acc[j] = N[rec * DD + (size_t)m * D + col0 + n0 + j];
        }
        const float* Mr = M + rec * DD + (size_t)m * D;
        for (int k = 0; k < D; ++k) {
            const float a = Mr[k];
#pragma unroll
            for (int j = 0; j < NPT; ++j) acc[j] = fmaf(a, Ss[k][n0 + j], acc[j]);
        }
        __syncthreads();  // every thread has read S before it is replaced
#pragma unroll
        for (int j = 0; j < NPT; ++j) Ss[m][n0 + j] = acc[j];
        __syncthreads();
    }
    if (s_final) {
#pragma unroll
        for (int j = 0; j < NPT; ++j)
            s_final[((size_t)b * H + h) * DD + (size_t)m * D + col0 + n0 + j] = Ss[m][n0 + j];
    }
}

}  // namespace

SegmentedLayout segmented_layout(int B, int T, int H, int D, int P, int dtype) {
    SegmentedLayout s{};
    const int nck = (T + kSegChunk - 1) / kSegChunk;
    const int P0 = P < 1 ? 1 : (P > nck ? nck : P);
    s.L = ((nck + P0 - 1) / P0) * kSegChunk;  // segment length: whole chunks
    s.P = (T + s.L - 1) / s.L;                  // non-empty segments
    const size_t docs = (size_t)B * s.P;
    const size_t states = docs * H * D * D * sizeof(float);
    size_t off = 0;
    s.off_inner = off;
    s.inner_bytes = dtype == GDN_BF16 ? prefill_workspace((int)docs, B * T, H, D, true).total : 0;
    off += seg_up(s.inner_bytes);
    s.off_cu = off;
    off += seg_up((docs + 1) * sizeof(int32_t));
    s.off_vzero = off;
    off += seg_up((size_t)B * T * H * D * (dtype == GDN_BF16 ? 2 : 4));
    s.off_eye = off;
    off += seg_up(states);
    s.off_m = off;
    off += seg_up(states);
    s.off_n = off;
    off += seg_up(states);
    s.off_start = off;
    off += seg_up(states);
    s.total = off;
    if (s.P <= 1)  // one segment runs as the plain prefill, with the plain workspace
        s.total = dtype == GDN_BF16 ? prefill_workspace(B, T, H, D, false).total : 0;
    return s;
}

cudaError_t launch_prefill_segmented(const PrefillArgs& a, int P, cudaStream_t st) {
    const int B = a.num_seqs, T = a.T, H = a.H, D = a.dk;
    const SegmentedLayout s = segmented_layout(B, T, H, D, P, a.dtype);
    if (s.P <= 1) return launch_prefill(a, st);  // one segment: the plain prefill
    if (a.ws == nullptr || a.ws_bytes < s.total) return cudaErrorInvalidValue;
    uint8_t* ws = static_cast<uint8_t*>(a.ws);
    int32_t* cu = reinterpret_cast<int32_t*>(ws + s.off_cu);
    void* vzero = ws + s.off_vzero;
    float* eye = reinterpret_cast<float*>(ws + s.off_eye);
    float* Mm = reinterpret_cast<float*>(ws + s.off_m);
    float* Nm = reinterpret_cast<float*>(ws + s.off_n);
    float* start = reinterpret_cast<float*>(ws + s.off_start);
    cudaError_t e;
    const size_t vbytes = (size_t)B * T * H * D * (a.dtype == GDN_BF16 ? 2 : 4);
    if ((e = cudaMemsetAsync(vzero, 0, vbytes, st)) != cudaSuccess) return e;
    seg_setup_kernel<<<296, 256, 0, st>>>(cu, eye, B, s.P, T, s.L, H, D);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the B sequences as B * P packed documents, in the layout the varlen path reads
    PrefillArgs seg = a;
    seg.cu_seqlens = cu;
    seg.num_seqs = B * s.P;
    seg.T = B * T;
    seg.ws = ws + s.off_inner;
    seg.ws_bytes = s.inner_bytes;
    // 1. M of every segment: v = 0 from S0 = I
    PrefillArgs r1 = seg;
    r1.v = vzero;
    r1.s0 = eye;
    r1.s_final = Mm;
    if ((e = launch_prefill(r1, st)) != cudaSuccess) return e;
    // 2. N of every segment: from S0 = 0
    PrefillArgs r2 = seg;
    r2.s0 = nullptr;
    r2.s_final = Nm;
    if ((e = launch_prefill(r2, st)) != cudaSuccess) return e;
    // 3. start states and the final state
    const unsigned grid = (unsigned)(B * H * (D / kScanCols));
    if (D == 128)
        seg_scan_kernel<128><<<grid, kScanThreads, 0, st>>>(Mm, Nm, a.s0, start, a.s_final, s.P, H);
    else
        seg_scan_kernel<64><<<grid, kScanThreads, 0, st>>>(Mm, Nm, a.s0, start, a.s_final, s.P, H);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 4. every segment from its start state: y
    PrefillArgs r3 = seg;
    r3.s0 = start;
    r3.s_final = nullptr;
    return launch_prefill(r3, st);
}

}  // namespace gdn
