// prefill_seq.cu -- token-by-token prefill for fp32 inputs.
//
// The tensor-core prefill (prefill.cu) takes bf16 q/k/v.  fp32 inputs run this kernel: one CTA
// per (sequence or document, head) walks the tokens in order with the fp32 state in registers,
// evaluating eqs. (1)-(4) of the Qwen3.8-Flash-Next summary (picx.dev, "Theoretical
// foundations") exactly as written, the output in the single-pass form
//     p = S^T kh, r = S^T qh (old state);  e = v - a p;  y = scale (a r + b (kh.qh) e);
//     S <- a S + b kh e^T.
// Layout: warp w owns rows 8w..8w+7 of the dk x dv state, lane l owns columns
// [l*CPL, l*CPL + CPL); the two dk reductions go through shared memory (double-buffered, one
// barrier per token).
#include "common.cuh"
#include "internal.h"

namespace gdn {

namespace {

template <int D, typename T>
__global__ void __launch_bounds__(D * 4)
seq_prefill_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ alpha, const float* __restrict__ beta,
                   const float* __restrict__ s0, T* __restrict__ y, float* __restrict__ s_final,
                   const int32_t* __restrict__ cu_seqlens, int T_len, int H, float scale,
                   int l2norm, const float* __restrict__ A_log,
                   const float* __restrict__ b_alpha) {
    constexpr int NW = D / 8, CPL = D / 32, PL = D / 32;
    __shared__ float s_kh[2][D];
    __shared__ float s_qh[2][D];
    __shared__ float s_kq[2];
    __shared__ float s_red[2][NW][2][D];
    const int chain = blockIdx.x;  // n * H + h
    const int n = chain / H, h = chain % H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c0 = lane * CPL;
    long t0, t1;
    if (cu_seqlens) {
        t0 = cu_seqlens[n];
        t1 = cu_seqlens[n + 1];
    } else {
        t0 = (long)n * T_len;
        t1 = t0 + T_len;
    }
    const size_t soff = (size_t)chain * D * D;
    float S[8][CPL];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < CPL; ++j)
            S[i][j] = s0 ? s0[soff + (size_t)(warp * 8 + i) * D + c0 + j] : 0.f;

    for (long t = t0; t < t1; ++t) {
        const int buf = (int)(t & 1);
        const size_t th = (size_t)t * H + h;
        if (warp == 0) {
            float kv[PL], qv[PL], sk = 0.f, sq = 0.f;
#pragma unroll
            for (int j = 0; j < PL; ++j) {
                kv[j] = to_f32(k[th * D + lane + 32 * j]);
                qv[j] = to_f32(q[th * D + lane + 32 * j]);
                sk += kv[j] * kv[j];
                sq += qv[j] * qv[j];
            }
            sk = warp_sum(sk);
            sq = warp_sum(sq);
            const float rk = l2norm ? 1.0f / sqrtf(sk + kNormEps) : 1.f;
            const float rq = l2norm ? 1.0f / sqrtf(sq + kNormEps) : 1.f;
            float kq = 0.f;
#pragma unroll
            for (int j = 0; j < PL; ++j) {
                s_kh[buf][lane + 32 * j] = kv[j] * rk;
                s_qh[buf][lane + 32 * j] = qv[j] * rq;
                kq += kv[j] * rk * qv[j] * rq;
            }
            kq = warp_sum(kq);
            if (lane == 0) s_kq[buf] = kq;
        }
        __syncthreads();
        float khr[8];
        float pk[CPL] = {}, pq[CPL] = {};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            khr[i] = s_kh[buf][warp * 8 + i];
            const float qr = s_qh[buf][warp * 8 + i];
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                pk[j] = fmaf(S[i][j], khr[i], pk[j]);
                pq[j] = fmaf(S[i][j], qr, pq[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            s_red[buf][warp][0][c0 + j] = pk[j];
            s_red[buf][warp][1][c0 + j] = pq[j];
        }
        __syncthreads();
        // gated form: alpha, beta hold the logits of eqs. (9)-(10)
        const float a = A_log ? expf(gate_log_decay(alpha[th], A_log[h], b_alpha[h])) : alpha[th];
        const float b = A_log ? gate_sigmoid(beta[th]) : beta[th];
        const float kq = s_kq[buf];
        float e[CPL];
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            float p = 0.f, r = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                p += s_red[buf][w][0][c0 + j];
                r += s_red[buf][w][1][c0 + j];
            }
            e[j] = to_f32(v[th * D + c0 + j]) - a * p;
            if (warp == 0) y[th * D + c0 + j] = from_f32<T>(scale * fmaf(a, r, b * kq * e[j]));
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < CPL; ++j) S[i][j] = fmaf(a, S[i][j], b * khr[i] * e[j]);
    }
    if (s_final) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < CPL; ++j) s_final[soff + (size_t)(warp * 8 + i) * D + c0 + j] = S[i][j];
    }
}

template <int D, typename T>
cudaError_t launch_t(const PrefillArgs& a, cudaStream_t st) {
    seq_prefill_kernel<D, T><<<a.num_seqs * a.H, D * 4, 0, st>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
        a.alpha, a.beta, a.s0, static_cast<T*>(a.y), a.s_final, a.cu_seqlens, a.T, a.H, a.scale,
        a.l2norm, a.A_log, a.b_alpha);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_seq(const PrefillArgs& a, cudaStream_t st) {
    if (a.dtype == GDN_FP32)
        return a.dk == 128 ? launch_t<128, float>(a, st) : launch_t<64, float>(a, st);
    return a.dk == 128 ? launch_t<128, __nv_bfloat16>(a, st) : launch_t<64, __nv_bfloat16>(a, st);
}

}  // namespace gdn
