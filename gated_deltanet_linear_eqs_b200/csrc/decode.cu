// decode.cu -- one-token decode step of the gated delta rule, streaming the fp32 state once.
//
// Eqs. (1)-(4) of the Qwen3.8-Flash-Next summary (picx.dev, "Theoretical foundations")
// with T = 1.  Substituting (1)-(3) into (4):
//     p = S^T k,  r = S^T q            (both from the OLD state)
//     e = v - alpha p
//     y = scale (alpha r + beta (k.q) e)
//     S <- alpha S + beta k e^T
// so one pass reads S once, reduces over dk twice, and writes S once.
//
// Work split: one CTA per (sequence, head, 64-column slice of dv), 128 threads.  A row
// slice of 64 fp32 (256 B) is read by 16 lanes with 16-byte loads, so one warp
// instruction covers two full rows; each thread owns 4 columns of DK/8 rows and keeps
// them in registers between the read and the write.  The dk reduction is a shuffle
// (between the two rows of a warp) plus a shared-memory sum over the 4 warps.
#include "common.cuh"
#include "internal.h"

namespace gdn {

namespace {

constexpr int kDecodeThreads = 128;
constexpr int kDecodeCols = 64;  // dv columns per CTA

template <int DK, typename T>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
              const float* __restrict__ alpha, const float* __restrict__ beta,
              float* __restrict__ state, T* __restrict__ y, int DV, float scale, int l2norm,
              int H, const float* __restrict__ A_log, const float* __restrict__ b_alpha) {
    constexpr int LPR = kDecodeCols / 4;          // lanes per row (16)
    constexpr int RPW = 32 / LPR;                 // rows per warp instruction (2)
    constexpr int NW = kDecodeThreads / 32;       // warps (4)
    constexpr int ROWS = DK / (RPW * NW);         // rows per thread (16 for DK=128)

    __shared__ float s_kh[DK];
    __shared__ float s_qh[DK];
    __shared__ float s_kq;
    __shared__ float4 s_red[NW][2][LPR];

    const int nh = blockIdx.x;             // (sequence, head) pair
    const int c0 = blockIdx.y * kDecodeCols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cg = lane % LPR, rsub = lane / LPR;
    const int col = c0 + cg * 4;

    float* S = state + (size_t)nh * DK * DV;

    // Issue the whole state slice first: 16-byte streaming loads, all in flight at once.
    float4 s[ROWS];
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int r = (i * NW + warp) * RPW + rsub;
        s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)r * DV + col));
    }

    if (warp == 0) {
        // L2-normalise k and q (fp32), and their dot product.
        float kk = 0.f, qq = 0.f, kq = 0.f;
        float kv[DK / 32], qv[DK / 32];
#pragma unroll
        for (int j = 0; j < DK / 32; ++j) {
            kv[j] = to_f32(k[(size_t)nh * DK + lane + 32 * j]);
            qv[j] = to_f32(q[(size_t)nh * DK + lane + 32 * j]);
            kk += kv[j] * kv[j];
            qq += qv[j] * qv[j];
            kq += kv[j] * qv[j];
        }
        kk = warp_sum(kk);
        qq = warp_sum(qq);
        kq = warp_sum(kq);
        const float rk = l2norm ? 1.0f / sqrtf(kk + kNormEps) : 1.0f;
        const float rq = l2norm ? 1.0f / sqrtf(qq + kNormEps) : 1.0f;
#pragma unroll
        for (int j = 0; j < DK / 32; ++j) {
            s_kh[lane + 32 * j] = kv[j] * rk;
            s_qh[lane + 32 * j] = qv[j] * rq;
        }
        if (lane == 0) s_kq = kq * rk * rq;
    }
    __syncthreads();

    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), r = p;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int row = (i * NW + warp) * RPW + rsub;
        const float kr = s_kh[row], qr = s_qh[row];
        p.x = fmaf(s[i].x, kr, p.x); p.y = fmaf(s[i].y, kr, p.y);
        p.z = fmaf(s[i].z, kr, p.z); p.w = fmaf(s[i].w, kr, p.w);
        r.x = fmaf(s[i].x, qr, r.x); r.y = fmaf(s[i].y, qr, r.y);
        r.z = fmaf(s[i].z, qr, r.z); r.w = fmaf(s[i].w, qr, r.w);
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
        p.x += __shfl_xor_sync(0xffffffffu, p.x, o); p.y += __shfl_xor_sync(0xffffffffu, p.y, o);
        p.z += __shfl_xor_sync(0xffffffffu, p.z, o); p.w += __shfl_xor_sync(0xffffffffu, p.w, o);
        r.x += __shfl_xor_sync(0xffffffffu, r.x, o); r.y += __shfl_xor_sync(0xffffffffu, r.y, o);
        r.z += __shfl_xor_sync(0xffffffffu, r.z, o); r.w += __shfl_xor_sync(0xffffffffu, r.w, o);
    }
    if (rsub == 0) {
        s_red[warp][0][cg] = p;
        s_red[warp][1][cg] = r;
    }
    __syncthreads();
    p = s_red[0][0][cg];
    r = s_red[0][1][cg];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
        const float4 a = s_red[w][0][cg], b = s_red[w][1][cg];
        p.x += a.x; p.y += a.y; p.z += a.z; p.w += a.w;
        r.x += b.x; r.y += b.y; r.z += b.z; r.w += b.w;
    }

    // gated form: alpha, beta hold the logits of eqs. (9)-(10)
    const int h = nh % H;
    const float a = A_log ? expf(gate_log_decay(alpha[nh], A_log[h], b_alpha[h])) : alpha[nh];
    const float b = A_log ? gate_sigmoid(beta[nh]) : beta[nh];
    const float kq = s_kq;
    const float4 vv = load4(v + (size_t)nh * DV + col);
    float4 e;
    e.x = vv.x - a * p.x; e.y = vv.y - a * p.y; e.z = vv.z - a * p.z; e.w = vv.w - a * p.w;
    if (warp == 0 && rsub == 0) {
        const float bk = b * kq;
        float4 yo;
        yo.x = scale * fmaf(a, r.x, bk * e.x); yo.y = scale * fmaf(a, r.y, bk * e.y);
        yo.z = scale * fmaf(a, r.z, bk * e.z); yo.w = scale * fmaf(a, r.w, bk * e.w);
        store4(y + (size_t)nh * DV + col, yo);
    }
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int row = (i * NW + warp) * RPW + rsub;
        const float bk = b * s_kh[row];
        float4 o;
        o.x = fmaf(a, s[i].x, bk * e.x); o.y = fmaf(a, s[i].y, bk * e.y);
        o.z = fmaf(a, s[i].z, bk * e.z); o.w = fmaf(a, s[i].w, bk * e.w);
        __stcs(reinterpret_cast<float4*>(S + (size_t)row * DV + col), o);
    }
}

template <int DK, typename T>
cudaError_t launch(const DecodeArgs& a, cudaStream_t st) {
    dim3 grid((unsigned)(a.N * a.H), (unsigned)(a.dv / kDecodeCols));
    decode_kernel<DK, T><<<grid, kDecodeThreads, 0, st>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
        a.alpha, a.beta, a.state, static_cast<T*>(a.y), a.dv, a.scale, a.l2norm, a.H, a.A_log,
        a.b_alpha);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
    if (a.N == 0) return cudaSuccess;
    if (a.dtype == GDN_BF16)
        return a.dk == 128 ? launch<128, __nv_bfloat16>(a, st) : launch<64, __nv_bfloat16>(a, st);
    return a.dk == 128 ? launch<128, float>(a, st) : launch<64, float>(a, st);
}

}  // namespace gdn
