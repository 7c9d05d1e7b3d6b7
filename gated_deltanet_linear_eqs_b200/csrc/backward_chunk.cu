// backward_chunk.cu -- the backward pass of eqs. (1)-(4) (Qwen3.8-Flash-Next summary, picx.dev,
// "Theoretical foundations"; the reverse recurrence of its Appendix B) in the chunked WY form of
// the forward, on 64-token chunks, with fp32 states and accumulation and the products on tensor
// cores.  For bf16 inputs every kernel runs tcgen05 tiles (bwdc_prep_tc, bwdc_fwd_tc,
// bwdc_rev_tc with exact or split bf16 operands; bwdc_local with tf32 operands); for fp32 inputs
// the chunk matrices and the chains run warp-level m16n8k8 tf32 tiles (the reverse chain's dS
// products with split 3 x tf32 operands, since their rounding accumulates into dS0).
//
// Per chunk, with q^ = rq q, k^ = rk k the normalised rows, Lg the inclusive cumsum of ln(alpha),
// gam = e^Lg, gC = gam of the chunk's last token, Gam_ij = e^(Lg_i - Lg_j), S = S^c the state at
// the chunk's start and dS' the gradient of the state at its end:
//   A = strictLower(diag(beta) (K^ K^T * Gam)),  T = (I + A)^-1
//   W = T diag(beta gam) K^,  Ut = T diag(beta) V,  U = Ut - W S
//   P = scale (Q^ K^T * Gam * lower-incl)
//   Y = scale diag(gam) Q^ S + P U,   S' = gC S + K^T diag(gC / gam) U
// The reverse chain is the transpose of the forward one:
//   dU = diag(gC / gam) K^ dS' + P^T dY
//   dS = gC dS' + scale Q^T diag(gam) dY - W^T dU
// and every other gradient is local to the chunk once S, dS' and dU are known:
//   dV = diag(beta) T^T dU,  dW = -dU S^T,  dT = dU (diag(beta) V)^T + dW (diag(beta gam) K^)^T,
//   dA = -T^T dT T^T (strictly lower),  dP = dY U^T (lower-incl),
//   dq^ = scale diag(gam) dY S^T + (scale dP * Gam) K^,
//   dk^ = diag(beta gam) T^T dW + diag(gC / gam) U dS'^T + E K^ + E^T K^ + (scale dP * Gam)^T Q^
//         with E = dA * beta_i Gam_ij,
//   dbeta, d ln(alpha) (through gam, gC and Gam: d Lg_i collects (dA * A + dP * P) row i minus
//   column i, and the gam / gC terms; d ln alpha is its reverse cumsum), and the L2-norm
//   backward dq = rq (dq^ - q^ (q^ . dq^)).
// Tokens past the end of a sequence are zero rows with alpha = 1, beta = 0, which makes them exact
// identity steps, so no masks are needed.  gam can be far below 1 (it decays over the whole
// chunk): the decay gradients are carried as gam_i d gam_i and gC d gC, and gC / gam_i as
// e^(Lg_last - Lg_i), so that no term divides by gam.
//
// Kernels (one launch each, in stream order):
//   bwdc_prep   one CTA per (chunk, head): norms, Lg, A / beta (kept for dbeta), P, T, W, Ut
//               (bwdc_prep_tc for bf16 inputs, which also writes split images of -W and P)
//   bwdc_fwd    one CTA per (sequence, head, state slice): S^c and U of every chunk
//               (bwdc_fwd_tc for bf16 inputs: 64-column slices; bwdc_fwd: 32)
//   bwdc_rev    one CTA per (sequence, head, state slice): dS' and dU of every chunk, dS0
//               (bwdc_rev_tc for bf16 inputs: 64-column slices; bwdc_rev: 32)
//   bwdc_local  one CTA per (chunk, head): all gradients of the chunk's tokens
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

constexpr int kCB = 64;   // chunk length
constexpr int kNVB = 32;  // state columns per chain CTA
constexpr int kL64 = 68;  // row stride (floats) of 64 x 64 shared matrices

// Workspace arrays (float offsets); one record per (sequence, chunk, head), r = (b nch + c) H + h.
struct BwdChunkWs {
    size_t W, Ut, P, Tm, At, SC, S, U, dSp, dU, Wi, Pi, total;
};
BwdChunkWs bwdc_ws(int B, int T, int H, int D) {
    const size_t nch = (size_t)(T + kCB - 1) / kCB, R = (size_t)B * nch * H;
    BwdChunkWs w{};
    size_t o = 0;
    w.W = o;   o += R * kCB * D;
    w.Ut = o;  o += R * kCB * D;
    w.P = o;   o += R * kCB * kCB;
    w.Tm = o;  o += R * kCB * kCB;
    w.At = o;  o += R * kCB * kCB;
    w.SC = o;  o += R * 256;  // rq[64], rk[64], Lg[64], beta[64]
    w.S = o;   o += R * D * D;
    w.U = o;   o += R * kCB * D;
    w.dSp = o; o += R * D * D;
    w.dU = o;  o += R * kCB * D;
    w.Wi = o;  o += R * kCB * D;    // -W as split bf16 images hi, lo (64 x D each)
    w.Pi = o;  o += R * kCB * kCB;  // P as split bf16 images hi, lo (64 x 64 each)
    w.total = o;
    return w;
}

// acc[n] += sum_k a[k * as] * b[k * bs + n], n < NC (rows of b 16-byte aligned)
template <int NC>
__device__ __forceinline__ void mm_nn(float* acc, const float* a, int as, const float* b, int bs, int K) {
#pragma unroll 2
    for (int k = 0; k < K; ++k) {
        const float x = a[k * as];
        const float4* br = reinterpret_cast<const float4*>(b + (size_t)k * bs);
#pragma unroll
        for (int n = 0; n < NC / 4; ++n) {
            const float4 y = br[n];
            acc[4 * n + 0] = fmaf(x, y.x, acc[4 * n + 0]);
            acc[4 * n + 1] = fmaf(x, y.y, acc[4 * n + 1]);
            acc[4 * n + 2] = fmaf(x, y.z, acc[4 * n + 2]);
            acc[4 * n + 3] = fmaf(x, y.w, acc[4 * n + 3]);
        }
    }
}

__device__ __forceinline__ size_t tok_off(int b, int t, int h, int T, int H) {
    return ((size_t)b * T + t) * H + h;
}

// 8 consecutive elements (16-byte aligned) -> fp32
__device__ __forceinline__ void ld8(const __nv_bfloat16* p, float* o) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        o[2 * j] = __uint_as_float(w[j] << 16);
        o[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
}
__device__ __forceinline__ void ld8(const float* p, float* o) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void st8(float* p, const float* x, float s) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0] * s, x[1] * s, x[2] * s, x[3] * s);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4] * s, x[5] * s, x[6] * s, x[7] * s);
}

// Rows t0 .. t0 + 63 of a [B, T, H, D] tensor (zero past nv) -> 64 x D fp32 shared tile of row
// stride LD, each row scaled by scl[i] (nullptr: 1); NT threads, all loads issued before any store.
template <int D, int LD, int NT, typename Tin>
__device__ __forceinline__ void load_rows(float* dst, const Tin* src, int b, int t0, int nv, int h, int T,
                                          int H, const float* scl, int tid) {
    constexpr int PER = kCB * D / 8 / NT;  // 8-element groups per thread
    static_assert(PER * NT * 8 == kCB * D, "tile split");
    float x[PER][8];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = (tid + u * NT) * 8, i = e / D, m = e % D;
        if (i < nv) ld8(src + tok_off(b, t0 + i, h, T, H) * D + m, x[u]);
        else {
#pragma unroll
            for (int j = 0; j < 8; ++j) x[u][j] = 0.f;
        }
    }
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = (tid + u * NT) * 8, i = e / D, m = e % D;
        st8(dst + i * LD + m, x[u], scl ? scl[i] : 1.f);
    }
}
// 64 x D fp32 record array (row-major) -> shared tile of row stride LD
template <int D, int LD, int NT>
__device__ __forceinline__ void load_rec(float* dst, const float* src, int tid) {
    constexpr int PER = kCB * D / 4 / NT;
    float4 x[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) x[u] = reinterpret_cast<const float4*>(src)[tid + u * NT];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = (tid + u * NT) * 4;
        *reinterpret_cast<float4*>(dst + (e / D) * LD + e % D) = x[u];
    }
}

// fp32 -> tf32 (round to nearest, ties away), for the tensor-core products
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// x rounded to tf32 (nearest, ties away) as an fp32 value with the low 13 bits clear
__device__ __forceinline__ float rtf(float x) { return __uint_as_float(to_tf32(x) & 0xffffe000u); }
__device__ __forceinline__ void mma_tf32(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// acc[t] (16 x 8 tile t at rows r0.., columns c0 + 8 t ..) += A B over k < K, tf32
template <int CT, typename FA, typename FB>
__device__ __forceinline__ void wmma_acc(float (&acc)[CT][4], int K, int r0, int c0, FA a, FB b, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t a0 = to_tf32(a(r0 + gid, k0 + tig)), a1 = to_tf32(a(r0 + gid + 8, k0 + tig));
        const uint32_t a2 = to_tf32(a(r0 + gid, k0 + tig + 4)), a3 = to_tf32(a(r0 + gid + 8, k0 + tig + 4));
#pragma unroll
        for (int t = 0; t < CT; ++t) {
            const int n = c0 + 8 * t + gid;
            mma_tf32(acc[t], a0, a1, a2, a3, to_tf32(b(k0 + tig, n)), to_tf32(b(k0 + tig + 4, n)));
        }
    }
}
template <int CT>
__device__ __forceinline__ void zero_acc(float (&acc)[CT][4]) {
#pragma unroll
    for (int t = 0; t < CT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
}
// sum over the 4 lanes of a quad (the lanes that share a tile row)
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}

// acc[t] += A B like wmma_acc, with every operand split into its tf32 value and a tf32
// remainder: A_lo B_hi + A_hi B_lo + A_hi B_hi.  That keeps the products' relative error near
// 2^-22 instead of tf32's 2^-11, for the products whose rounding accumulates along a chain.
template <int CT, typename FA, typename FB>
__device__ __forceinline__ void wmma_acc3(float (&acc)[CT][4], int K, int r0, int c0, FA a, FB b, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 8) {
        const float af[4] = {a(r0 + gid, k0 + tig), a(r0 + gid + 8, k0 + tig), a(r0 + gid, k0 + tig + 4),
                             a(r0 + gid + 8, k0 + tig + 4)};
        // the high part's low 13 bits are cleared so that it reads back as the exact tf32 value
        uint32_t ah[4], al[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            ah[e] = to_tf32(af[e]) & 0xffffe000u;
            al[e] = to_tf32(af[e] - __uint_as_float(ah[e]));
        }
#pragma unroll
        for (int t = 0; t < CT; ++t) {
            const int n = c0 + 8 * t + gid;
            const float b0 = b(k0 + tig, n), b1 = b(k0 + tig + 4, n);
            const uint32_t bh0 = to_tf32(b0) & 0xffffe000u, bh1 = to_tf32(b1) & 0xffffe000u;
            const uint32_t bl0 = to_tf32(b0 - __uint_as_float(bh0)), bl1 = to_tf32(b1 - __uint_as_float(bh1));
            mma_tf32(acc[t], al[0], al[1], al[2], al[3], bh0, bh1);
            mma_tf32(acc[t], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
            mma_tf32(acc[t], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
        }
    }
}

// ============================================================================ bwdc_prep
template <int D>
struct PrepB {
    static constexpr int LD = D + 4;
    static constexpr int BYTES = (2 * kCB * LD + 2 * kCB * kL64 + 5 * kCB + 768) * 4;  // two CTAs per SM
};

template <int D, typename Tin>
__global__ void __launch_bounds__(256, 2) bwdc_prep(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                 const Tin* __restrict__ v, const float* __restrict__ alpha,
                                                 const float* __restrict__ beta, float* __restrict__ ws,
                                                 const BwdChunkWs w, int T, int H, int nch, float scale,
                                                 int l2norm, const float* __restrict__ A_log,
                                                 const float* __restrict__ b_alpha) {
    constexpr int LD = PrepB<D>::LD;
    extern __shared__ float smf[];
    float* qh = smf;
    float* kh = qh + kCB * LD;
    float* vs = qh;  // V takes Q's place once the Gram products are done
    float* Am = kh + kCB * LD;
    float* Tm = Am + kCB * kL64;
    float* rq = Tm + kCB * kL64;
    float* rk = rq + kCB;
    float* Lg = rk + kCB;
    float* be = Lg + kCB;
    float* gam = be + kCB;
    float* Xs = gam + kCB;  // 3 x 16 x 16 block products
    const size_t r = blockIdx.x;
    const int h = (int)(r % H);
    const int gr = (int)(r / H);
    const int c = gr % nch, b = gr / nch;
    const int t0 = c * kCB, nv = min(kCB, T - t0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    load_rows<D, LD, 256>(qh, q, b, t0, nv, h, T, H, nullptr, tid);
    load_rows<D, LD, 256>(kh, k, b, t0, nv, h, T, H, nullptr, tid);
    if (tid < kCB) {
        const size_t o = tok_off(b, t0 + tid, h, T, H);
        float bt = 0.f, lg = 0.f;  // rows past the end: beta = 0, alpha = 1
        if (tid < nv) {
            // gated form: alpha, beta hold the logits of eqs. (9)-(10)
            bt = A_log ? gate_sigmoid(beta[o]) : beta[o];
            lg = A_log ? gate_log_decay(alpha[o], A_log[h], b_alpha[h]) : logf(alpha[o]);
        }
        be[tid] = bt;
        Lg[tid] = lg;
    }
    __syncthreads();
    for (int rr = 0; rr < 16; ++rr) {  // warp w: rows 16 w .. 16 w + 15 of [q; k]
        const int row = warp * 16 + rr;
        const float* x = row < kCB ? qh + row * LD : kh + (row - kCB) * LD;
        float s = 0.f;
        for (int m = lane; m < D; m += 32) s = fmaf(x[m], x[m], s);
        s = warp_sum(s);
        if (lane == 0) {
            const float rn = l2norm ? 1.0f / sqrtf(s + kNormEps) : 1.0f;
            if (row < kCB) rq[row] = rn; else rk[row - kCB] = rn;
        }
    }
    if (tid == 0) {
        float acc = 0.f;
        for (int i = 0; i < kCB; ++i) { acc += Lg[i]; Lg[i] = acc; }
    }
    __syncthreads();
    if (tid < kCB) gam[tid] = expf(Lg[tid]);
    for (int e = tid; e < kCB * D; e += 256) {
        const int i = e / D, m = e % D;
        qh[i * LD + m] *= rq[i];
        kh[i * LD + m] *= rk[i];
    }
    __syncthreads();
    // A / beta and P: K^ K^T and Q^ K^T as 16 x 8 tensor-core tiles (tf32 operands, fp32
    // accumulation); warp w owns rows 16 (w & 3) .. +15 and columns 32 (w >> 2) .. +31, and lane
    // (gid, tig) of tile t holds rows gid, gid + 8 and columns 8 t + 2 tig, 8 t + 2 tig + 1
    {
        const int gid = lane >> 2, tig = lane & 3;
        const int r0 = (warp & 3) * 16, c0 = (warp >> 2) * 32;
        const float* khp = kh;
        const float* qhp = qh;
        float kk[4][4], qk[4][4];
        zero_acc(kk);
        zero_acc(qk);
        auto bKt = [khp](int k2, int n) { return khp[n * LD + k2]; };
        wmma_acc(kk, D, r0, c0, [khp](int i, int k2) { return khp[i * LD + k2]; }, bKt, lane);
        wmma_acc(qk, D, r0, c0, [qhp](int i, int k2) { return qhp[i * LD + k2]; }, bKt, lane);
        float* Atg = ws + w.At + r * kCB * kCB;
        float* Pg = ws + w.P + r * kCB * kCB;
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = r0 + gid + 8 * hh, j = c0 + 8 * t + 2 * tig;
                float at[2], pp[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const float gm = expf(fminf(Lg[i] - Lg[j + u], 0.f));
                    at[u] = j + u < i ? kk[t][2 * hh + u] * gm : 0.f;
                    pp[u] = j + u <= i ? scale * qk[t][2 * hh + u] * gm : 0.f;
                    Am[i * kL64 + j + u] = be[i] * at[u];
                }
                *reinterpret_cast<float2*>(Atg + i * kCB + j) = make_float2(at[0], at[1]);
                *reinterpret_cast<float2*>(Pg + i * kCB + j) = make_float2(pp[0], pp[1]);
            }
    }
    __syncthreads();
    load_rows<D, LD, 256>(vs, v, b, t0, nv, h, T, H, nullptr, tid);  // Q is no longer read
    // T = (I + A)^-1 by 16 x 16 blocks: the diagonal blocks by forward substitution (one column
    // per thread), then T_ij = -T_ii sum_{j <= m < i} A_im T_mj for block distance 1, 2, 3
    if (tid < kCB) {
        const int bb = tid >> 4, m = tid & 15, o = 16 * bb;
        for (int ii = 0; ii < 16; ++ii) {
            float acc = 0.f;
            for (int j = 0; j < ii; ++j) acc = fmaf(Am[(o + ii) * kL64 + o + j], Tm[(o + j) * kL64 + o + m], acc);
            Tm[(o + ii) * kL64 + o + m] = ii < m ? 0.f : (ii == m ? 1.f : -acc);
        }
    }
    for (int e = tid; e < kCB * kCB; e += 256) {  // zero the blocks above the diagonal
        const int ii = e / kCB, j = e % kCB;
        if ((j >> 4) > (ii >> 4)) Tm[ii * kL64 + j] = 0.f;
    }
    __syncthreads();
    for (int dd = 1; dd < 4; ++dd) {
        const int npair = 4 - dd;
        for (int e = tid; e < npair * 256; e += 256) {  // X = sum_m A_im T_mj
            const int pb = e >> 8, ii = (e >> 4) & 15, j = e & 15;
            const int bi = pb + dd, bj = pb;
            float acc = 0.f;
            for (int m = 16 * bj; m < 16 * bi; ++m)
                acc = fmaf(Am[(16 * bi + ii) * kL64 + m], Tm[m * kL64 + 16 * bj + j], acc);
            Xs[e] = acc;
        }
        __syncthreads();
        for (int e = tid; e < npair * 256; e += 256) {  // T_ij = -T_ii X
            const int pb = e >> 8, ii = (e >> 4) & 15, j = e & 15;
            const int bi = pb + dd, bj = pb;
            float acc = 0.f;
            for (int m = 0; m < 16; ++m) acc = fmaf(Tm[(16 * bi + ii) * kL64 + 16 * bi + m], Xs[(pb << 8) + (m << 4) + j], acc);
            Tm[(16 * bi + ii) * kL64 + 16 * bj + j] = -acc;
        }
        __syncthreads();
    }
    for (int e = tid; e < kCB * kCB; e += 256) ws[w.Tm + r * kCB * kCB + e] = rtf(Tm[(e / kCB) * kL64 + e % kCB]);
    // W = T diag(beta gam) K^, Ut = T diag(beta) V: 64 x D tensor-core tiles (tf32, fp32
    // accumulation), the diagonal scales folded into the B operand; warp w owns rows
    // 16 (w & 3) .. +15 and columns (D / 2)(w >> 2) .. +D/2-1
    {
        constexpr int CT = D / 16;
        const int gid = lane >> 2, tig = lane & 3;
        const int r0 = (warp & 3) * 16, c0 = (warp >> 2) * (D / 2);
        const float* Tp = Tm;
        const float* khp = kh;
        const float* vp = vs;
        const float* bep = be;
        const float* gp = gam;
        float wa[CT][4], ua[CT][4];
        zero_acc(wa);
        zero_acc(ua);
        auto aT = [Tp](int i, int j) { return Tp[i * kL64 + j]; };
        wmma_acc(wa, kCB, r0, c0, aT,
                 [bep, gp, khp](int j, int n) { return bep[j] * gp[j] * khp[j * LD + n]; }, lane);
        wmma_acc(ua, kCB, r0, c0, aT, [bep, vp](int j, int n) { return bep[j] * vp[j * LD + n]; },
                 lane);
        float* Wg = ws + w.W + r * kCB * D;
        float* Ug = ws + w.Ut + r * kCB * D;
#pragma unroll
        for (int t = 0; t < CT; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const size_t o = (size_t)(r0 + gid + 8 * hh) * D + c0 + 8 * t + 2 * tig;
                *reinterpret_cast<float2*>(Wg + o) = make_float2(wa[t][2 * hh], wa[t][2 * hh + 1]);
                *reinterpret_cast<float2*>(Ug + o) = make_float2(ua[t][2 * hh], ua[t][2 * hh + 1]);
            }
    }
    if (tid < kCB) {
        float* sc = ws + w.SC + r * 256;
        sc[tid] = rq[tid]; sc[64 + tid] = rk[tid]; sc[128 + tid] = Lg[tid]; sc[192 + tid] = be[tid];
    }
}

// hi = bf16(x), lo = bf16(x - hi) for a pair, as two packed bf16x2 words
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// ---------------------------------------------------------------------------- bwdc_prep_tc
// The same chunk matrices for bf16 inputs, with the products on tcgen05 (kind::f16, M = 64
// tiles, fp32 accumulators in TMEM).  q, k and v arrive by TMA as 128-byte-swizzled bf16 panels
// (64 features x 64 tokens per box), unnormalised: K K^T and Q K^T are exact in fp32 from bf16
// operands, and the row scales rq, rk enter in the epilogue.  The products with T, W and Ut,
// take T diag(beta gam rk) and T diag(beta) as split images hi + lo (hi = bf16(x), lo =
// bf16(x - hi): relative error below 2^-16, finer than tf32) against k and v as MN-major
// operands, two MMAs each.  Eight warps: warp w reads the accumulator rows 16 (w % 4) .. +15 of
// its TMEM lane quarter in the m16n8 fragment layout, columns by halves (w / 4).
// byte offset of element (r, m) in a bf16 panel tile of R rows (64 elements per 128-byte row)
__device__ __forceinline__ uint32_t bpan(int R, int r, int m) {
    return (uint32_t)((((m >> 6) * R + r) << 7) + (((((m & 63) >> 3) ^ (r & 7))) << 4) + ((m & 7) << 1));
}
template <int D>
struct PrepTC {
    static constexpr int BF = kCB * D * 2;                 // a 64 x D bf16 tile
    static constexpr int QV = 0, KP = QV + BF, TI = KP + BF;  // Q (then V), K, four 64 x 64 images
    static constexpr int AM = TI + 4 * 8192, TM = AM + kCB * kL64 * 4, XS = TM + kCB * kL64 * 4;
    static constexpr int SCAL = XS + 768 * 4;             // rq, rk, Lg, beta, gam
    static constexpr int BAR = SCAL + 5 * kCB * 4;
    static constexpr int MISC = BAR + 8 * 8;
    static constexpr int BYTES = MISC + 16 + 1024;        // two CTAs per SM
    static constexpr uint32_t TCOLS = 256;
};
enum PrepTcBar { PT_IN = 0, PT_V, PT_M1, PT_M2, PT_DRAIN };

template <int D>
__global__ void __launch_bounds__(256, 2) bwdc_prep_tc(const float* __restrict__ alpha,
                                                    const float* __restrict__ beta, float* __restrict__ ws,
                                                    const BwdChunkWs w, int T, int H, int nch, float scale,
                                                    int l2norm, const float* __restrict__ A_log,
                                                    const float* __restrict__ b_alpha, int* __restrict__ status,
                                                    const __grid_constant__ CUtensorMap map_q,
                                                    const __grid_constant__ CUtensorMap map_k,
                                                    const __grid_constant__ CUtensorMap map_v) {
    using L = PrepTC<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* Am = reinterpret_cast<float*>(sm + L::AM);
    float* Tm = reinterpret_cast<float*>(sm + L::TM);
    float* Xs = reinterpret_cast<float*>(sm + L::XS);
    float* rq = reinterpret_cast<float*>(sm + L::SCAL);
    float* rk = rq + kCB;
    float* Lg = rk + kCB;
    float* be = Lg + kCB;
    float* gam = be + kCB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* never = reinterpret_cast<volatile int*>(sm + L::MISC + 8);
    const size_t r = blockIdx.x;
    const int h = (int)(r % H);
    const int gr = (int)(r / H);
    const int c = gr % nch, b = gr / nch;
    const int t0 = c * kCB, nv = min(kCB, T - t0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int r0 = (warp & 3) * 16;
    const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t sa = sm100::smem_u32(sm);
    const int z0 = b * T + t0;  // token row of the chunk's first token in the [B T, H, D] maps

    if (tid == 0) {
        for (int i = 0; i < 8; ++i) sm100::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        *never = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tmap(&map_q);
        sm100::prefetch_tmap(&map_k);
        sm100::prefetch_tmap(&map_v);
    }
    if (warp == 0) sm100::tmem_alloc(tmem_slot, L::TCOLS);
    if (tid < kCB) {
        const size_t o = tok_off(b, t0 + tid, h, T, H);
        float bt = 0.f, lg = 0.f;  // rows past the end: beta = 0, alpha = 1
        if (tid < nv) {
            // gated form: alpha, beta hold the logits of eqs. (9)-(10)
            bt = A_log ? gate_sigmoid(beta[o]) : beta[o];
            lg = A_log ? gate_log_decay(alpha[o], A_log[h], b_alpha[h]) : logf(alpha[o]);
        }
        be[tid] = bt;
        Lg[tid] = lg;
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t copies = 0;  // (thread 0) copy barriers armed
    if (tid == 0) {
        copies |= 1u << PT_IN;
        sm100::mbar_arrive_expect_tx(&bars[PT_IN], 2u * L::BF);
        for (int p = 0; p < D / 64; ++p) {
            sm100::tma_load_3d(sm + L::QV + p * 8192, &map_q, 64 * p, h, z0, &bars[PT_IN]);
            sm100::tma_load_3d(sm + L::KP + p * 8192, &map_k, 64 * p, h, z0, &bars[PT_IN]);
        }
    }
    auto wait_bar = [&](int i) {
        bool okw = sm100::mbar_wait_warp(&bars[i], 0, abort_flag);
        okw = __syncthreads_and(okw) != 0;
        sm100::tc_fence_after();
        return okw;
    };
    bool ok = wait_bar(PT_IN);
    if (ok) {
        // rows past the end of the sequence are zero (the box may have read the next one's)
        if (nv < kCB)
            for (int e = tid; e < 2 * (D / 64) * (kCB - nv) * 8; e += 256) {
                const int ch = e & 7, rowi = nv + ((e >> 3) % (kCB - nv)), pp = (e >> 3) / (kCB - nv);
                *reinterpret_cast<uint4*>(sm + (pp & 1 ? L::KP : L::QV) + (pp >> 1) * 8192 + rowi * 128 + ch * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
        __syncthreads();
        // sums of squares: thread t takes half (t % 2) of row t / 2 of [q; k]
        {
            const int row = tid >> 1, half = tid & 1;
            const uint8_t* tile = sm + (row < kCB ? L::QV : L::KP);
            const int i = row & (kCB - 1);
            float s = 0.f;
#pragma unroll
            for (int u = 0; u < D / 16; ++u) {
                const int m = half * (D / 2) + 8 * u;
                const uint4 x = *reinterpret_cast<const uint4*>(tile + bpan(kCB, i, m));
                const uint32_t wv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float lo = __uint_as_float(wv[j] << 16), hi = __uint_as_float(wv[j] & 0xffff0000u);
                    s = fmaf(lo, lo, fmaf(hi, hi, s));
                }
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            if (half == 0) {
                const float rn = l2norm ? 1.0f / sqrtf(s + kNormEps) : 1.0f;
                if (row < kCB) rq[i] = rn; else rk[i] = rn;
            }
        }
        if (warp == 0) {  // inclusive cumsum of ln alpha: lane l holds 2 l, 2 l + 1
            const float a0 = Lg[2 * lane], a1 = Lg[2 * lane + 1];
            float pre = a0 + a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, pre, o);
                if (lane >= o) pre += y;
            }
            Lg[2 * lane + 1] = pre;
            Lg[2 * lane] = pre - a1;
            gam[2 * lane + 1] = expf(pre);
            gam[2 * lane] = expf(pre - a1);
        }
        sm100::fence_proxy_async_smem();
        sm100::tc_fence_before();
        __syncthreads();
        sm100::tc_fence_after();
        if (tid == 0) {
            constexpr uint32_t ID = sm100::idesc_bf16(64, 64, false, false);
            for (int kb = 0; kb < D / 64; ++kb)
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t off = kb * 8192 + kk * 32;
                    const uint64_t dk_ = sm100::sdesc(sa + L::KP + off, 16, 1024);
                    const uint64_t dq_ = sm100::sdesc(sa + L::QV + off, 16, 1024);
                    sm100::mma_bf16(tmem + 0, dk_, dk_, ID, (kb | kk) != 0);    // K K^T
                    sm100::mma_bf16(tmem + 64, dq_, dk_, ID, (kb | kk) != 0);   // Q K^T
                }
            sm100::mma_commit(&bars[PT_M1]);
        }
        ok = wait_bar(PT_M1);
    }
    if (ok) {
        if (tid == 0) {  // V into Q's place (Q is read no more)
            copies |= 1u << PT_V;
            sm100::mbar_arrive_expect_tx(&bars[PT_V], (uint32_t)L::BF);
            for (int p = 0; p < D / 64; ++p)
                sm100::tma_load_3d(sm + L::QV + p * 8192, &map_v, 64 * p, h, z0, &bars[PT_V]);
        }
        // A / beta and P from the fragments of K K^T and Q K^T
        float kk4[4][4], qk4[4][4];
        const int c0 = (warp >> 2) * 32;
        sm100::tmem_ld_frag<4>(tmem + lq + 0 + c0, &kk4[0][0]);
        sm100::tmem_ld_frag<4>(tmem + lq + 64 + c0, &qk4[0][0]);
        float* Atg = ws + w.At + r * kCB * kCB;
        float* Pg = ws + w.P + r * kCB * kCB;
        __nv_bfloat16* Pig = reinterpret_cast<__nv_bfloat16*>(ws + w.Pi) + r * 2 * kCB * kCB;
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = r0 + gid + 8 * hh, j = c0 + 8 * t + 2 * tig;
                float at[2], pp[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const float gm = expf(fminf(Lg[i] - Lg[j + u], 0.f));
                    at[u] = j + u < i ? rk[i] * rk[j + u] * kk4[t][2 * hh + u] * gm : 0.f;
                    pp[u] = j + u <= i ? scale * rq[i] * rk[j + u] * qk4[t][2 * hh + u] * gm : 0.f;
                    Am[i * kL64 + j + u] = be[i] * at[u];
                }
                *reinterpret_cast<float2*>(Atg + i * kCB + j) = make_float2(at[0], at[1]);
                *reinterpret_cast<float2*>(Pg + i * kCB + j) = make_float2(pp[0], pp[1]);
                uint32_t phi, plo;  // P's split images for the reverse chain
                split2(pp[0], pp[1], phi, plo);
                *reinterpret_cast<uint32_t*>(Pig + i * kCB + j) = phi;
                *reinterpret_cast<uint32_t*>(Pig + (kCB + i) * kCB + j) = plo;
            }
        __syncthreads();
        // T = (I + A)^-1 by 16 x 16 blocks: the diagonal blocks by forward substitution (one
        // column per thread), then T_ij = -T_ii sum_{j <= m < i} A_im T_mj for block distance 1, 2, 3
        if (tid < kCB) {
            const int bb = tid >> 4, m = tid & 15, o = 16 * bb;
            for (int ii = 0; ii < 16; ++ii) {
                float acc = 0.f;
                for (int j = 0; j < ii; ++j) acc = fmaf(Am[(o + ii) * kL64 + o + j], Tm[(o + j) * kL64 + o + m], acc);
                Tm[(o + ii) * kL64 + o + m] = ii < m ? 0.f : (ii == m ? 1.f : -acc);
            }
        }
        for (int e = tid; e < kCB * kCB; e += 256) {  // zero the blocks above the diagonal
            const int ii = e / kCB, j = e % kCB;
            if ((j >> 4) > (ii >> 4)) Tm[ii * kL64 + j] = 0.f;
        }
        __syncthreads();
        for (int dd = 1; dd < 4; ++dd) {
            const int npair = 4 - dd;
            for (int e = tid; e < npair * 256; e += 256) {  // X = sum_m A_im T_mj
                const int pb = e >> 8, ii = (e >> 4) & 15, j = e & 15;
                const int bi = pb + dd, bj = pb;
                float acc = 0.f;
                for (int m = 16 * bj; m < 16 * bi; ++m)
                    acc = fmaf(Am[(16 * bi + ii) * kL64 + m], Tm[m * kL64 + 16 * bj + j], acc);
                Xs[e] = acc;
            }
            __syncthreads();
            for (int e = tid; e < npair * 256; e += 256) {  // T_ij = -T_ii X
                const int pb = e >> 8, ii = (e >> 4) & 15, j = e & 15;
                const int bi = pb + dd, bj = pb;
                float acc = 0.f;
                for (int m = 0; m < 16; ++m) acc = fmaf(Tm[(16 * bi + ii) * kL64 + 16 * bi + m], Xs[(pb << 8) + (m << 4) + j], acc);
                Tm[(16 * bi + ii) * kL64 + 16 * bj + j] = -acc;
            }
            __syncthreads();
        }
        // T (tf32-rounded, for the local-gradient kernel) and the split images of
        // T diag(beta gam rk) and T diag(beta): thread -> (row, 8-column group)
        float* Tg = ws + w.Tm + r * kCB * kCB;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + 256 * u, i = e >> 3, j0 = (e & 7) * 8;
            float tv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) tv[j] = Tm[i * kL64 + j0 + j];
            *reinterpret_cast<float4*>(Tg + i * kCB + j0) = make_float4(rtf(tv[0]), rtf(tv[1]), rtf(tv[2]), rtf(tv[3]));
            *reinterpret_cast<float4*>(Tg + i * kCB + j0 + 4) = make_float4(rtf(tv[4]), rtf(tv[5]), rtf(tv[6]), rtf(tv[7]));
            uint32_t wh[4], wl[4], uh[4], ul[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                float x2[2], y2[2];
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    const int j = j0 + 2 * jj + s2;
                    x2[s2] = tv[2 * jj + s2] * be[j] * gam[j] * rk[j];
                    y2[s2] = tv[2 * jj + s2] * be[j];
                }
                const __nv_bfloat162 xh = __floats2bfloat162_rn(x2[0], x2[1]);
                const __nv_bfloat162 yh = __floats2bfloat162_rn(y2[0], y2[1]);
                const float2 xf = __bfloat1622float2(xh), yf = __bfloat1622float2(yh);
                const __nv_bfloat162 xl = __floats2bfloat162_rn(x2[0] - xf.x, x2[1] - xf.y);
                const __nv_bfloat162 yl = __floats2bfloat162_rn(y2[0] - yf.x, y2[1] - yf.y);
                wh[jj] = *reinterpret_cast<const uint32_t*>(&xh);
                wl[jj] = *reinterpret_cast<const uint32_t*>(&xl);
                uh[jj] = *reinterpret_cast<const uint32_t*>(&yh);
                ul[jj] = *reinterpret_cast<const uint32_t*>(&yl);
            }
            const uint32_t off = bpan(kCB, i, j0);
            *reinterpret_cast<uint4*>(sm + L::TI + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
            *reinterpret_cast<uint4*>(sm + L::TI + 8192 + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
            *reinterpret_cast<uint4*>(sm + L::TI + 16384 + off) = make_uint4(uh[0], uh[1], uh[2], uh[3]);
            *reinterpret_cast<uint4*>(sm + L::TI + 24576 + off) = make_uint4(ul[0], ul[1], ul[2], ul[3]);
        }
        sm100::fence_proxy_async_smem();
        sm100::tc_fence_before();
        ok = wait_bar(PT_V);  // (a barrier for every thread, then the copy of V)
        if (ok && tid == 0) {
            // W = T diag(beta gam rk) k and Ut = T diag(beta) v, k and v as MN-major operands
            constexpr uint32_t ID = sm100::idesc_bf16(64, D, false, true);
            for (int half = 0; half < 2; ++half)
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ta = sm100::sdesc(sa + L::TI + half * 8192 + kk * 32, 16, 1024);
                    const uint64_t tb = sm100::sdesc(sa + L::TI + 16384 + half * 8192 + kk * 32, 16, 1024);
                    const uint64_t kb = sm100::sdesc(sa + L::KP + kk * 2048, 8192, 1024);
                    const uint64_t vb = sm100::sdesc(sa + L::QV + kk * 2048, 8192, 1024);
                    sm100::mma_bf16(tmem + 0, ta, kb, ID, (half | kk) != 0);
                    sm100::mma_bf16(tmem + D, tb, vb, ID, (half | kk) != 0);
                }
            sm100::mma_commit(&bars[PT_M2]);
        }
        if (ok) ok = wait_bar(PT_M2);
    }
    if (ok) {
        float* Wg = ws + w.W + r * kCB * D;
        float* Ug = ws + w.Ut + r * kCB * D;
        __nv_bfloat16* Wig = reinterpret_cast<__nv_bfloat16*>(ws + w.Wi) + r * 2 * kCB * D;
        const int c0 = (warp >> 2) * (D / 2);
#pragma unroll
        for (int g = 0; g < D / 64; ++g) {  // 32 columns (4 tiles) at a time
            float wa[4][4], ua[4][4];
            sm100::tmem_ld_frag<4>(tmem + lq + 0 + c0 + 32 * g, &wa[0][0]);
            sm100::tmem_ld_frag<4>(tmem + lq + D + c0 + 32 * g, &ua[0][0]);
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const size_t o = (size_t)(r0 + gid + 8 * hh) * D + c0 + 32 * g + 8 * t + 2 * tig;
                    *reinterpret_cast<float2*>(Wg + o) = make_float2(wa[t][2 * hh], wa[t][2 * hh + 1]);
                    *reinterpret_cast<float2*>(Ug + o) = make_float2(ua[t][2 * hh], ua[t][2 * hh + 1]);
                    uint32_t whi, wlo;  // -W's split images for the reverse chain
                    split2(-wa[t][2 * hh], -wa[t][2 * hh + 1], whi, wlo);
                    *reinterpret_cast<uint32_t*>(Wig + o) = whi;
                    *reinterpret_cast<uint32_t*>(Wig + kCB * D + o) = wlo;
                }
        }
        if (tid < kCB) {
            float* sc = ws + w.SC + r * 256;
            sc[tid] = rq[tid]; sc[64 + tid] = rk[tid]; sc[128 + tid] = Lg[tid]; sc[192 + tid] = be[tid];
        }
    }
    if (!ok && tid == 0) {
        record_status(status, GDN_ERR_TIMEOUT);
        sm100::mma_commit(&bars[PT_DRAIN]);
        sm100::mbar_wait(&bars[PT_DRAIN], 0, never, 100000000ull);
        for (int i = PT_IN; i <= PT_V; ++i)
            if (copies & (1u << i)) sm100::mbar_wait(&bars[i], 0, never, 100000000ull);
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, L::TCOLS);
    }
}

// ---------------------------------------------------------------------------- bwdc_fwd_tc
// The forward chain for bf16 inputs on tcgen05 (kind::f16): one CTA per (sequence, head,
// 64-column slice of the state), 256 threads, two per SM.  Per chunk, with S the state slice at
// the chunk's start (fp32, in registers: thread = row, 32 columns):
//   (i)   D1 = (-W) S  (-W's split images from bwdc_prep_tc; S as split images; hi hi + hi lo + lo hi)
//   (ii)  U = Ut + D1 -> workspace, and U' = diag(dec rk) U as split images
//   (iii) D2 = k^T U'  (k exact in bf16, as the MN-major operand)
//   (iv)  S <- gC S + D2
// The -W images and the chunk scalars for chunk c+1 are copied as soon as (i) and the U epilogue
// are done with theirs; k for chunk c+1 once (iii) is.
template <int D>
struct FwdTC {
    static constexpr int BF = kCB * D * 2, T8 = kCB * kCB * 2, SB = D * kCB * 2;
    static constexpr int KP = 0, WH = KP + BF, WL = WH + BF, SH = WL + BF, SL = SH + SB, UH = SL + SB,
                         UL = UH + T8;
    static constexpr int SC = UL + T8;              // the chunk's rq, rk, Lg, beta (copied)
    static constexpr int SCL = SC + 4 * kCB * 4;    // dec rk
    static constexpr int BAR = SCL + kCB * 4;
    static constexpr int MISC = BAR + 8 * 8;
    static constexpr int BYTES = MISC + 16 + 1024;  // two CTAs per SM
    static constexpr uint32_t TD1 = 0, TD2 = 64, TCOLS = 128;
};
enum FwdBar { FB_A = 0, FB_K, FB_M1, FB_M2, FB_DRAIN };

template <int D>
__global__ void __launch_bounds__(256, 2) bwdc_fwd_tc(const float* __restrict__ s0, float* __restrict__ ws,
                                                   const BwdChunkWs w, int T, int H, int nch,
                                                   int* __restrict__ status,
                                                   const __grid_constant__ CUtensorMap map_k,
                                                   const __grid_constant__ CUtensorMap map_wi) {
    using L = FwdTC<D>;
    constexpr int NSL = D / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const float* sc = reinterpret_cast<const float*>(sm + L::SC);
    float* decrk = reinterpret_cast<float*>(sm + L::SCL);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* never = reinterpret_cast<volatile int*>(sm + L::MISC + 8);
    const int jsl = blockIdx.x % NSL, h = (blockIdx.x / NSL) % H, b = blockIdx.x / (NSL * H);
    const int n0 = 64 * jsl;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int r0 = (warp & 3) * 16;
    const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t sa = sm100::smem_u32(sm);
    const bool has_row = (D == 128) || lane < 16;
    const int mrow = D == 128 ? 32 * (warp & 3) + lane : 16 * (warp & 3) + (lane & 15);
    const int cb = 32 * (warp >> 2);
    const int c0 = 32 * (warp >> 2);  // the warp's columns in 64 x 64 results

    if (tid == 0) {
        for (int i = 0; i < 8; ++i) sm100::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        *never = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tmap(&map_k);
        sm100::prefetch_tmap(&map_wi);
    }
    if (warp == 0) sm100::tmem_alloc(tmem_slot, L::TCOLS);
    float S[32];  // the state slice (row mrow, columns n0 + cb ..)
    {
        const float* src = s0 ? s0 + (((size_t)b * H + h) * D + mrow) * D + n0 + cb : nullptr;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float4 x = (src && has_row) ? *reinterpret_cast<const float4*>(src + 4 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[4 * u] = x.x; S[4 * u + 1] = x.y; S[4 * u + 2] = x.z; S[4 * u + 3] = x.w;
        }
    }
    auto write_S_images = [&]() {
        if (!has_row) return;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) split2(S[8 * u + 2 * p], S[8 * u + 2 * p + 1], hi[p], lo[p]);
            const uint32_t off = bpan(D, mrow, cb + 8 * u);
            *reinterpret_cast<uint4*>(sm + L::SH + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sm + L::SL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
    };
    write_S_images();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t pend = 0, ppar = 0;
    auto arm = [&](int i, int par, uint32_t bytes) {
        pend |= 1u << i;
        ppar = (ppar & ~(1u << i)) | ((uint32_t)par << i);
        sm100::mbar_arrive_expect_tx(&bars[i], bytes);
    };
    auto issue_A = [&](int cc, int par) {  // -W's images and the scalars of chunk cc
        const long rr = ((long)b * nch + cc) * H + h;
        arm(FB_A, par, (uint32_t)(2 * L::BF + 4 * kCB * 4));
        for (int p = 0; p < D / 64; ++p) {
            sm100::tma_load_2d(sm + L::WH + p * 8192, &map_wi, 64 * p, (int)(rr * 128), &bars[FB_A]);
            sm100::tma_load_2d(sm + L::WL + p * 8192, &map_wi, 64 * p, (int)(rr * 128 + 64), &bars[FB_A]);
        }
        sm100::bulk_load(sm + L::SC, ws + w.SC + rr * 256, 4 * kCB * 4, &bars[FB_A]);
    };
    auto issue_K = [&](int cc, int par) {  // k of chunk cc
        arm(FB_K, par, (uint32_t)L::BF);
        for (int p = 0; p < D / 64; ++p)
            sm100::tma_load_3d(sm + L::KP + p * 8192, &map_k, 64 * p, h, b * T + cc * kCB, &bars[FB_K]);
    };
    auto wait_bar = [&](int i, int par) {
        bool okw = sm100::mbar_wait_warp(&bars[i], (uint32_t)par, abort_flag);
        okw = __syncthreads_and(okw) != 0;
        sm100::tc_fence_after();
        if (tid == 0 && okw) pend &= ~(1u << i);
        return okw;
    };
    auto sync_issue = [&]() {
        sm100::fence_proxy_async_smem();
        sm100::tc_fence_before();
        __syncthreads();
        sm100::tc_fence_after();
    };
    if (tid == 0) {
        issue_A(0, 0);
        issue_K(0, 0);
    }
    constexpr uint32_t ID1 = sm100::idesc_bf16(64, 64, false, true);   // (-W) S
    constexpr uint32_t ID2 = sm100::idesc_bf16(D, 64, true, true);     // k^T U'
    bool ok = true;
    for (int c = 0; ok && c < nch; ++c) {
        const int par = c & 1;
        const long rr = ((long)b * nch + c) * H + h;
        const int nvc = min(kCB, T - c * kCB);
        // S^c -> workspace (tf32-rounded, for the local-gradient kernel)
        if (has_row) {
            float* g = ws + w.S + rr * D * D + (size_t)mrow * D + n0 + cb;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                *reinterpret_cast<float4*>(g + 4 * u) =
                    make_float4(rtf(S[4 * u]), rtf(S[4 * u + 1]), rtf(S[4 * u + 2]), rtf(S[4 * u + 3]));
        }
        // this warp's fragment of Ut (read while the products run)
        float2 ut[4][2];
        {
            const float* Utg = ws + w.Ut + rr * kCB * D + n0;
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    ut[t][hh] = *reinterpret_cast<const float2*>(Utg + (size_t)(r0 + gid + 8 * hh) * D + c0 + 8 * t + 2 * tig);
        }
        ok = wait_bar(FB_A, par);
        if (!ok) break;
        const float gC = expf(sc[128 + kCB - 1]);
        if (tid < kCB) decrk[tid] = expf(sc[128 + kCB - 1] - sc[128 + tid]) * sc[64 + tid];
        sync_issue();
        if (tid == 0) {  // D1 = (-W) S: hi hi + hi lo + lo hi
            for (int kb = 0; kb < D / 64; ++kb)
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t ao = kb * 8192 + kk * 32, bo = (kb * 4 + kk) * 2048;
                    const uint64_t ah = sm100::sdesc(sa + L::WH + ao, 16, 1024);
                    const uint64_t al = sm100::sdesc(sa + L::WL + ao, 16, 1024);
                    const uint64_t bh = sm100::sdesc(sa + L::SH + bo, L::SB, 1024);
                    const uint64_t bl = sm100::sdesc(sa + L::SL + bo, L::SB, 1024);
                    sm100::mma_bf16(tmem + L::TD1, ah, bh, ID1, (kb | kk) != 0);
                    sm100::mma_bf16(tmem + L::TD1, ah, bl, ID1, 1);
                    sm100::mma_bf16(tmem + L::TD1, al, bh, ID1, 1);
                }
            sm100::mma_commit(&bars[FB_M1]);
        }
        ok = wait_bar(FB_M1, par);
        if (!ok) break;
        {  // U = Ut + D1 -> workspace (tf32-rounded); U' = diag(dec rk) U as split images
            float d1[4][4];
            sm100::tmem_ld_frag<4>(tmem + lq + L::TD1 + c0, &d1[0][0]);
            float* Ug = ws + w.U + rr * kCB * D + n0;
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = r0 + gid + 8 * hh, n = c0 + 8 * t + 2 * tig;
                    const float u0 = ut[t][hh].x + d1[t][2 * hh], u1 = ut[t][hh].y + d1[t][2 * hh + 1];
                    *reinterpret_cast<float2*>(Ug + (size_t)i * D + n) = make_float2(rtf(u0), rtf(u1));
                    uint32_t hi, lo;
                    split2(decrk[i] * u0, decrk[i] * u1, hi, lo);
                    *reinterpret_cast<uint32_t*>(sm + L::UH + bpan(kCB, i, n)) = hi;
                    *reinterpret_cast<uint32_t*>(sm + L::UL + bpan(kCB, i, n)) = lo;
                }
        }
        ok = wait_bar(FB_K, par);
        if (!ok) break;
        if (nvc < kCB)  // rows past the end of the sequence are zero
            for (int e = tid; e < (D / 64) * (kCB - nvc) * 8; e += 256) {
                const int ch = e & 7, rowi = nvc + ((e >> 3) % (kCB - nvc)), pp = (e >> 3) / (kCB - nvc);
                *reinterpret_cast<uint4*>(sm + L::KP + pp * 8192 + rowi * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
        sync_issue();
        if (tid == 0) {  // D2 = k^T (U'_hi + U'_lo)
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = sm100::sdesc(sa + L::KP + kk * 2048, 8192, 1024);
                sm100::mma_bf16(tmem + L::TD2, a, sm100::sdesc(sa + L::UH + kk * 2048, 8192, 1024), ID2, kk != 0);
                sm100::mma_bf16(tmem + L::TD2, a, sm100::sdesc(sa + L::UL + kk * 2048, 8192, 1024), ID2, 1);
            }
            sm100::mma_commit(&bars[FB_M2]);
            if (c + 1 < nch) issue_A(c + 1, par ^ 1);  // -W and the scalars are read no more
        }
        ok = wait_bar(FB_M2, par);
        if (!ok) break;
        if (tid == 0 && c + 1 < nch) issue_K(c + 1, par ^ 1);  // k is read no more
        {  // S <- gC S + D2, and its split images for the next chunk
            float d2[32];
            sm100::tmem_ld32(tmem + lq + L::TD2 + cb, d2);
            if (has_row)
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] = fmaf(gC, S[j], d2[j]);
            write_S_images();
        }
    }
    if (!ok && tid == 0) {
        record_status(status, GDN_ERR_TIMEOUT);
        sm100::mma_commit(&bars[FB_DRAIN]);
        sm100::mbar_wait(&bars[FB_DRAIN], 0, never, 100000000ull);
        for (int i = FB_A; i <= FB_K; ++i)
            if (pend & (1u << i)) sm100::mbar_wait(&bars[i], (ppar >> i) & 1u, never, 100000000ull);
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, L::TCOLS);
    }
}

// ---------------------------------------------------------------------------- bwdc_rev_tc
// The reverse chain for bf16 inputs on tcgen05 (kind::f16): one CTA per (sequence, head,
// 64-column slice of the state gradient), 256 threads, chunks in reverse.  Per chunk, with dS the
// slice of the state gradient at the chunk's end (fp32, in registers: thread = row, 32 columns):
//   (i)   D1 = k dS (k exact in bf16; dS as split images hi + lo), D2 = P^T dY (P as split images)
//   (ii)  dU = diag(dec rk) D1 + D2 -> workspace, and dU's split images
//   (iii) D3 = q^T diag(s) dY - W^T dU (q exact; diag(s) dY and W as split images; the product of
//         two split operands takes hi hi + hi lo + lo hi), s = scale gam rq
//   (iv)  dS <- gC dS + D3
// Split images keep a product's relative error below about 2^-16 (tf32: 2^-11).  k, q, dY arrive
// by TMA as bf16 panels; the split images of -W and P were written by bwdc_prep_tc.  The copies
// for chunk c-1 start as soon as chunk c's products are done with their buffers.
template <int D>
struct RevTC {
    static constexpr int BF = kCB * D * 2, T8 = kCB * kCB * 2, SB = D * kCB * 2;  // 64 x D, 64 x 64, D x 64 bf16
    static constexpr int KP = 0, QP = KP + BF, WH = QP + BF, WL = WH + BF, PH = WL + BF, PL = PH + T8,
                         DY = PL + T8, SH = DY + T8, SL = SH + SB, UH = SL + SB, UL = UH + T8,
                         YH = UL + T8, YL = YH + T8;
    static constexpr int SC = YL + T8;              // the chunk's rq, rk, Lg, beta (copied)
    static constexpr int SCL = SC + 4 * kCB * 4;    // dec rk, s
    static constexpr int BAR = SCL + 2 * kCB * 4;
    static constexpr int MISC = BAR + 8 * 8;
    static constexpr int BYTES = MISC + 16 + 1024;
    static constexpr uint32_t TD1 = 0, TD2 = 64, TD3 = 128, TCOLS = 256;
};
enum RevBar { RB_A = 0, RB_B, RB_M1, RB_M2, RB_DRAIN };


template <int D>
__global__ void __launch_bounds__(256, 1) bwdc_rev_tc(const float* __restrict__ ds_final, float* __restrict__ ds0,
                                                   float* __restrict__ ws, const BwdChunkWs w, int T, int H, int nch,
                                                   float scale, int* __restrict__ status,
                                                   const __grid_constant__ CUtensorMap map_q,
                                                   const __grid_constant__ CUtensorMap map_k,
                                                   const __grid_constant__ CUtensorMap map_dy,
                                                   const __grid_constant__ CUtensorMap map_wi,
                                                   const __grid_constant__ CUtensorMap map_pi) {
    using L = RevTC<D>;
    constexpr int NSL = D / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const float* sc = reinterpret_cast<const float*>(sm + L::SC);
    float* decrk = reinterpret_cast<float*>(sm + L::SCL);
    float* sy = decrk + kCB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* never = reinterpret_cast<volatile int*>(sm + L::MISC + 8);
    const int jsl = blockIdx.x % NSL, h = (blockIdx.x / NSL) % H, b = blockIdx.x / (NSL * H);
    const int n0 = 64 * jsl;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int r0 = (warp & 3) * 16;
    const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t sa = sm100::smem_u32(sm);
    // the thread's row of the state-gradient slice and its 32 columns (M = 128: row = TMEM lane;
    // M = 64: rows 16 (w % 4) + lane for lanes 0..15)
    const bool has_row = (D == 128) || lane < 16;
    const int mrow = D == 128 ? 32 * (warp & 3) + lane : 16 * (warp & 3) + (lane & 15);
    const int cb = 32 * (warp >> 2);

    if (tid == 0) {
        for (int i = 0; i < 8; ++i) sm100::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        *never = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tmap(&map_q);
        sm100::prefetch_tmap(&map_k);
        sm100::prefetch_tmap(&map_dy);
        sm100::prefetch_tmap(&map_wi);
        sm100::prefetch_tmap(&map_pi);
    }
    if (warp == 0) sm100::tmem_alloc(tmem_slot, L::TCOLS);
    // the state gradient at the end of the sequence
    float dS[32];
    {
        const float* src = ds_final ? ds_final + (((size_t)b * H + h) * D + mrow) * D + n0 + cb : nullptr;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float4 x = (src && has_row) ? *reinterpret_cast<const float4*>(src + 4 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
            dS[4 * u] = x.x; dS[4 * u + 1] = x.y; dS[4 * u + 2] = x.z; dS[4 * u + 3] = x.w;
        }
    }
    // dS's split images (rows m, columns n of the slice: the MN-major operand of k dS)
    auto write_dS_images = [&]() {
        if (!has_row) return;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) split2(dS[8 * u + 2 * p], dS[8 * u + 2 * p + 1], hi[p], lo[p]);
            const uint32_t off = bpan(D, mrow, cb + 8 * u);
            *reinterpret_cast<uint4*>(sm + L::SH + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sm + L::SL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
    };
    write_dS_images();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t pend = 0, ppar = 0;  // (thread 0) copy barriers armed and not yet waited for, their parities
    auto arm = [&](int i, int par, uint32_t bytes) {
        pend |= 1u << i;
        ppar = (ppar & ~(1u << i)) | ((uint32_t)par << i);
        sm100::mbar_arrive_expect_tx(&bars[i], bytes);
    };
    auto issue_A = [&](int cc, int par) {  // k, P's images, the dY slice and the scalars of chunk cc
        const long rr = ((long)b * nch + cc) * H + h;
        const int z = b * T + cc * kCB;
        arm(RB_A, par, (uint32_t)(L::BF + 3 * L::T8 + 4 * kCB * 4));
        for (int p = 0; p < D / 64; ++p) sm100::tma_load_3d(sm + L::KP + p * 8192, &map_k, 64 * p, h, z, &bars[RB_A]);
        sm100::tma_load_2d(sm + L::PH, &map_pi, 0, (int)(rr * 128), &bars[RB_A]);
        sm100::tma_load_2d(sm + L::PL, &map_pi, 0, (int)(rr * 128 + 64), &bars[RB_A]);
        sm100::tma_load_3d(sm + L::DY, &map_dy, n0, h, z, &bars[RB_A]);
        sm100::bulk_load(sm + L::SC, ws + w.SC + rr * 256, 4 * kCB * 4, &bars[RB_A]);
    };
    auto issue_B = [&](int cc, int par) {  // q and -W's images of chunk cc
        const long rr = ((long)b * nch + cc) * H + h;
        const int z = b * T + cc * kCB;
        arm(RB_B, par, (uint32_t)(3 * L::BF));
        for (int p = 0; p < D / 64; ++p) {
            sm100::tma_load_3d(sm + L::QP + p * 8192, &map_q, 64 * p, h, z, &bars[RB_B]);
            sm100::tma_load_2d(sm + L::WH + p * 8192, &map_wi, 64 * p, (int)(rr * 128), &bars[RB_B]);
            sm100::tma_load_2d(sm + L::WL + p * 8192, &map_wi, 64 * p, (int)(rr * 128 + 64), &bars[RB_B]);
        }
    };
    auto wait_bar = [&](int i, int par) {
        bool okw = sm100::mbar_wait_warp(&bars[i], (uint32_t)par, abort_flag);
        okw = __syncthreads_and(okw) != 0;
        sm100::tc_fence_after();
        if (tid == 0 && okw) pend &= ~(1u << i);
        return okw;
    };
    auto sync_issue = [&]() {
        sm100::fence_proxy_async_smem();
        sm100::tc_fence_before();
        __syncthreads();
        sm100::tc_fence_after();
    };
    if (tid == 0) {
        issue_A(nch - 1, 0);
        issue_B(nch - 1, 0);
    }
    constexpr uint32_t ID64 = sm100::idesc_bf16(64, 64, false, true);     // k dS
    constexpr uint32_t IDP = sm100::idesc_bf16(64, 64, true, true);       // P^T dY
    constexpr uint32_t ID3 = sm100::idesc_bf16(D, 64, true, true);        // q^T sdY, (-W)^T dU
    bool ok = true;
    for (int it = 0, c = nch - 1; ok && c >= 0; ++it, --c) {
        const int par = it & 1;
        const long rr = ((long)b * nch + c) * H + h;
        const int nvc = min(kCB, T - c * kCB);
        // dS' of chunk c -> workspace (tf32-rounded, for the local-gradient kernel)
        if (has_row) {
            float* g = ws + w.dSp + rr * D * D + (size_t)mrow * D + n0 + cb;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                *reinterpret_cast<float4*>(g + 4 * u) =
                    make_float4(rtf(dS[4 * u]), rtf(dS[4 * u + 1]), rtf(dS[4 * u + 2]), rtf(dS[4 * u + 3]));
        }
        ok = wait_bar(RB_A, par);
        if (!ok) break;
        if (nvc < kCB)  // token rows past the end of the sequence are zero (k, dY)
            for (int e = tid; e < (D / 64 + 1) * (kCB - nvc) * 8; e += 256) {
                const int ch = e & 7, rowi = nvc + ((e >> 3) % (kCB - nvc)), pp = (e >> 3) / (kCB - nvc);
                *reinterpret_cast<uint4*>(sm + (pp < D / 64 ? L::KP + pp * 8192 : L::DY) + rowi * 128 + ch * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
        const float gC = expf(sc[128 + kCB - 1]);
        if (tid < kCB) {
            decrk[tid] = expf(sc[128 + kCB - 1] - sc[128 + tid]) * sc[64 + tid];
            sy[tid] = scale * expf(sc[128 + tid]) * sc[tid];
        }
        __syncthreads();
        {  // diag(s) dY as split images: thread -> row j = tid / 4, 16 columns
            const int j = tid >> 2;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int c8 = (tid & 3) * 16 + 8 * u;
                const uint32_t off = bpan(kCB, j, c8);
                const uint4 x = *reinterpret_cast<const uint4*>(sm + L::DY + off);
                const uint32_t wv[4] = {x.x, x.y, x.z, x.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    split2(sy[j] * __uint_as_float(wv[p] << 16), sy[j] * __uint_as_float(wv[p] & 0xffff0000u), hi[p], lo[p]);
                *reinterpret_cast<uint4*>(sm + L::YH + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(sm + L::YL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
        sync_issue();
        if (tid == 0) {
            for (int hl = 0; hl < 2; ++hl)  // D1 = k dS_hi + k dS_lo
                for (int kb = 0; kb < D / 64; ++kb)
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a = sm100::sdesc(sa + L::KP + kb * 8192 + kk * 32, 16, 1024);
                        const uint64_t bd = sm100::sdesc(sa + (hl ? L::SL : L::SH) + (kb * 4 + kk) * 2048, L::SB, 1024);
                        sm100::mma_bf16(tmem + L::TD1, a, bd, ID64, (hl | kb | kk) != 0);
                    }
            for (int hl = 0; hl < 2; ++hl)  // D2 = P_hi^T dY + P_lo^T dY
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = sm100::sdesc(sa + (hl ? L::PL : L::PH) + kk * 2048, 8192, 1024);
                    const uint64_t bd = sm100::sdesc(sa + L::DY + kk * 2048, 8192, 1024);
                    sm100::mma_bf16(tmem + L::TD2, a, bd, IDP, (hl | kk) != 0);
                }
            sm100::mma_commit(&bars[RB_M1]);
        }
        ok = wait_bar(RB_M1, par);
        if (!ok) break;
        if (tid == 0 && c > 0) issue_A(c - 1, par ^ 1);  // k, P, dY and the scalars are read no more
        {  // dU = diag(dec rk) D1 + D2 -> workspace (tf32-rounded) and its split images
            const int c0 = 32 * (warp >> 2);
            float d1[4][4], d2[4][4];
            sm100::tmem_ld_frag<4>(tmem + lq + L::TD1 + c0, &d1[0][0]);
            sm100::tmem_ld_frag<4>(tmem + lq + L::TD2 + c0, &d2[0][0]);
            float* dUg = ws + w.dU + rr * kCB * D + n0;
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = r0 + gid + 8 * hh, n = c0 + 8 * t + 2 * tig;
                    const float u0 = fmaf(decrk[i], d1[t][2 * hh], d2[t][2 * hh]);
                    const float u1 = fmaf(decrk[i], d1[t][2 * hh + 1], d2[t][2 * hh + 1]);
                    *reinterpret_cast<float2*>(dUg + (size_t)i * D + n) = make_float2(rtf(u0), rtf(u1));
                    uint32_t hi, lo;
                    split2(u0, u1, hi, lo);
                    *reinterpret_cast<uint32_t*>(sm + L::UH + bpan(kCB, i, n)) = hi;
                    *reinterpret_cast<uint32_t*>(sm + L::UL + bpan(kCB, i, n)) = lo;
                }
        }
        ok = wait_bar(RB_B, par);
        if (!ok) break;
        sync_issue();
        if (tid == 0) {
            for (int kk = 0; kk < 4; ++kk) {  // q^T (sdY_hi + sdY_lo)
                const uint64_t a = sm100::sdesc(sa + L::QP + kk * 2048, 8192, 1024);
                sm100::mma_bf16(tmem + L::TD3, a, sm100::sdesc(sa + L::YH + kk * 2048, 8192, 1024), ID3, kk != 0);
                sm100::mma_bf16(tmem + L::TD3, a, sm100::sdesc(sa + L::YL + kk * 2048, 8192, 1024), ID3, 1);
            }
            for (int kk = 0; kk < 4; ++kk) {  // (-W)^T dU: hi hi + hi lo + lo hi
                const uint64_t ah = sm100::sdesc(sa + L::WH + kk * 2048, 8192, 1024);
                const uint64_t al = sm100::sdesc(sa + L::WL + kk * 2048, 8192, 1024);
                const uint64_t bh = sm100::sdesc(sa + L::UH + kk * 2048, 8192, 1024);
                const uint64_t bl = sm100::sdesc(sa + L::UL + kk * 2048, 8192, 1024);
                sm100::mma_bf16(tmem + L::TD3, ah, bh, ID3, 1);
                sm100::mma_bf16(tmem + L::TD3, ah, bl, ID3, 1);
                sm100::mma_bf16(tmem + L::TD3, al, bh, ID3, 1);
            }
            sm100::mma_commit(&bars[RB_M2]);
        }
        ok = wait_bar(RB_M2, par);
        if (!ok) break;
        if (tid == 0 && c > 0) issue_B(c - 1, par ^ 1);  // q and -W are read no more
        {  // dS <- gC dS + D3, and its split images for the next chunk's k dS
            float d3[32];
            sm100::tmem_ld32(tmem + lq + L::TD3 + cb, d3);
            if (has_row)
#pragma unroll
                for (int j = 0; j < 32; ++j) dS[j] = fmaf(gC, dS[j], d3[j]);
            write_dS_images();
        }
    }
    if (ok && ds0 && has_row) {
        float* g = ds0 + (((size_t)b * H + h) * D + mrow) * D + n0 + cb;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            *reinterpret_cast<float4*>(g + 4 * u) = make_float4(dS[4 * u], dS[4 * u + 1], dS[4 * u + 2], dS[4 * u + 3]);
    }
    if (!ok && tid == 0) {
        record_status(status, GDN_ERR_TIMEOUT);
        sm100::mma_commit(&bars[RB_DRAIN]);
        sm100::mbar_wait(&bars[RB_DRAIN], 0, never, 100000000ull);
        for (int i = RB_A; i <= RB_B; ++i)
            if (pend & (1u << i)) sm100::mbar_wait(&bars[i], (ppar >> i) & 1u, never, 100000000ull);
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, L::TCOLS);
    }
}

// ============================================================================ chains
template <int D>
struct ChainB {
    static constexpr int LDS = kNVB + 8;  // rows k and k + 1..3 of a B operand: distinct banks
    static constexpr int LD = D + 4;
    static constexpr int FWD_BYTES = (D * LDS + 2 * kCB * LD + kCB * LDS + 2 * kCB) * 4;
    static constexpr int REV_BYTES = (D * LDS + 2 * kCB * LD + 2 * kCB * LDS + 3 * kCB) * 4;
};

// Per-thread registers holding one chunk's operands between their load and their store to shared
// memory: the copy for the next chunk is issued before the current chunk's arithmetic.
template <int D>
struct ChunkRegs {
    static constexpr int PW = kCB * D / 4 / 256;  // float4 of W
    static constexpr int PR = kCB * D / 8 / 256;  // 8-element groups of a token tile
    float4 w[PW];
    float k[PR][8];
    float2 y[4];  // Ut at this lane's positions of the U tiles (tile t, row half hh: y[2 t + hh])
};

// Forward: S^c and U of every chunk, 32 state columns per CTA.
template <int D, typename Tin>
__global__ void __launch_bounds__(256) bwdc_fwd(const Tin* __restrict__ k, const float* __restrict__ s0,
                                                float* __restrict__ ws, const BwdChunkWs w, int T, int H,
                                                int nch) {
    using L = ChainB<D>;
    using R = ChunkRegs<D>;
    constexpr int LDS = L::LDS, LD = L::LD;
    extern __shared__ float smf[];
    float* Ss = smf;
    float* Wt = Ss + D * LDS;
    float* Kt = Wt + kCB * LD;   // raw K rows
    float* Us = Kt + kCB * LD;
    float* dec = Us + kCB * LDS;  // gC / gam
    float* rks = dec + kCB;
    constexpr int nsl = D / kNVB;
    const int jsl = blockIdx.x % nsl, h = (blockIdx.x / nsl) % H, b = blockIdx.x / (nsl * H);
    const int col0 = jsl * kNVB, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    // U (64 x 32) tiles: warp w owns rows 16 (w & 3) .. +15 and columns 16 (w >> 2) .. +15
    const int ur0 = (warp & 3) * 16, uc0 = (warp >> 2) * 16;
    R rg;
    auto fetch = [&](int c) {
        const size_t r = ((size_t)b * nch + c) * H + h;
        const float4* Wg = reinterpret_cast<const float4*>(ws + w.W + r * kCB * D);
#pragma unroll
        for (int u = 0; u < R::PW; ++u) rg.w[u] = Wg[tid + u * 256];
        const int t0c = c * kCB, nvc = min(kCB, T - t0c);
#pragma unroll
        for (int u = 0; u < R::PR; ++u) {
            const int e = (tid + u * 256) * 8, i = e / D, m = e % D;
            if (i < nvc) ld8(k + tok_off(b, t0c + i, h, T, H) * D + m, rg.k[u]);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) rg.k[u][j] = 0.f;
            }
        }
        const float* Utg = ws + w.Ut + r * kCB * D + col0;  // Ut at this lane's U tile positions
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                rg.y[2 * t + hh] = *reinterpret_cast<const float2*>(
                    Utg + (size_t)(ur0 + gid + 8 * hh) * D + uc0 + 8 * t + 2 * tig);
    };
    for (int e = tid; e < D * kNVB; e += 256) {
        const int m = e / kNVB, n = e % kNVB;
        Ss[m * LDS + n] = s0 ? s0[(((size_t)b * H + h) * D + m) * D + col0 + n] : 0.f;
    }
    fetch(0);
    for (int c = 0; c < nch; ++c) {
        const size_t r = ((size_t)b * nch + c) * H + h;
        __syncthreads();
        float* Sg = ws + w.S + r * D * D;
        for (int e = tid; e < D * kNVB; e += 256) {
            const int m = e / kNVB, n = e % kNVB;
            Sg[(size_t)m * D + col0 + n] = rtf(Ss[m * LDS + n]);
        }
#pragma unroll
        for (int u = 0; u < R::PW; ++u) {
            const int e = (tid + u * 256) * 4;
            *reinterpret_cast<float4*>(Wt + (e / D) * LD + e % D) = rg.w[u];
        }
#pragma unroll
        for (int u = 0; u < R::PR; ++u) {
            const int e = (tid + u * 256) * 8;
            st8(Kt + (e / D) * LD + e % D, rg.k[u], 1.f);
        }
        float2 ut[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) ut[j] = rg.y[j];
        const float* SCg = ws + w.SC + r * 256;
        if (tid < kCB) {
            dec[tid] = expf(SCg[128 + kCB - 1] - SCg[128 + tid]);
            rks[tid] = SCg[64 + tid];
        }
        const float gC = expf(SCg[128 + kCB - 1]);
        __syncthreads();
        if (c + 1 < nch) fetch(c + 1);
        {  // U = Ut - W S as 16 x 8 tensor-core tiles (tf32 operands, fp32 accumulation)
            float acc[2][4];
            zero_acc(acc);
            const float* Wp = Wt;
            const float* Sp = Ss;
            wmma_acc(acc, D, ur0, uc0, [Wp](int i, int k2) { return Wp[i * LD + k2]; },
                     [Sp](int k2, int n) { return Sp[k2 * LDS + n]; }, lane);
            float* Ug = ws + w.U + r * kCB * D + col0;
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = ur0 + gid + 8 * hh, n = uc0 + 8 * t + 2 * tig;
                    const float2 u = make_float2(ut[2 * t + hh].x - acc[t][2 * hh],
                                                 ut[2 * t + hh].y - acc[t][2 * hh + 1]);
                    *reinterpret_cast<float2*>(Us + i * LDS + n) = u;
                    *reinterpret_cast<float2*>(Ug + (size_t)i * D + n) = make_float2(rtf(u.x), rtf(u.y));
                }
        }
        __syncthreads();
        {  // S = gC S + K^T diag(rk gC / gam) U as tensor-core tiles (tf32, fp32 accumulation);
           // the D x 32 slice is D / 16 row blocks by 8 / (D / 16) column groups, one per warp
            constexpr int RB = D / 16, CG = 8 / RB, CT = 4 / CG;
            const int sr0 = 16 * (warp % RB), sc0 = (32 / CG) * (warp / RB);
            float acc[CT][4];
            zero_acc(acc);
            const float* Kp = Kt;
            const float* Up = Us;
            const float* dp = dec;
            const float* rp = rks;
            wmma_acc(acc, kCB, sr0, sc0,
                     [Kp, dp, rp](int m, int i) { return Kp[i * LD + m] * (dp[i] * rp[i]); },
                     [Up](int i, int n) { return Up[i * LDS + n]; }, lane);
#pragma unroll
            for (int t = 0; t < CT; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float* sp = Ss + (sr0 + gid + 8 * hh) * LDS + sc0 + 8 * t + 2 * tig;
                    const float2 o = *reinterpret_cast<const float2*>(sp);
                    *reinterpret_cast<float2*>(sp) =
                        make_float2(fmaf(gC, o.x, acc[t][2 * hh]), fmaf(gC, o.y, acc[t][2 * hh + 1]));
                }
        }
    }
}

// Reverse: dS' and dU of every chunk, and dS0, 32 state columns per CTA.  The dU step reads K and
// P, the dS step Q and W: the two pairs take turns in the same two tiles (two CTAs per SM).
template <int D, typename Tin>
__global__ void __launch_bounds__(256, 2) bwdc_rev(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                   const Tin* __restrict__ dy, const float* __restrict__ ds_final,
                                                   float* __restrict__ ds0, float* __restrict__ ws,
                                                   const BwdChunkWs w, int T, int H, int nch, float scale) {
    using L = ChainB<D>;
    constexpr int LDS = L::LDS, LD = L::LD;
    extern __shared__ float smf[];
    float* Ss = smf;                 // dS slice
    float* X1 = Ss + D * LDS;        // K^ (dU step), then scale gam Q^ (dS step)
    float* X2 = X1 + kCB * LD;       // P (dU step, row stride kL64), then W (dS step)
    float* dYs = X2 + kCB * LD;
    float* dUs = dYs + kCB * LDS;
    float* dec = dUs + kCB * LDS;    // gC / gam
    float* ysc = dec + kCB;          // scale gam rq
    float* rks = ysc + kCB;
    constexpr int nsl = D / kNVB;
    const int jsl = blockIdx.x % nsl, h = (blockIdx.x / nsl) % H, b = blockIdx.x / (nsl * H);
    const int col0 = jsl * kNVB, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    // dU (64 x 32) tiles: warp w owns rows 16 (w & 3) .. +15 and columns 16 (w >> 2) .. +15;
    // dS (D x 32): D / 16 row blocks by 8 / (D / 16) column groups, one per warp
    const int ur0 = (warp & 3) * 16, uc0 = (warp >> 2) * 16;
    constexpr int RB = D / 16, CG = 8 / RB, SCT = 4 / CG;
    const int sr0 = 16 * (warp % RB), sc0 = (32 / CG) * (warp / RB);
    for (int e = tid; e < D * kNVB; e += 256) {
        const int m = e / kNVB, n = e % kNVB;
        Ss[m * LDS + n] = ds_final ? ds_final[(((size_t)b * H + h) * D + m) * D + col0 + n] : 0.f;
    }
    for (int c = nch - 1; c >= 0; --c) {
        const size_t r = ((size_t)b * nch + c) * H + h;
        __syncthreads();
        float* dSg = ws + w.dSp + r * D * D;
        for (int e = tid; e < D * kNVB; e += 256) {
            const int m = e / kNVB, n = e % kNVB;
            dSg[(size_t)m * D + col0 + n] = rtf(Ss[m * LDS + n]);
        }
        const float* SCg = ws + w.SC + r * 256;
        if (tid < kCB) {
            dec[tid] = expf(SCg[128 + kCB - 1] - SCg[128 + tid]);
            ysc[tid] = scale * expf(SCg[128 + tid]) * SCg[tid];
            rks[tid] = SCg[64 + tid];
        }
        const float gC = expf(SCg[128 + kCB - 1]);
        load_rec<kCB, kL64, 256>(X2, ws + w.P + r * kCB * kCB, tid);
        {  // dY slice: 64 rows x 32 columns, one 8-element group per thread
            const int i = tid >> 2, n = (tid & 3) * 8, t = c * kCB + i;
            float x[8];
            if (t < T) ld8(dy + tok_off(b, t, h, T, H) * D + col0 + n, x);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = 0.f;
            }
            st8(dYs + i * LDS + n, x, 1.f);
        }
        __syncthreads();
        const int nvc = min(kCB, T - c * kCB);
        load_rows<D, LD, 256>(X1, k, b, c * kCB, nvc, h, T, H, rks, tid);
        __syncthreads();
        {  // dU = diag(gC / gam) K^ dS + P^T dY as tensor-core tiles (tf32, fp32 accumulation)
            float a1[2][4], a2[2][4];
            zero_acc(a1);
            zero_acc(a2);
            const float* Kp = X1;
            const float* Pp = X2;
            const float* Sp = Ss;
            const float* Yp = dYs;
            wmma_acc(a1, D, ur0, uc0, [Kp](int i, int m) { return Kp[i * LD + m]; },
                     [Sp](int m, int n) { return Sp[m * LDS + n]; }, lane);
            wmma_acc(a2, kCB, ur0, uc0, [Pp](int i, int j) { return Pp[j * kL64 + i]; },
                     [Yp](int j, int n) { return Yp[j * LDS + n]; }, lane);
            float* dUg = ws + w.dU + r * kCB * D + col0;
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = ur0 + gid + 8 * hh, n = uc0 + 8 * t + 2 * tig;
                    const float2 du = make_float2(fmaf(dec[i], a1[t][2 * hh], a2[t][2 * hh]),
                                                  fmaf(dec[i], a1[t][2 * hh + 1], a2[t][2 * hh + 1]));
                    *reinterpret_cast<float2*>(dUs + i * LDS + n) = du;
                    *reinterpret_cast<float2*>(dUg + (size_t)i * D + n) = make_float2(rtf(du.x), rtf(du.y));
                }
        }
        __syncthreads();
        load_rows<D, LD, 256>(X1, q, b, c * kCB, nvc, h, T, H, ysc, tid);
        load_rec<D, LD, 256>(X2, ws + w.W + r * kCB * D, tid);
        __syncthreads();
        {  // dS = gC dS + (scale gam Q^)^T dY - W^T dU as tensor-core tiles with split (3 x tf32)
           // operands: these products feed the state gradient along the whole chain
            float a1[SCT][4], a2[SCT][4];
            zero_acc(a1);
            zero_acc(a2);
            const float* Qp = X1;
            const float* Wp = X2;
            const float* Yp = dYs;
            const float* Up = dUs;
            wmma_acc3(a1, kCB, sr0, sc0, [Qp](int m, int i) { return Qp[i * LD + m]; },
                      [Yp](int i, int n) { return Yp[i * LDS + n]; }, lane);
            wmma_acc3(a2, kCB, sr0, sc0, [Wp](int m, int i) { return Wp[i * LD + m]; },
                      [Up](int i, int n) { return Up[i * LDS + n]; }, lane);
#pragma unroll
            for (int t = 0; t < SCT; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float* sp = Ss + (sr0 + gid + 8 * hh) * LDS + sc0 + 8 * t + 2 * tig;
                    const float2 o = *reinterpret_cast<const float2*>(sp);
                    *reinterpret_cast<float2*>(sp) =
                        make_float2(fmaf(gC, o.x, a1[t][2 * hh] - a2[t][2 * hh]),
                                    fmaf(gC, o.y, a1[t][2 * hh + 1] - a2[t][2 * hh + 1]));
                }
        }
    }
    __syncthreads();
    if (ds0)
        for (int e = tid; e < D * kNVB; e += 256) {
            const int m = e / kNVB, n = e % kNVB;
            ds0[(((size_t)b * H + h) * D + m) * D + col0 + n] = Ss[m * LDS + n];
        }
}

// ============================================================================ bwdc_local
// Every product runs on tcgen05 tensor cores as M = 64 tiles with tf32 operands and fp32
// accumulators in TMEM; one thread issues the products and the tensor copies, all 16 warps stage
// the token tiles and run the epilogues.  Operands sit in shared memory as 128-byte-swizzled
// panels (below), K-major on both sides; a product that contracts over the token index takes a
// transposed copy, written when the operand is staged or produced.  The fp32 records of the
// workspace (dU, U, S, dS', T; rounded to tf32 by the kernels that write them) arrive by TMA
// straight into panels.  Each warp owns the same part of every 64-row result as the fragment
// layout of a warp-level m16n8 MMA: rows 16 (w % 4) .. +15 and, in 64 x D results, columns
// (w / 4) D/4 .. +D/4 - 1 (in 64 x 64 results columns 16 (w / 4) .. +15); lane (gid, tig) holds
// rows gid, gid + 8 and columns 2 tig, 2 tig + 1 of each 16 x 8 tile, read out of TMEM with the
// 16x256b load shape from the warp's own quarter of the lanes.  dq^ and dk^ stay in registers in
// that layout across the products that feed them.
//
// Shared-memory panels: a matrix of R rows (a multiple of 8) and C columns (a multiple of 32) is
// stored as C / 32 panels of R rows x 128 bytes, 1024-byte aligned; the 16-byte chunk c of row r
// of a panel sits at chunk position c ^ (r % 8) (the layout a 32 x R fp32 TMA box with the
// 128-byte swizzle writes).  Values are tf32 (rounded to nearest), so that the MMA's truncation
// to tf32 is exact.
__device__ __forceinline__ uint32_t pan(int R, int r, int c) {
    return (uint32_t)((((c >> 5) * R + r) << 7) + (((((c & 31) >> 2) ^ (r & 7))) << 4) + ((c & 3) << 2));
}

// Stage rows 0..63 x C columns (C = 64 or 128) into panels: row-major into `dst` (64 rows) and/or
// transposed into `dstT` (C rows x 64 columns).  `src(r, c, x)` yields the 8 values of row r,
// columns c .. c + 7.  Lane l of warp w takes row 32 (w % 2) + l and the 8-column groups
// w / 2 + 8 u: a warp's transposed stores then fill one 128-byte row (distinct banks), its
// row-major 16-byte stores spread over the 8 swizzled chunk positions.  All loads are issued
// before any store.
template <int C, typename Src>
__device__ __forceinline__ void stage(uint8_t* dst, uint8_t* dstT, Src src, int tid) {
    constexpr int PER = C / 64;
    const int lane = tid & 31, warp = tid >> 5;
    const int r = 32 * (warp & 1) + lane;
    float x[PER][8];
#pragma unroll
    for (int u = 0; u < PER; ++u) src(r, 8 * ((warp >> 1) + 8 * u), x[u]);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int c = 8 * ((warp >> 1) + 8 * u);
        float y[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) y[j] = rtf(x[u][j]);
        if (dst) {
            *reinterpret_cast<float4*>(dst + pan(kCB, r, c)) = make_float4(y[0], y[1], y[2], y[3]);
            *reinterpret_cast<float4*>(dst + pan(kCB, r, c + 4)) = make_float4(y[4], y[5], y[6], y[7]);
        }
        if (dstT) {
#pragma unroll
            for (int j = 0; j < 8; ++j) *reinterpret_cast<float*>(dstT + pan(C, c + j, r)) = y[j];
        }
    }
}
// 8 values of row r, columns c .. c + 7, of a 64-row panel tile in shared memory
__device__ __forceinline__ void pan_ld8(const uint8_t* t, int r, int c, float* x) {
    const float4 a = *reinterpret_cast<const float4*>(t + pan(kCB, r, c));
    const float4 b = *reinterpret_cast<const float4*>(t + pan(kCB, r, c + 4));
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// D[0..63][0..N) (+)= A B^T over K (a multiple of 8): A = 64-row panels at shared address a,
// B = b_rows-row panels at b (its first N rows are used), both K-major.  One thread issues.
__device__ __forceinline__ void tc_gemm(uint32_t d, uint32_t a, uint32_t b, int b_rows, int K, uint32_t idesc,
                                        bool accumulate) {
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t kc = (uint32_t)(k0 & 31) * 4;
        const uint64_t da = sm100::sdesc(a + (uint32_t)(k0 >> 5) * kCB * 128 + kc, 16, 1024);
        const uint64_t db = sm100::sdesc(b + (uint32_t)(k0 >> 5) * b_rows * 128 + kc, 16, 1024);
        sm100::mma_tf32_tc(d, da, db, idesc, (accumulate || k0 > 0) ? 1u : 0u);
    }
}
// TMA copy of a 64 x C fp32 record (rows y0 .. y0 + 63 of a C-wide tensor map) into 64-row panels
__device__ __forceinline__ void tma_rec(uint8_t* dst, const CUtensorMap* map, int C, long y0, uint64_t* bar) {
    for (int p = 0; p < C / 32; ++p) sm100::tma_load_2d(dst + p * kCB * 128, map, 32 * p, (int)y0, bar);
}

__device__ __forceinline__ float2 ld2(const __nv_bfloat16* p) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ float2 ld2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ void st2(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void st2(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
}

// Shared-memory layout (bytes from a 1024-byte aligned base) and TMEM columns of bwdc_local.
// Five 64 x D tiles (B0..B4) and three 64 x 64 tiles (S0..S2) are reused as the products go:
//   B0: dU, dW, dS' rows 0..63, F      B1: dY, k^T            B2: S rows 0..63 (then 64..127), k
//   B3: dU^T, dW^T, dS' rows 64..127, F^T diag(rq)           B4: V, U, q^T
//   S0: T^T, M2 = T^T dT               S1: T, E^T diag(rk)    S2: dT^T, E diag(rk)
// (k and q unnormalised: the row scales rk, rq are applied in the epilogues and folded into the
// other operand of the products that contract over the token index.)
// TMEM: Z (T^T dU, T^T dW, then dk^'s last products), W (dU S^T, U dS'^T, then F K^), G (dY S^T,
// then dP), X (dU V^T, then M2), Y (dW k^T, then M2 T^T).
template <int D>
struct LocalB {
    static constexpr int BIG = kCB * D * 4, SMALL = kCB * kCB * 4;
    static constexpr int B0 = 0, B1 = B0 + BIG, B2 = B1 + BIG, B3 = B2 + BIG, B4 = B3 + BIG;
    static constexpr int S0 = B4 + BIG, S1 = S0 + SMALL, S2 = S1 + SMALL;
    static constexpr int NROW = 10;                       // row accumulators of 64
    static constexpr int SCAL = S2 + SMALL;               // rq, rk, Lg, beta, gam
    static constexpr int RACC = SCAL + 5 * kCB * 4;
    static constexpr int BAR = RACC + (NROW * kCB + 32) * 4;
    static constexpr int NBAR = 16;
    static constexpr int MISC = BAR + NBAR * 8;           // TMEM base, abort flag, zero word
    static constexpr int BYTES = MISC + 16 + 1024;        // + alignment slack
    static constexpr uint32_t TZ = 0, TW = D, TG = 2 * D, TX = 3 * D, TY = 3 * D + 64, TCOLS = 512;
    static_assert(TY + 64 <= TCOLS, "TMEM columns");
    static_assert(BAR % 8 == 0, "mbarrier alignment");
};
// mbarriers: products (one commit each) and tensor copies
enum LocalBar { LB_P0 = 0, LB_P1, LB_P2, LB_P3, LB_P4, LB_P5, LB_DRAIN, LB_C0, LB_C1, LB_C2, LB_C3 };

template <int D, typename Tin>
__global__ void __launch_bounds__(512, 1) bwdc_local(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                     const Tin* __restrict__ v, const Tin* __restrict__ dy,
                                                     const float* __restrict__ alpha, Tin* __restrict__ dq,
                                                     Tin* __restrict__ dk, Tin* __restrict__ dv,
                                                     float* __restrict__ dalpha, float* __restrict__ dbeta,
                                                     const float* __restrict__ ws, const BwdChunkWs w, int T,
                                                     int H, int nch, float scale, int l2norm,
                                                     const float* __restrict__ A_log,
                                                     const float* __restrict__ b_alpha,
                                                     float* __restrict__ dA_log,
                                                     float* __restrict__ db_alpha, int* __restrict__ status,
                                                     const __grid_constant__ CUtensorMap map_d,
                                                     const __grid_constant__ CUtensorMap map_64) {
    using L = LocalB<D>;
    constexpr int CT = D / 32;  // 8-column tiles per warp in 64 x D results
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* rq = reinterpret_cast<float*>(sm + L::SCAL);
    float* rk = rq + kCB;
    float* Lg = rk + kCB;
    float* be = Lg + kCB;
    float* gam = be + kCB;
    float* racc = reinterpret_cast<float*>(sm + L::RACC);  // NROW row accumulators of 64
    float* r_dbe = racc;          // v . T^T dU  + sum_j dA_ij At_ij
    float* r_dbg = racc + 64;     // k^ . T^T dW  (d (beta gam))
    float* r_g1 = racc + 128;     // q^ . dY S^T
    float* r_dr = racc + 192;     // k^ . U dS'^T  (d (gC / gam))
    float* rowM = racc + 256;     // row sums of dA * A + dP * P
    float* colM = racc + 320;     // column sums
    float* r_pq = racc + 384;     // q^ . dq^
    float* r_pk = racc + 448;     // k^ . dk^
    float* dLg = racc + 512;
    float* red = racc + 640;      // [0]: gC d gC
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* never = reinterpret_cast<volatile int*>(sm + L::MISC + 8);
    const size_t r = blockIdx.x;
    const int h = (int)(r % H);
    const int gr = (int)(r / H);
    const int c = gr % nch, b = gr / nch;
    const int t0 = c * kCB, nv = min(kCB, T - t0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int r0 = (warp & 3) * 16;             // tile rows of this warp
    const int cD = (warp >> 2) * (D / 4);       // first column in 64 x D results
    const int c64 = (warp >> 2) * 16;           // first column in 64 x 64 results
    const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's TMEM lane quarter
    const float* Sg = ws + w.S + r * D * D;
    const float* Atg = ws + w.At + r * kCB * kCB;
    const float* Pg = ws + w.P + r * kCB * kCB;
    // rows of the workspace's records in the D-wide and 64-wide tensor maps
    const long y_dU = (long)(w.dU / D) + (long)r * kCB, y_U = (long)(w.U / D) + (long)r * kCB;
    const long y_S = (long)(w.S / D) + (long)r * D, y_dS = (long)(w.dSp / D) + (long)r * D;
    const long y_T = (long)(w.Tm / kCB) + (long)r * kCB;
    const uint32_t sa = sm100::smem_u32(sm);

    if (tid == 0) {
        for (int i = 0; i < L::NBAR; ++i) sm100::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        *never = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tmap(&map_d);
        sm100::prefetch_tmap(&map_64);
    }
    if (warp == 0) sm100::tmem_alloc(tmem_slot, L::TCOLS);
    // L2 prefetches: At and P (read late), the chunk's q and k rows (read in several epilogues)
    if (warp == 1 && lane < 2) sm100::bulk_prefetch_l2(lane ? Pg : Atg, kCB * kCB * 4);
    if (tid >= 64 && tid < 192 && ((tid - 64) & 63) < nv)
        sm100::bulk_prefetch_l2((tid < 128 ? q : k) + tok_off(b, t0 + ((tid - 64) & 63), h, T, H) * D,
                                (uint32_t)(D * sizeof(Tin)));
    // dY and V rows into registers (stored once the barriers are set up)
    constexpr int PER = D / 64;
    const int rr = 32 * (warp & 1) + lane;  // the row this thread stages (see stage())
    float xy[PER][8], xv[PER][8];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int m = 8 * ((warp >> 1) + 8 * u);
        if (rr < nv) {
            ld8(dy + tok_off(b, t0 + rr, h, T, H) * D + m, xy[u]);
            ld8(v + tok_off(b, t0 + rr, h, T, H) * D + m, xv[u]);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) xy[u][j] = xv[u][j] = 0.f;
        }
    }
    for (int e = tid; e < L::NROW * kCB + 32; e += 512) racc[e] = 0.f;
    sm100::tc_fence_before();
    __syncthreads();  // barriers initialised, TMEM allocated
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t copies = 0;  // (thread 0) the copy barriers armed so far
    if (tid == 0) {  // dU, S rows 0..63 and T by TMA; the chunk scalars rq, rk, Lg, beta
        copies |= 1u << LB_C0;
        sm100::mbar_arrive_expect_tx(&bars[LB_C0], (uint32_t)(2 * L::BIG + L::SMALL + 4 * kCB * 4));
        tma_rec(sm + L::B0, &map_d, D, y_dU, &bars[LB_C0]);
        tma_rec(sm + L::B2, &map_d, D, y_S, &bars[LB_C0]);
        tma_rec(sm + L::S1, &map_64, kCB, y_T, &bars[LB_C0]);
        sm100::bulk_load(sm + L::SCAL, ws + w.SC + r * 256, 4 * kCB * 4, &bars[LB_C0]);
    }

    auto tok = [=](const Tin* p) {  // token rows of a [B, T, H, D] tensor (zero past the end)
        return [=](int i, int m, float* x) {
            if (i < nv) {
                ld8(p + tok_off(b, t0 + i, h, T, H) * D + m, x);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = 0.f;
            }
        };
    };
    // elements (i, n), (i, n + 1) of token row i of a [B, T, H, D] tensor (zero past the end)
    auto gpair = [&](const Tin* p, int i, int n) {
        return i < nv ? ld2(p + tok_off(b, t0 + i, h, T, H) * D + n) : make_float2(0.f, 0.f);
    };
    auto tpair = [&](int off, int i, int n) {  // elements (i, n), (i, n + 1) of a 64-row panel tile
        return *reinterpret_cast<const float2*>(sm + off + pan(kCB, i, n));
    };
    // all threads: operand stores visible to the tensor core, TMEM reads ordered before the next
    // products; then thread 0 issues
    auto sync_issue = [&]() {
        sm100::fence_proxy_async_smem();
        sm100::tc_fence_before();
        __syncthreads();
        sm100::tc_fence_after();
    };
    // all threads: wait for barrier i (products or copies); the result is the same everywhere
    auto wait_bar = [&](int i) {
        bool okw = sm100::mbar_wait_warp(&bars[i], 0, abort_flag);
        okw = __syncthreads_and(okw) != 0;
        sm100::tc_fence_after();
        return okw;
    };
    auto frag = [&](uint32_t col, auto& acc) {  // this warp's fragment of a 64-row result
        sm100::tmem_ld_frag<sizeof(acc) / 16>(tmem + lq + col, &acc[0][0]);
    };
    auto row_add = [&](float* acc, float lo, float hi) {
        lo = quad_sum(lo);
        hi = quad_sum(hi);
        if (tig == 0) {
            atomicAdd(&acc[r0 + gid], lo);
            atomicAdd(&acc[r0 + gid + 8], hi);
        }
    };
    constexpr uint32_t ID_N = sm100::idesc_tf32(64, D), ID_64 = sm100::idesc_tf32(64, 64);

    // ---- stage 1: dY -> B1, V -> B4; dU^T -> B3 and T^T -> S0 from the copies
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int cc = 8 * ((warp >> 1) + 8 * u);
        float a[8], bb[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) { a[j] = rtf(xy[u][j]); bb[j] = rtf(xv[u][j]); }
        *reinterpret_cast<float4*>(sm + L::B1 + pan(kCB, rr, cc)) = make_float4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<float4*>(sm + L::B1 + pan(kCB, rr, cc + 4)) = make_float4(a[4], a[5], a[6], a[7]);
        *reinterpret_cast<float4*>(sm + L::B4 + pan(kCB, rr, cc)) = make_float4(bb[0], bb[1], bb[2], bb[3]);
        *reinterpret_cast<float4*>(sm + L::B4 + pan(kCB, rr, cc + 4)) = make_float4(bb[4], bb[5], bb[6], bb[7]);
    }
    bool ok = wait_bar(LB_C0);
    if (ok) {
        if (tid < kCB) gam[tid] = expf(Lg[tid]);
        const uint8_t* du = sm + L::B0;
        const uint8_t* tt = sm + L::S1;
        stage<D>(nullptr, sm + L::B3, [du](int i, int m, float* x) { pan_ld8(du, i, m, x); }, tid);
        stage<kCB>(nullptr, sm + L::S0, [tt](int i, int m, float* x) { pan_ld8(tt, i, m, x); }, tid);
        sync_issue();
        if (tid == 0) {
            tc_gemm(tmem + L::TZ, sa + L::S0, sa + L::B3, D, kCB, ID_N, false);  // Z1 = T^T dU
            tc_gemm(tmem + L::TW, sa + L::B0, sa + L::B2, kCB, D, ID_64, false);  // dU S^T, columns 0..63
            tc_gemm(tmem + L::TG, sa + L::B1, sa + L::B2, kCB, D, ID_64, false);  // dY S^T, columns 0..63
            tc_gemm(tmem + L::TX, sa + L::B0, sa + L::B4, kCB, D, ID_64, false);  // X = dU V^T
            sm100::mma_commit(&bars[LB_P0]);
        }
        ok = wait_bar(LB_P0);
    }
    if constexpr (D == 128) {
        if (ok) {
            if (tid == 0) {  // S rows 64..127
                copies |= 1u << LB_C1;
                sm100::mbar_arrive_expect_tx(&bars[LB_C1], (uint32_t)L::BIG);
                tma_rec(sm + L::B2, &map_d, D, y_S + 64, &bars[LB_C1]);
            }
        }
    }
    float dqa[CT][4], dka[CT][4];
    if (ok) {
        // Z1 = T^T dU: dV = diag(beta) Z1, dbeta += v . Z1
        float z[CT][4];
        frag(L::TZ + cD, z);
        float lo = 0.f, hi = 0.f;
#pragma unroll
        for (int t = 0; t < CT; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = r0 + gid + 8 * hh, n = cD + 8 * t + 2 * tig;
                const float2 vv = tpair(L::B4, i, n);
                const float pv = vv.x * z[t][2 * hh] + vv.y * z[t][2 * hh + 1];
                if (hh == 0) lo += pv; else hi += pv;
                if (i < nv) st2(dv + tok_off(b, t0 + i, h, T, H) * D + n, be[i] * z[t][2 * hh], be[i] * z[t][2 * hh + 1]);
            }
        row_add(r_dbe, lo, hi);
    }
    if constexpr (D == 128) {
        if (ok) ok = wait_bar(LB_C1);
        if (ok) {
            sync_issue();
            if (tid == 0) {
                tc_gemm(tmem + L::TW + 64, sa + L::B0, sa + L::B2, kCB, D, ID_64, false);
                tc_gemm(tmem + L::TG + 64, sa + L::B1, sa + L::B2, kCB, D, ID_64, false);
                sm100::mma_commit(&bars[LB_P1]);
            }
            ok = wait_bar(LB_P1);
        }
    } else {
        if (ok) sync_issue();  // every thread is past Z1's epilogue (V in B4 is read no more)
    }
    if (ok) {
        if (tid == 0) {  // U -> B4 (V is read no more)
            copies |= 1u << LB_C2;
            sm100::mbar_arrive_expect_tx(&bars[LB_C2], (uint32_t)L::BIG);
            tma_rec(sm + L::B4, &map_d, D, y_U, &bars[LB_C2]);
        }
        // k -> B2 (loaded first: its latency overlaps the epilogues below)
        {
            float xk[PER][8];
            auto lk = tok(k);
#pragma unroll
            for (int u = 0; u < PER; ++u) lk(rr, 8 * ((warp >> 1) + 8 * u), xk[u]);
            // G1 = dY S^T: dq^ = scale gam G1, q^ . G1 for d gam
            float x[CT][4];
            frag(L::TG + cD, x);
            float lo = 0.f, hi = 0.f;
#pragma unroll
            for (int t = 0; t < CT; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = r0 + gid + 8 * hh, n = cD + 8 * t + 2 * tig;
                    const float2 qv = gpair(q, i, n);
                    dqa[t][2 * hh] = scale * gam[i] * x[t][2 * hh];
                    dqa[t][2 * hh + 1] = scale * gam[i] * x[t][2 * hh + 1];
                    const float pv = rq[i] * (qv.x * x[t][2 * hh] + qv.y * x[t][2 * hh + 1]);
                    if (hh == 0) lo += pv; else hi += pv;
                }
            row_add(r_g1, lo, hi);
            // dW = -dU S^T -> B0 (row-major) and B3 (transposed)
            frag(L::TW + cD, x);
#pragma unroll
            for (int t = 0; t < CT; ++t)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = r0 + gid + 8 * hh, n = cD + 8 * t + 2 * tig;
                    const float w0 = rtf(-x[t][2 * hh]), w1 = rtf(-x[t][2 * hh + 1]);
                    *reinterpret_cast<float2*>(sm + L::B0 + pan(kCB, i, n)) = make_float2(w0, w1);
                    *reinterpret_cast<float*>(sm + L::B3 + pan(D, n, i)) = w0;
                    *reinterpret_cast<float*>(sm + L::B3 + pan(D, n + 1, i)) = w1;
                }
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int cc = 8 * ((warp >> 1) + 8 * u);
                float a[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = rtf(xk[u][j]);
                *reinterpret_cast<float4*>(sm + L::B2 + pan(kCB, rr, cc)) = make_float4(a[0], a[1], a[2], a[3]);
                *reinterpret_cast<float4*>(sm + L::B2 + pan(kCB, rr, cc + 4)) = make_float4(a[4], a[5], a[6], a[7]);
            }
        }
        sync_issue();
        if (tid == 0) {
            tc_gemm(tmem + L::TZ, sa + L::S0, sa + L::B3, D, kCB, ID_N, false);  // Z2 = T^T dW
            tc_gemm(tmem + L::TY, sa + L::B0, sa + L::B2, kCB, D, ID_64, false);  // Y' = dW k^T
            sm100::mma_commit(&bars[LB_P2]);
        }
        ok = wait_bar(LB_P2);
    }
    if (ok) {
        if (tid == 0) {  // dS' rows 0..63 -> B0, 64..127 -> B3 (dW, dW^T are read no more)
            copies |= 1u << LB_C3;
            sm100::mbar_arrive_expect_tx(&bars[LB_C3], (uint32_t)(D / 64) * L::BIG);
            tma_rec(sm + L::B0, &map_d, D, y_dS, &bars[LB_C3]);
            if constexpr (D == 128) tma_rec(sm + L::B3, &map_d, D, y_dS + 64, &bars[LB_C3]);
        }
        // Z2 = T^T dW: dk^ = diag(beta gam) Z2, d(beta gam) = k^ . Z2
        float z[CT][4];
        frag(L::TZ + cD, z);
        float lo = 0.f, hi = 0.f;
#pragma unroll
        for (int t = 0; t < CT; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = r0 + gid + 8 * hh, n = cD + 8 * t + 2 * tig;
                const float2 kv = tpair(L::B2, i, n);
                dka[t][2 * hh] = be[i] * gam[i] * z[t][2 * hh];
                dka[t][2 * hh + 1] = be[i] * gam[i] * z[t][2 * hh + 1];
                const float pv = rk[i] * (kv.x * z[t][2 * hh] + kv.y * z[t][2 * hh + 1]);
                if (hh == 0) lo += pv; else hi += pv;
            }
        row_add(r_dbg, lo, hi);
        // dT = (dU V^T + dW (gam K^)^T) diag(beta), K^ = diag(rk) k -> S2 transposed
        float xx[2][4], yy[2][4];
        frag(L::TX + c64, xx);
        frag(L::TY + c64, yy);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = r0 + gid + (e >> 1) * 8, j = c64 + 8 * t + 2 * tig + (e & 1);
                *reinterpret_cast<float*>(sm + L::S2 + pan(kCB, j, i)) =
                    rtf(be[j] * fmaf(gam[j] * rk[j], yy[t][e], xx[t][e]));
            }
        ok = wait_bar(LB_C2) && wait_bar(LB_C3);
        if (ok) {
            sync_issue();
            if (tid == 0) {
                tc_gemm(tmem + L::TX, sa + L::S0, sa + L::S2, kCB, kCB, ID_64, false);  // M2 = T^T dT
                tc_gemm(tmem + L::TW, sa + L::B4, sa + L::B0, kCB, D, ID_64, false);    // G2 = U dS'^T
                if constexpr (D == 128) tc_gemm(tmem + L::TW + 64, sa + L::B4, sa + L::B3, kCB, D, ID_64, false);
                tc_gemm(tmem + L::TG, sa + L::B1, sa + L::B4, kCB, D, ID_64, false);    // dP = dY U^T
                sm100::mma_commit(&bars[LB_P3]);
            }
            ok = wait_bar(LB_P3);
        }
    }
    if (ok) {
        // M2 -> S0 (T^T is read no more); dA' = M2 T^T
        float x[2][4];
        frag(L::TX + c64, x);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = r0 + gid + 8 * hh, j = c64 + 8 * t + 2 * tig;
                *reinterpret_cast<float2*>(sm + L::S0 + pan(kCB, i, j)) =
                    make_float2(rtf(x[t][2 * hh]), rtf(x[t][2 * hh + 1]));
            }
        sync_issue();
        if (tid == 0) {
            tc_gemm(tmem + L::TY, sa + L::S0, sa + L::S1, kCB, kCB, ID_64, false);
            sm100::mma_commit(&bars[LB_P4]);
        }
        // gC <S, dS'>: S from L2 (copied in by this CTA a moment ago), dS' from B0 / B3
        const float gC = expf(Lg[kCB - 1]);
        {
            float s = 0.f;
            constexpr int NE = D * D / 4 / 512;
            float4 a4[NE];
#pragma unroll
            for (int u = 0; u < NE; ++u) a4[u] = __ldg(reinterpret_cast<const float4*>(Sg) + tid + u * 512);
#pragma unroll
            for (int u = 0; u < NE; ++u) {
                const int e = (tid + u * 512) * 4, n = e / D, m = e % D;
                const float4 dd = *reinterpret_cast<const float4*>(sm + (n < 64 ? L::B0 : L::B3) + pan(kCB, n & 63, m));
                s = fmaf(a4[u].x, dd.x, fmaf(a4[u].y, dd.y, fmaf(a4[u].z, dd.z, fmaf(a4[u].w, dd.w, s))));
            }
            s = warp_sum(s);
            if (lane == 0) atomicAdd(red, s * gC);
        }
        // G2 = U dS'^T: dk^ += (gC / gam) G2, k^ . G2 = d (gC / gam_i)
        float y[CT][4];
        frag(L::TW + cD, y);
        float lo = 0.f, hi = 0.f;
#pragma unroll
        for (int t = 0; t < CT; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = r0 + gid + 8 * hh, n = cD + 8 * t + 2 * tig;
                const float dec = expf(Lg[kCB - 1] - Lg[i]);
                const float2 kv = tpair(L::B2, i, n);
                dka[t][2 * hh] = fmaf(dec, y[t][2 * hh], dka[t][2 * hh]);
                dka[t][2 * hh + 1] = fmaf(dec, y[t][2 * hh + 1], dka[t][2 * hh + 1]);
                const float pv = rk[i] * (kv.x * y[t][2 * hh] + kv.y * y[t][2 * hh + 1]);
                if (hh == 0) lo += pv; else hi += pv;
            }
        row_add(r_dr, lo, hi);
        ok = wait_bar(LB_P4);
    }
    if (ok) {
        // dA = -(T^T dT) T^T, strictly lower
        float da[2][4];
        frag(L::TY + c64, da);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = r0 + gid + (e >> 1) * 8, j = c64 + 8 * t + 2 * tig + (e & 1);
                da[t][e] = j < i ? -da[t][e] : 0.f;
            }
        // dP = dY U^T (lower-incl); the scalar terms of dA and dP; E = dA * beta_i Gam and
        // F = scale dP * Gam, stored as the products below take them against the unnormalised
        // k^T and q^T: E diag(rk), E^T diag(rk), F diag(rk) and F^T diag(rq)
        float x[2][4];
        frag(L::TG + c64, x);
        float mlo = 0.f, mhi = 0.f, plo = 0.f, phi = 0.f;
        float cs[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = r0 + gid + (e >> 1) * 8, j = c64 + 8 * t + 2 * tig + (e & 1);
                const float dp = j <= i ? x[t][e] : 0.f;
                const float at = Atg[i * kCB + j];
                const float mij = da[t][e] * be[i] * at + dp * Pg[i * kCB + j];
                if (e < 2) { mlo += mij; plo += da[t][e] * at; } else { mhi += mij; phi += da[t][e] * at; }
                cs[t][e & 1] += mij;
                const float gm = j <= i ? expf(fminf(Lg[i] - Lg[j], 0.f)) : 0.f;
                const float ev = da[t][e] * be[i] * gm, fv = scale * dp * gm;
                *reinterpret_cast<float*>(sm + L::S2 + pan(kCB, i, j)) = rtf(ev * rk[j]);  // E diag(rk)
                *reinterpret_cast<float*>(sm + L::S1 + pan(kCB, j, i)) = rtf(ev * rk[i]);  // E^T diag(rk)
                *reinterpret_cast<float*>(sm + L::B0 + pan(kCB, i, j)) = rtf(fv * rk[j]);  // F diag(rk)
                *reinterpret_cast<float*>(sm + L::B3 + pan(kCB, j, i)) = rtf(fv * rq[i]);  // F^T diag(rq)
            }
        row_add(rowM, mlo, mhi);
        row_add(r_dbe, plo, phi);
        // column sums: over the 8 row pairs of the quad column (lanes with equal tig)
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float v0 = cs[t][u];
                v0 += __shfl_xor_sync(0xffffffffu, v0, 4);
                v0 += __shfl_xor_sync(0xffffffffu, v0, 8);
                v0 += __shfl_xor_sync(0xffffffffu, v0, 16);
                if (gid == 0) atomicAdd(&colM[c64 + 8 * t + 2 * tig + u], v0);
            }
        // ---- stage 4: k^T (from k in B2) -> B1, q^T -> B4 (dY and U are read no more)
        const uint8_t* kk = sm + L::B2;
        stage<D>(nullptr, sm + L::B1, [kk](int i, int m, float* x8) { pan_ld8(kk, i, m, x8); }, tid);
        stage<D>(nullptr, sm + L::B4, tok(q), tid);
        sync_issue();
        if (tid == 0) {
            // dk^ += E K^ + E^T K^ + F^T Q^;  dq^ += F K^
            tc_gemm(tmem + L::TZ, sa + L::S2, sa + L::B1, D, kCB, ID_N, false);
            tc_gemm(tmem + L::TZ, sa + L::S1, sa + L::B1, D, kCB, ID_N, true);
            tc_gemm(tmem + L::TZ, sa + L::B3, sa + L::B4, D, kCB, ID_N, true);
            tc_gemm(tmem + L::TW, sa + L::B0, sa + L::B1, D, kCB, ID_N, false);
            sm100::mma_commit(&bars[LB_P5]);
        }
        ok = wait_bar(LB_P5);
    }
    if (ok) {
        float x[CT][4], qh[CT][4], kh2[CT][4];
        frag(L::TZ + cD, x);
#pragma unroll
        for (int t = 0; t < CT; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) dka[t][e] += x[t][e];
        frag(L::TW + cD, x);
#pragma unroll
        for (int t = 0; t < CT; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) dqa[t][e] += x[t][e];
        // row dots for the norm backward (k from B2, q from q^T in B4)
        float ql = 0.f, qh_ = 0.f, kl = 0.f, kh_ = 0.f;
#pragma unroll
        for (int t = 0; t < CT; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = r0 + gid + 8 * hh, n = cD + 8 * t + 2 * tig;
                const float2 kv = tpair(L::B2, i, n);
                qh[t][2 * hh] = rq[i] * *reinterpret_cast<const float*>(sm + L::B4 + pan(D, n, i));
                qh[t][2 * hh + 1] = rq[i] * *reinterpret_cast<const float*>(sm + L::B4 + pan(D, n + 1, i));
                kh2[t][2 * hh] = rk[i] * kv.x;
                kh2[t][2 * hh + 1] = rk[i] * kv.y;
                const float pq = qh[t][2 * hh] * dqa[t][2 * hh] + qh[t][2 * hh + 1] * dqa[t][2 * hh + 1];
                const float pk = kh2[t][2 * hh] * dka[t][2 * hh] + kh2[t][2 * hh + 1] * dka[t][2 * hh + 1];
                if (hh == 0) { ql += pq; kl += pk; } else { qh_ += pq; kh_ += pk; }
            }
        row_add(r_pq, ql, qh_);
        row_add(r_pk, kl, kh_);
        __syncthreads();
        // d Lg_i = gam_i d gam_i + rowM_i - colM_i (+ gC d gC for the last token); reverse cumsum
        if (warp < 2) {
            const int i = tid;
            const float dec = expf(Lg[kCB - 1] - Lg[i]);
            const float dlg = r_dbg[i] * be[i] * gam[i] + scale * gam[i] * r_g1[i] - r_dr[i] * dec;
            dLg[i] = dlg + rowM[i] - colM[i];
            const float rs = warp_sum(r_dr[i] * dec);
            if (lane == 0) atomicAdd(red, rs);
        }
        __syncthreads();
        if (warp == 0) {  // d ln(alpha_i) = red + sum_{i' >= i} dLg_i': lane l holds 2 l, 2 l + 1
            const float a0 = dLg[2 * lane], a1 = dLg[2 * lane + 1];
            float suf = a0 + a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += y;
            }
            const float base = red[0] + suf;
            dLg[2 * lane] = base;
            dLg[2 * lane + 1] = base - a0;
        }
        __syncthreads();
        float pA = 0.f, pba = 0.f;  // this token's share of dA_log[h], db_alpha[h] (gated form)
        if (tid < nv) {
            const int i = tid;
            const size_t o = tok_off(b, t0 + i, h, T, H);
            const float dbe = r_dbe[i] + r_dbg[i] * gam[i];
            if (A_log) {
                // ln alpha = -e^A softplus(x), x = a + b_alpha: d a = -e^A sigmoid(x) d ln alpha,
                // d A = ln alpha d ln alpha, d b_alpha = d a; beta = sigmoid(b): d b = beta (1-beta) d beta
                const float xa = alpha[o] + b_alpha[h], ea = expf(A_log[h]);
                const float dda = -ea * gate_sigmoid(xa) * dLg[i];
                dalpha[o] = dda;
                dbeta[o] = dbe * be[i] * (1.f - be[i]);
                pA = -ea * gate_softplus(xa) * dLg[i];
                pba = dda;
            } else {
                dalpha[o] = dLg[i] / alpha[o];
                dbeta[o] = dbe;
            }
        }
        if (A_log && tid < kCB) {  // warps 0 and 1, whole warps
            pA = warp_sum(pA);
            pba = warp_sum(pba);
            if (lane == 0) {
                atomicAdd(&dA_log[h], pA);
                atomicAdd(&db_alpha[h], pba);
            }
        }
        // dx = r (dx^ - x^ (x^ . dx^))
#pragma unroll
        for (int t = 0; t < CT; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = r0 + gid + 8 * hh, n = cD + 8 * t + 2 * tig;
                if (i < nv) {
                    const size_t o = tok_off(b, t0 + i, h, T, H) * D + n;
                    float gq[2], gk[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int e = 2 * hh + u;
                        gq[u] = l2norm ? rq[i] * (dqa[t][e] - qh[t][e] * r_pq[i]) : dqa[t][e];
                        gk[u] = l2norm ? rk[i] * (dka[t][e] - kh2[t][e] * r_pk[i]) : dka[t][e];
                    }
                    st2(dq + o, gq[0], gq[1]);
                    st2(dk + o, gk[0], gk[1]);
                }
            }
    }
    if (!ok && tid == 0) {
        // a wait gave up: record it, let the issued products and copies drain, then release TMEM
        record_status(status, GDN_ERR_TIMEOUT);
        sm100::mma_commit(&bars[LB_DRAIN]);
        sm100::mbar_wait(&bars[LB_DRAIN], 0, never, 100000000ull);
        for (int i = LB_C0; i <= LB_C3; ++i)
            if (copies & (1u << i)) sm100::mbar_wait(&bars[i], 0, never, 100000000ull);
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, L::TCOLS);
    }
}

// 2-D tensor map over the workspace viewed as rows of C fp32 values: box 32 x 64 (one 64-row panel
// of 128-byte rows), 128-byte swizzle.
typedef CUresult (*BwdEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                CUtensorMapFloatOOBfill);
BwdEncodeFn bwd_encode_fn() {
    static const BwdEncodeFn fn = [] {
        cudaDriverEntryPointQueryResult qr;
        void* f = nullptr;
        return (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &qr) == cudaSuccess &&
                qr == cudaDriverEntryPointSuccess)
                   ? reinterpret_cast<BwdEncodeFn>(f)
                   : nullptr;
    }();
    return fn;
}
bool make_ws_map(CUtensorMap* m, void* base, size_t rows, int C) {
    const BwdEncodeFn enc = bwd_encode_fn();
    if (!enc || (reinterpret_cast<uintptr_t>(base) & 15u)) return false;
    cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)C * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)kCB};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D tensor map over a [B T, H, D] bf16 token tensor: box 64 (features) x 1 (head) x 64 (tokens),
// 128-byte swizzle.
bool make_tok_map(CUtensorMap* m, const void* base, long tokens, int H, int D) {
    const BwdEncodeFn enc = bwd_encode_fn();
    if (!enc || (reinterpret_cast<uintptr_t>(base) & 15u)) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kCB};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D tensor map over a row-major bf16 array of `rows` x C (C = 64 or 128): box 64 x 64, 128-byte
// swizzle (the split images of -W and P).
bool make_img_map(CUtensorMap* m, void* base, size_t rows, int C) {
    const BwdEncodeFn enc = bwd_encode_fn();
    if (!enc || (reinterpret_cast<uintptr_t>(base) & 15u)) return false;
    cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)C * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kCB};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, typename Tin>
cudaError_t launch_chunked(const BackwardArgs& a, cudaStream_t st) {
    const int nch = (a.T + kCB - 1) / kCB;
    const BwdChunkWs w = bwdc_ws(a.B, a.T, a.H, D);
    if (a.ws == nullptr || a.ws_bytes < w.total * sizeof(float)) return cudaErrorInvalidValue;
    float* ws = static_cast<float*>(a.ws);
    CUtensorMap map_d, map_64;  // the workspace as rows of D and of 64 floats (bwdc_local's copies)
    if (!make_ws_map(&map_d, ws, w.total / D, D) || !make_ws_map(&map_64, ws, w.total / kCB, kCB))
        return cudaErrorInvalidValue;
    const Tin* q = static_cast<const Tin*>(a.q);
    const Tin* k = static_cast<const Tin*>(a.k);
    const Tin* v = static_cast<const Tin*>(a.v);
    const Tin* dy = static_cast<const Tin*>(a.dy);
    const unsigned R = (unsigned)((size_t)a.B * nch * a.H);
    const unsigned chains = (unsigned)(a.B * a.H * (D / kNVB));
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(bwdc_prep<D, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PrepB<D>::BYTES)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwdc_fwd<D, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  ChainB<D>::FWD_BYTES)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwdc_rev<D, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  ChainB<D>::REV_BYTES)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwdc_local<D, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  LocalB<D>::BYTES)) != cudaSuccess)
        return e;
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
        CUtensorMap mq, mk, mv, mdy, mwi, mpi;
        const long tokens = (long)a.B * a.T;
        if (!make_tok_map(&mq, q, tokens, a.H, D) || !make_tok_map(&mk, k, tokens, a.H, D) ||
            !make_tok_map(&mv, v, tokens, a.H, D) || !make_tok_map(&mdy, dy, tokens, a.H, D) ||
            !make_img_map(&mwi, ws + w.Wi, (size_t)R * 2 * kCB, D) ||
            !make_img_map(&mpi, ws + w.Pi, (size_t)R * 2 * kCB, kCB))
            return cudaErrorInvalidValue;
        if ((e = cudaFuncSetAttribute(bwdc_prep_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      PrepTC<D>::BYTES)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(bwdc_fwd_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      FwdTC<D>::BYTES)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(bwdc_rev_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      RevTC<D>::BYTES)) != cudaSuccess)
            return e;
        bwdc_prep_tc<D><<<R, 256, PrepTC<D>::BYTES, st>>>(a.alpha, a.beta, ws, w, a.T, a.H, nch, a.scale,
                                                          a.l2norm, a.A_log, a.b_alpha, a.status, mq, mk, mv);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const unsigned slice_ctas = (unsigned)(a.B * a.H * (D / 64));  // 64-column state slices
        bwdc_fwd_tc<D><<<slice_ctas, 256, FwdTC<D>::BYTES, st>>>(a.s0, ws, w, a.T, a.H, nch, a.status, mk, mwi);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        bwdc_rev_tc<D><<<slice_ctas, 256, RevTC<D>::BYTES, st>>>(a.ds_final, a.ds0, ws, w, a.T, a.H, nch,
                                                                 a.scale, a.status, mq, mk, mdy, mwi, mpi);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else {
        bwdc_prep<D, Tin><<<R, 256, PrepB<D>::BYTES, st>>>(q, k, v, a.alpha, a.beta, ws, w, a.T, a.H, nch,
                                                            a.scale, a.l2norm, a.A_log, a.b_alpha);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        bwdc_fwd<D, Tin><<<chains, 256, ChainB<D>::FWD_BYTES, st>>>(k, a.s0, ws, w, a.T, a.H, nch);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        bwdc_rev<D, Tin><<<chains, 256, ChainB<D>::REV_BYTES, st>>>(q, k, dy, a.ds_final, a.ds0, ws, w, a.T,
                                                                     a.H, nch, a.scale);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (a.A_log) {
        if ((e = cudaMemsetAsync(a.dA_log, 0, sizeof(float) * a.H, st)) != cudaSuccess ||
            (e = cudaMemsetAsync(a.db_alpha, 0, sizeof(float) * a.H, st)) != cudaSuccess)
            return e;
    }
    bwdc_local<D, Tin><<<R, 512, LocalB<D>::BYTES, st>>>(
        q, k, v, dy, a.alpha, static_cast<Tin*>(a.dq), static_cast<Tin*>(a.dk), static_cast<Tin*>(a.dv),
        a.dalpha, a.dbeta, ws, w, a.T, a.H, nch, a.scale, a.l2norm, a.A_log, a.b_alpha, a.dA_log,
        a.db_alpha, a.status, map_d, map_64);
    return cudaGetLastError();
}

}  // namespace

size_t backward_chunked_workspace_bytes(int B, int T, int H, int dk, int dv) {
    (void)dv;
    return bwdc_ws(B, T, H, dk).total * sizeof(float);
}

cudaError_t launch_backward_chunked(const BackwardArgs& a, cudaStream_t st) {
    if (a.dtype == GDN_BF16)
        return a.dkdim == 128 ? launch_chunked<128, __nv_bfloat16>(a, st)
                              : launch_chunked<64, __nv_bfloat16>(a, st);
    return a.dkdim == 128 ? launch_chunked<128, float>(a, st) : launch_chunked<64, float>(a, st);
}

}  // namespace gdn
