// backward.cu -- reverse-mode gradients of the gated delta rule, token-loop form: the path of
// gdn_backward_noalloc, whose scratch is a fixed array (gdn_backward runs the chunked form in
// backward_chunk.cu).
//
// Forward (Qwen3.8-Flash-Next summary, picx.dev, "Theoretical foundations", eqs. (1)-(4)), per
// head with normalised kh, qh:  St = a S;  e = v - St^T kh;  S' = St + b kh e^T;  y = scale S'^T qh.
// The derivative is taken token by token in reverse (the chain rule applied to those four
// steps), with dS = dL/dS' carried backwards:
//     dS += scale qh dy^T;   dqh = scale S' dy
//     db  = kh^T dS e;        de = b dS^T kh;        dkh = b dS e - St de;      dv = de
//     dSt = dS - kh de^T;     da = <dSt, S>;         dS  = a dSt
// and dS0 is the final dS.  Gradients reach the raw q, k through the L2 normalisation:
// dx = (dxh - xh <xh, dxh>) / sqrt(|x|^2 + eps).
//
// Two kernels, one CTA per (sequence, head), fp32 state in registers:
//   ckpt_kernel  forward over the sequence, storing the state at every 64-token chunk start
//                (workspace part 1: [B*H][nchunks][dk][dv]);
//   bwd_kernel   chunks in reverse: replay the chunk forward from its checkpoint, storing the 64
//                per-token states (workspace part 2: [B*H][64][dk][dv]), then walk the chunk's
//                tokens backwards.  Per-token k_hat, q_hat and the row gradients live in shared
//                memory; the norm backward is applied once per chunk.
// Thread layout: warp w owns rows 8w..8w+7 of the dk x dv state, lane l owns columns
// [l*CPL, l*CPL + CPL).  Column (dk) reductions go through shared memory, row (dv) reductions
// through warp shuffles.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace gdn {

namespace {

constexpr int kC = 64;  // tokens per chunk (checkpoint spacing)

template <int D>
struct BwdCfg {
    static constexpr int NW = D / 8;          // warps
    static constexpr int NT = NW * 32;        // threads
    static constexpr int CPL = D / 32;        // columns per lane
    static constexpr int E = 8 * CPL;         // state elements per thread
};

template <int CPL>
struct Vec;
template <>
struct Vec<4> {
    static __device__ __forceinline__ void load(const float* p, float* x) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* x) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};
template <>
struct Vec<2> {
    static __device__ __forceinline__ void load(const float* p, float* x) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x[0] = v.x; x[1] = v.y;
    }
    static __device__ __forceinline__ void store(float* p, const float* x) {
        *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    }
};

template <typename T>
__device__ __forceinline__ void load_cols(const T* p, float* x, int n) {
    for (int j = 0; j < n; ++j) x[j] = to_f32(p[j]);
}

// Normalise one token's q and k (a warp per token) into shared memory.
template <int D, typename T>
__device__ __forceinline__ void norm_token(const T* q, const T* k, float* qh, float* kh,
                                           float* rq_out, float* rk_out, float* kq_out,
                                           int l2norm, int lane) {
    constexpr int PL = D / 32;
    float qv[PL], kv[PL], sq = 0.f, sk = 0.f;
#pragma unroll
    for (int j = 0; j < PL; ++j) {
        qv[j] = to_f32(q[lane + 32 * j]);
        kv[j] = to_f32(k[lane + 32 * j]);
        sq += qv[j] * qv[j];
        sk += kv[j] * kv[j];
    }
    sq = warp_sum(sq);
    sk = warp_sum(sk);
    const float rq = l2norm ? 1.0f / sqrtf(sq + kNormEps) : 1.f;
    const float rk = l2norm ? 1.0f / sqrtf(sk + kNormEps) : 1.f;
    float kq = 0.f;
#pragma unroll
    for (int j = 0; j < PL; ++j) {
        qh[lane + 32 * j] = qv[j] * rq;
        kh[lane + 32 * j] = kv[j] * rk;
        kq += qv[j] * rq * kv[j] * rk;
    }
    kq = warp_sum(kq);
    if (lane == 0) {
        *rq_out = rq;
        *rk_out = rk;
        *kq_out = kq;
    }
}

// ----------------------------------------------------------------------------- checkpoints
template <int D, typename T>
__global__ void __launch_bounds__(BwdCfg<D>::NT)
ckpt_kernel(const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ alpha,
            const float* __restrict__ beta, const float* __restrict__ s0, float* __restrict__ ckpt,
            int T_len, int H, int l2norm) {
    using C = BwdCfg<D>;
    constexpr int CPL = C::CPL;
    __shared__ float s_kh[D];
    __shared__ float s_red[2][C::NW][D];
    const int chain = blockIdx.x;  // b * H + h
    const int b = chain / H, h = chain % H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c0 = lane * CPL;
    const int nchunks = (T_len + kC - 1) / kC;
    float S[8][CPL];
    const size_t soff = (size_t)chain * D * D;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = warp * 8 + i;
        if (s0) Vec<CPL>::load(s0 + soff + (size_t)r * D + c0, S[i]);
        else
#pragma unroll
            for (int j = 0; j < CPL; ++j) S[i][j] = 0.f;
    }
    for (int t = 0; t < T_len; ++t) {
        if (t % kC == 0) {
            float* dst = ckpt + ((size_t)chain * nchunks + t / kC) * D * D;
#pragma unroll
            for (int i = 0; i < 8; ++i) Vec<CPL>::store(dst + (size_t)(warp * 8 + i) * D + c0, S[i]);
        }
        const size_t th = ((size_t)b * T_len + t) * H + h;
        if (warp == 0) {
            constexpr int PL = D / 32;
            float kv[PL], sk = 0.f;
#pragma unroll
            for (int j = 0; j < PL; ++j) {
                kv[j] = to_f32(k[th * D + lane + 32 * j]);
                sk += kv[j] * kv[j];
            }
            sk = warp_sum(sk);
            const float rk = l2norm ? 1.0f / sqrtf(sk + kNormEps) : 1.f;
#pragma unroll
            for (int j = 0; j < PL; ++j) s_kh[lane + 32 * j] = kv[j] * rk;
        }
        __syncthreads();
        const float a = alpha[th], bb = beta[th];
        float part[CPL] = {};
        float khr[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            khr[i] = s_kh[warp * 8 + i];
#pragma unroll
            for (int j = 0; j < CPL; ++j) part[j] = fmaf(S[i][j], khr[i], part[j]);
        }
        float* red = s_red[t & 1][0];
#pragma unroll
        for (int j = 0; j < CPL; ++j) red[warp * D + c0 + j] = part[j];
        __syncthreads();
        float e[CPL];
        float vv[CPL];
        load_cols(v + th * D + c0, vv, CPL);
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            float p = 0.f;
#pragma unroll
            for (int w = 0; w < C::NW; ++w) p += red[w * D + c0 + j];
            e[j] = vv[j] - a * p;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < CPL; ++j) S[i][j] = fmaf(a, S[i][j], bb * khr[i] * e[j]);
    }
}

// ----------------------------------------------------------------------------- backward
struct BwdParams {
    const void *q, *k, *v, *dy;
    const float *alpha, *beta, *ds_final;
    void *dq, *dk, *dv;
    float *dalpha, *dbeta, *ds0;
    const float* ckpt;
    float* tok;  // [B*H][64][D][D]
    int T_len, H;
    float scale;
    int l2norm;
};

template <int D>
struct BwdSmem {
    float kh[kC][D];
    float qh[kC][D];
    float dkh[kC][D];
    float dqh[kC][D];
    float red[2][BwdCfg<D>::NW][2][D];
    float part[BwdCfg<D>::NW][kC][2];
    float rk[kC], rq[kC], kq[kC], a[kC], b[kC];
};

template <int D, typename T>
__global__ void __launch_bounds__(BwdCfg<D>::NT, 1) bwd_kernel(const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr int CPL = C::CPL, NW = C::NW;
    extern __shared__ uint8_t smem_raw[];
    BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(smem_raw);
    const T* q = static_cast<const T*>(p.q);
    const T* k = static_cast<const T*>(p.k);
    const T* v = static_cast<const T*>(p.v);
    const T* dy = static_cast<const T*>(p.dy);
    T* dq = static_cast<T*>(p.dq);
    T* dk = static_cast<T*>(p.dk);
    T* dvo = static_cast<T*>(p.dv);
    const int chain = blockIdx.x;
    const int H = p.H, T_len = p.T_len;
    const int b = chain / H, h = chain % H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c0 = lane * CPL;
    const int nchunks = (T_len + kC - 1) / kC;
    const size_t soff = (size_t)chain * D * D;
    float* tok = p.tok + (size_t)chain * kC * D * D;

    float dS[8][CPL];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = warp * 8 + i;
        if (p.ds_final) Vec<CPL>::load(p.ds_final + soff + (size_t)r * D + c0, dS[i]);
        else
#pragma unroll
            for (int j = 0; j < CPL; ++j) dS[i][j] = 0.f;
    }

    for (int ci = nchunks - 1; ci >= 0; --ci) {
        const int t0 = ci * kC;
        const int n = min(kC, T_len - t0);
        // per-token normalised q, k and gates of this chunk
        for (int u = warp; u < n; u += NW) {
            const size_t th = ((size_t)b * T_len + t0 + u) * H + h;
            norm_token<D, T>(q + th * D, k + th * D, sm.qh[u], sm.kh[u], &sm.rq[u], &sm.rk[u],
                             &sm.kq[u], p.l2norm, lane);
            if (lane == 0) {
                sm.a[u] = p.alpha[th];
                sm.b[u] = p.beta[th];
            }
        }
        __syncthreads();

        // replay the chunk forward from its checkpoint; tok[u] = state before token u
        {
            float S[8][CPL];
            const float* ck = p.ckpt + ((size_t)chain * nchunks + ci) * D * D;
#pragma unroll
            for (int i = 0; i < 8; ++i) Vec<CPL>::load(ck + (size_t)(warp * 8 + i) * D + c0, S[i]);
            for (int u = 0; u < n; ++u) {
                float* dst = tok + (size_t)u * D * D;
                float part[CPL] = {};
                float khr[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    Vec<CPL>::store(dst + (size_t)(warp * 8 + i) * D + c0, S[i]);
                    khr[i] = sm.kh[u][warp * 8 + i];
#pragma unroll
                    for (int j = 0; j < CPL; ++j) part[j] = fmaf(S[i][j], khr[i], part[j]);
                }
                float* red = sm.red[u & 1][0][0];
#pragma unroll
                for (int j = 0; j < CPL; ++j) red[warp * 2 * D + c0 + j] = part[j];
                __syncthreads();
                const size_t th = ((size_t)b * T_len + t0 + u) * H + h;
                float vv[CPL];
                load_cols(v + th * D + c0, vv, CPL);
                const float a = sm.a[u], bb = sm.b[u];
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    float pk = 0.f;
#pragma unroll
                    for (int w = 0; w < NW; ++w) pk += red[w * 2 * D + c0 + j];
                    const float e = vv[j] - a * pk;
#pragma unroll
                    for (int i = 0; i < 8; ++i) S[i][j] = fmaf(a, S[i][j], bb * khr[i] * e);
                }
            }
        }
        __syncthreads();

        // reverse through the chunk
        for (int u = n - 1; u >= 0; --u) {
            const size_t th = ((size_t)b * T_len + t0 + u) * H + h;
            const float* src = tok + (size_t)u * D * D;
            float Sp[8][CPL];
            float khr[8], qhr[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                Vec<CPL>::load(src + (size_t)(warp * 8 + i) * D + c0, Sp[i]);
                khr[i] = sm.kh[u][warp * 8 + i];
                qhr[i] = sm.qh[u][warp * 8 + i];
            }
            // column sums of Sp^T kh and dS^T kh (before adding scale qh dy^T)
            float p1[CPL] = {}, p2[CPL] = {};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    p1[j] = fmaf(Sp[i][j], khr[i], p1[j]);
                    p2[j] = fmaf(dS[i][j], khr[i], p2[j]);
                }
            float* red = sm.red[u & 1][0][0];
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                red[(warp * 2 + 0) * D + c0 + j] = p1[j];
                red[(warp * 2 + 1) * D + c0 + j] = p2[j];
            }
            __syncthreads();
            const float a = sm.a[u], bb = sm.b[u], kq = sm.kq[u];
            float vv[CPL], dyv[CPL], e[CPL], de[CPL];
            load_cols(v + th * D + c0, vv, CPL);
            load_cols(dy + th * D + c0, dyv, CPL);
            float edy = 0.f;
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                float pk = 0.f, dsk = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    pk += red[(w * 2 + 0) * D + c0 + j];
                    dsk += red[(w * 2 + 1) * D + c0 + j];
                }
                e[j] = vv[j] - a * pk;
                // dS gains scale qh dy^T before its transpose meets kh
                de[j] = bb * (dsk + p.scale * kq * dyv[j]);
                edy = fmaf(e[j], dyv[j], edy);
            }
            edy = warp_sum(edy);
            if (warp == 0) {
                T* dvp = dvo + th * D + c0;
#pragma unroll
                for (int j = 0; j < CPL; ++j) dvp[j] = from_f32<T>(de[j]);
            }
            // row quantities: Sp dy, dS e (after the output term), Sp de
            float dqh_acc[8], dse[8], spde[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float x = 0.f, y = 0.f, z = 0.f;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    dS[i][j] = fmaf(p.scale * qhr[i], dyv[j], dS[i][j]);
                    x = fmaf(Sp[i][j], dyv[j], x);
                    y = fmaf(dS[i][j], e[j], y);
                    z = fmaf(Sp[i][j], de[j], z);
                }
                dqh_acc[i] = warp_sum(x);
                dse[i] = warp_sum(y);
                spde[i] = warp_sum(z);
            }
            float dbp = 0.f, dap = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = warp * 8 + i;
                // dqh = scale S' dy with S' = a Sp + b kh e^T
                const float dqh = p.scale * (a * dqh_acc[i] + bb * khr[i] * edy);
                const float dkh = bb * dse[i] - a * spde[i];
                if (lane == i) {
                    sm.dqh[u][r] = dqh;
                    sm.dkh[u][r] = dkh;
                }
                dbp = fmaf(khr[i], dse[i], dbp);
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    const float dst = dS[i][j] - khr[i] * de[j];
                    dap = fmaf(dst, Sp[i][j], dap);
                    dS[i][j] = a * dst;
                }
            }
            dap = warp_sum(dap);
            if (lane == 0) {
                sm.part[warp][u][0] = dap;
                sm.part[warp][u][1] = dbp;  // already identical on all lanes
            }
        }
        __syncthreads();
        // gate gradients and the norm backward for the chunk's tokens
        for (int u = threadIdx.x; u < n; u += C::NT) {
            float da = 0.f, db = 0.f;
            for (int w = 0; w < NW; ++w) {
                da += sm.part[w][u][0];
                db += sm.part[w][u][1];
            }
            const size_t th = ((size_t)b * T_len + t0 + u) * H + h;
            p.dalpha[th] = da;
            p.dbeta[th] = db;
        }
        for (int u = warp; u < n; u += NW) {
            const size_t th = ((size_t)b * T_len + t0 + u) * H + h;
            constexpr int PL = D / 32;
            float xk = 0.f, xq = 0.f;
#pragma unroll
            for (int j = 0; j < PL; ++j) {
                const int c = lane + 32 * j;
                xk = fmaf(sm.kh[u][c], sm.dkh[u][c], xk);
                xq = fmaf(sm.qh[u][c], sm.dqh[u][c], xq);
            }
            xk = warp_sum(xk);
            xq = warp_sum(xq);
            const float rk = sm.rk[u], rq = sm.rq[u];
#pragma unroll
            for (int j = 0; j < PL; ++j) {
                const int c = lane + 32 * j;
                float gk = sm.dkh[u][c], gq = sm.dqh[u][c];
                if (p.l2norm) {
                    gk = (gk - sm.kh[u][c] * xk) * rk;
                    gq = (gq - sm.qh[u][c] * xq) * rq;
                }
                dk[th * D + c] = from_f32<T>(gk);
                dq[th * D + c] = from_f32<T>(gq);
            }
        }
        __syncthreads();
    }
    if (p.ds0) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            Vec<CPL>::store(p.ds0 + soff + (size_t)(warp * 8 + i) * D + c0, dS[i]);
    }
}

template <int D, typename T>
cudaError_t launch_t(const BackwardArgs& a, cudaStream_t st) {
    using C = BwdCfg<D>;
    const int chains = a.B * a.H;
    const int nchunks = (a.T + kC - 1) / kC;
    float* ckpt = static_cast<float*>(a.ws);
    float* tok = ckpt + (size_t)chains * nchunks * D * D;
    ckpt_kernel<D, T><<<chains, C::NT, 0, st>>>(static_cast<const T*>(a.k),
                                                static_cast<const T*>(a.v), a.alpha, a.beta,
                                                a.s0, ckpt, a.T, a.H, a.l2norm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    BwdParams p{a.q, a.k, a.v, a.dy, a.alpha, a.beta, a.ds_final, a.dq, a.dk, a.dv,
                a.dalpha, a.dbeta, a.ds0, ckpt, tok, a.T, a.H, a.scale, a.l2norm};
    const int smem = (int)sizeof(BwdSmem<D>);
    e = cudaFuncSetAttribute(bwd_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    bwd_kernel<D, T><<<chains, C::NT, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

// ----------------------------------------------------------------------------- fixed scratch
// Scratch for gdn_backward_noalloc: a file-scope device array that every GPU loading the
// library holds until the process exits.  Host code must never hand g_bwd_fixed_scratch itself
// to a kernel (on the host the name is only a stand-in for the symbol, not a device address);
// the device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_bwd_fixed_scratch[kBackwardFixedScratchBytes];

namespace {
std::mutex g_fixed_mu;
void* g_fixed_ptr[64] = {};
}  // namespace

int backward_fixed_scratch(void** ptr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_fixed_mu);
    if (!g_fixed_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bwd_fixed_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return GDN_ERR_CUDA;
        }
        g_fixed_ptr[dev] = p;
    }
    *ptr = g_fixed_ptr[dev];
    return GDN_OK;
}

size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv) {
    const size_t chunks = (size_t)(T + kC - 1) / kC;
    return (chunks + kC) * (size_t)B * H * dk * dv * sizeof(float);
}

cudaError_t launch_backward_tokenloop(const BackwardArgs& a, cudaStream_t st) {
    if (a.dtype == GDN_BF16)
        return a.dkdim == 128 ? launch_t<128, __nv_bfloat16>(a, st) : launch_t<64, __nv_bfloat16>(a, st);
    return a.dkdim == 128 ? launch_t<128, float>(a, st) : launch_t<64, float>(a, st);
}

}  // namespace gdn
