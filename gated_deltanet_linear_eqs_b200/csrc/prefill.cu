// prefill.cu -- chunked (64-token) gated-delta-rule forward on the sm_100a tensor cores.
//
// Method: eqs. (1)-(4) of the Qwen3.8-Flash-Next summary (picx.dev, "Theoretical foundations")
// with L2-normalised q and k ("Methodology", "1. GDN Hybrid Token Mixing"), evaluated chunk by
// chunk in the WY/UT form (the chunkwise gated delta rule of Yang, Kautz & Hatamizadeh 2024).
// For a chunk of C = 64 tokens starting from state S (dk x dv), with G = inclusive cumsum of
// log2(alpha), gamma = 2^G, Gam_ij = 2^(G_i - G_j):
//
//   A   = strictly-lower( diag(beta) (Kh Kh^T * Gam) ),   T = (I + A)^-1
//   W   = T diag(beta gamma) Kh         Ut = diag(beta) V + strict(T) diag(beta) V
//   U   = Ut - W S                      (the chunk's pseudo-values, beta included)
//   Y   = scale ( diag(gamma) Qh S + (Qh Kh^T * Gam * lower-incl) U )
//   S'  = gamma_C S + Kh^T diag(Gam_C,.) U
//
// Kh = diag(rk) K, Qh = diag(rq) Q are the normalised rows; the norms are applied as fp32 row or
// column scales so that the MMA operands K, Q, V stay the exact bf16 inputs.
//
// A, T, W, Ut and P = scale diag(rq) (Q K^T * Gam * lower-incl) diag(rk) depend on the chunk
// alone; only U, Y and S' need the state.  The forward therefore runs as
//   chunk-base scan (packed documents only): first record index of every document
//   prep kernel   one CTA per (chunk, head), every chunk of every document at once: decay, norms,
//                 A and P, the 64x64 triangular inverse, W and Ut, written to a workspace record
//                 as ready-made tensor-core operand tiles
//   chain kernel  one CTA per (document, head, 64-column slice of dv) walks its chunks in order
//                 with the fp32 state in registers: U = Ut - W S, S' and Y on the tensor cores.
// Only the chain kernel is sequential, and it does the state-dependent work alone.
//
// Workspace record of (chunk record g, head h), r = g * H + h:
//   W  [r][dk/64][64 tokens][128 B]  -W, bf16, 128-byte swizzled rows (K-major MMA operand)
//   P  [r][64 tokens][128 B]          P, bf16, 128-byte swizzled rows
//   U  [r][dv/64][64 tokens][256 B]   Ut, fp32, 16-byte chunk q of row i at position q ^ (i % 8)
//   SC [r][256] fp32                  [0,64) rk_i Gam_C/gamma_i (0 past the end), [64,128)
//                                     scale gamma_i rq_i, [128] gamma_C
#include <mutex>

// The prefill kernels carry bounds guards (shared-memory rows, global extents), each recording
// the failing index in the device status words and skipping the access.
#ifndef GDN_DEBUG
#define GDN_DEBUG 1
#endif
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kChunk = 64;
constexpr int kLd = 72;  // bf16 row stride (elements) of the A / T scratch: 144-byte rows
constexpr int kNV = 32;  // dv columns per chain CTA (operand tiles stay 64 columns wide)
constexpr uint32_t kRecP = 8192;
constexpr uint32_t kRecS = 1024;

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
}
__device__ __forceinline__ void unpack8(const uint4& u, float* x) {
    float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z), d = unpack_bf16(u.w);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y; x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
}
__device__ __forceinline__ uint4 pack8(const float* x) {
    return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                      pack_bf16(x[6], x[7]));
}
// Round-to-nearest bf16 pair on the FP32 pipe instead of the conversion unit (which runs at a
// fraction of the FP32 rate): Veltkamp's splitting with the factor 2^16 + 1 leaves the 8
// leading significand bits of x in hi (the low 16 bits of hi are zero), and the two upper halves
// are packed with one byte permute.  Valid for |x| < 2^111.
__device__ __forceinline__ uint32_t pack_bf16_fma(float a, float b) {
    const float ca = __fmul_rn(a, 65537.f), cb = __fmul_rn(b, 65537.f);
    const float ha = __fsub_rn(ca, __fsub_rn(ca, a)), hb = __fsub_rn(cb, __fsub_rn(cb, b));
    return __byte_perm(__float_as_uint(ha), __float_as_uint(hb), 0x7632);
}
__device__ __forceinline__ uint4 pack8_fma(const float* x) {
    return make_uint4(pack_bf16_fma(x[0], x[1]), pack_bf16_fma(x[2], x[3]),
                      pack_bf16_fma(x[4], x[5]), pack_bf16_fma(x[6], x[7]));
}
// 32 floats -> 4 swizzled 16-byte chunks, half of them rounded on each pipe
__device__ __forceinline__ void store_half_row_mixed(uint8_t* tile, int row, int c0, const float* x) {
    *reinterpret_cast<uint4*>(tile + swz(row, c0 + 0)) = pack8(x);
    *reinterpret_cast<uint4*>(tile + swz(row, c0 + 1)) = pack8_fma(x + 8);
    *reinterpret_cast<uint4*>(tile + swz(row, c0 + 2)) = pack8(x + 16);
    *reinterpret_cast<uint4*>(tile + swz(row, c0 + 3)) = pack8_fma(x + 24);
}
// 32 floats -> 4 swizzled 16-byte chunks (chunk index c0..c0+3) of a 128-byte bf16 row
// (shared or global memory: the same tile image)
__device__ __forceinline__ void store_half_row(uint8_t* tile, int row, int c0, const float* x) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(tile + swz(row, c0 + c)) = pack8(x + 8 * c);
}
__device__ __forceinline__ void load_half_row(const uint8_t* tile, int row, int c0, float* x) {
#pragma unroll
    for (int c = 0; c < 4; ++c) unpack8(*reinterpret_cast<const uint4*>(tile + swz(row, c0 + c)), x + 8 * c);
}
// Sum of squares of one swizzled bf16 row of 64 elements.
__device__ __forceinline__ float row_sumsq(const uint8_t* tile, int row) {
    float s[8] = {};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float x[8];
        unpack8(*reinterpret_cast<const uint4*>(tile + swz(row, c)), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) s[e] = fmaf(x[e], x[e], s[e]);
    }
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ============================================================================ chunk-base scan
// cb[n] = sum over documents m < n of ceil(len_m / 64); cb[num_seqs] = total chunk records.
// Then, for every record g < nrec, map[g] = (first token, valid tokens) of the chunk it holds
// ((0, 0) past the last record), so that a prep CTA finds its chunk with one load.
constexpr int kMapSmem = 8192;  // documents whose bases are searched in shared memory
__global__ void __launch_bounds__(1024) chunk_base_kernel(const int32_t* __restrict__ cu, int n,
                                                           int nrec, int32_t* __restrict__ cb,
                                                           int2* __restrict__ map) {
    __shared__ int wsum[32];
    __shared__ int carry;
    __shared__ int scb[kMapSmem + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < n; base += 1024) {
        const int i = base + tid;
        int v = 0;
        if (i < n) {
            const int len = cu[i + 1] - cu[i];
            v = len > 0 ? (len + kChunk - 1) / kChunk : 0;
        }
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int s = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            wsum[lane] = s;
        }
        __syncthreads();
        const int incl = carry + (warp > 0 ? wsum[warp - 1] : 0) + x;
        if (i < n) cb[i] = incl - v;
        __syncthreads();
        if (tid == 1023) carry = incl;
        __syncthreads();
    }
    if (tid == 0) cb[n] = carry;
    __syncthreads();
    const bool in_smem = n <= kMapSmem;
    if (in_smem)
        for (int i = tid; i <= n; i += 1024) scb[i] = cb[i];
    __syncthreads();
    const int total = carry;
    for (int g = tid; g < nrec; g += 1024) {
        int2 m = make_int2(0, 0);
        if (g < total) {
            int lo = 0, hi = n;  // the last document whose first record is <= g
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if ((in_smem ? scb[mid] : cb[mid]) <= g) lo = mid; else hi = mid - 1;
            }
            const int t0 = cu[lo] + (g - (in_smem ? scb[lo] : cb[lo])) * kChunk;
            m = make_int2(t0, min(kChunk, cu[lo + 1] - t0));
        }
        map[g] = m;
    }
}

// ============================================================================ prep kernel
template <int D>
struct PrepLayout {
    static constexpr int KB = D / 64;
    static constexpr int KQ = 0;                      // per dk block: K rows 0-63, Q rows 64-127
    static constexpr int V = KB * 16384;              // V: dv/64 blocks of 64 tokens x 64 columns
    static constexpr int AF = V + KB * 8192;          // A, bf16 64 x kLd
    static constexpr int TF = AF + 64 * kLd * 2;      // T, bf16 64 x kLd
    static constexpr int TWN = AF;                    // 128 rows: T_w (0-63), N_b (64-127), written
                                                      // over A and T once T is in registers
    static constexpr int XB = TF + 64 * kLd * 2;      // 4 warps x 16 x 24 bf16
    static constexpr int AB = XB + 4 * 16 * 24 * 2;   // alpha[64], beta[64]
    static constexpr int SC = AB + 512;               // scalar arrays, 64 floats each
    static constexpr int BAR = SC + 8 * 256;
    static constexpr int MISC = BAR + 8 * 8;          // tmem base, abort flag, zero word
    static constexpr int BYTES = MISC + 16;
    static constexpr int TX = KB * 16384 + KB * 8192;
    static constexpr uint32_t T_D1 = 0;               // [K K^T | Q K^T] (64 columns), then
    static constexpr uint32_t T_D3 = 0;               // W (D columns, lanes 0-63)
    static constexpr uint32_t T_DU = D;               // N_b V (D columns, lanes 64-127)
    static constexpr uint32_t T_COLS = 2 * D;
    static_assert(TWN % 1024 == 0 && TF + 64 * kLd * 2 >= TWN + 16384, "T_w / N_b tile");
    static_assert(3 * (BYTES + 1024 + 1024) <= 233472, "three prep CTAs per SM");
};
enum { PS_G = 0, PS_GAM, PS_BETA, PS_RK, PS_RQ, PS_FTW, PS_CARRY, PS_COLF };
enum { PB_FULL = 0, PB_TMEM, PB_M1, PB_RA1, PB_M3, PB_FIN, PB_COUNT };

struct PrepParams {
    const float* alpha;
    const float* beta;
    const int2* map;            // varlen: (first token, valid tokens) per record; nullptr if dense
    int num_seqs, T, H;
    int nchunk_dense;           // dense: chunks per sequence
    int ntask;                  // CTAs of the grid: chunk records x heads
    int ahead;                  // CTA index distance of the L2 prefetch (two CTAs per SM)
    float scale;
    int l2norm;
    uint8_t* ws_w;
    uint8_t* ws_p;
    uint8_t* ws_u;
    float* ws_s;
    int* status;
    long long ab_elems;
};

constexpr int kPrepThreads = 320;  // warp 0 loads, warp 1 TMEM + tensor cores, 2..9 compute

// Two CTAs share an SM (registers and TMEM allow two).  The TMEM allocation is made by warp 1
// alone; everything that needs no TMEM (the input copies, decay and norms) runs before it is
// awaited, so a CTA that must wait for columns still gets its inputs in.
template <int D>
__global__ void __launch_bounds__(kPrepThreads, 2)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const PrepParams p) {
    using L = PrepLayout<D>;
    constexpr int KB = L::KB;
    const int bid = blockIdx.x;
    const int h = bid % p.H;
    const int g = bid / p.H;
    long base;
    int nvalid;
    if (p.map) {
        const int2 m = p.map[g];
        if (m.y <= 0) return;  // grid sized for the worst case
        base = m.x;
        nvalid = m.y;
    } else {
        const int n = g / p.nchunk_dense, c = g % p.nchunk_dense;
        base = (long)n * p.T + (long)c * kChunk;
        nvalid = min(kChunk, p.T - c * kChunk);
    }
    const size_t rec = (size_t)g * p.H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* never = reinterpret_cast<volatile int*>(sm + L::MISC + 8);
    if (tid == 0) {
        mbar_init(&bars[PB_FULL], 32);
        for (int b = PB_TMEM; b < PB_COUNT; ++b) mbar_init(&bars[b], 1);
        *abort_flag = 0;
        *never = 0;
        fence_mbar_init();
    }
    __syncthreads();

#define GUARD(cond, code, detail) GDN_GUARD(cond, p.status, code, detail)
    auto fail = [&](int bar) {
        (void)GUARD(false, DBG_WAIT, (long)bar * 65536 + g);
        *abort_flag = 1;
        record_status(p.status, GDN_ERR_TIMEOUT);
    };
    auto wwait = [&](int bar, uint32_t parity) {
        const bool ok = mbar_wait_warp(&bars[bar], parity, abort_flag);
        if (!ok && lane == 0) fail(bar);
        return ok;
    };
    auto scal = [&](int which) { return reinterpret_cast<float*>(sm + L::SC + which * 256); };

    if (warp == 0) {
        // ---------------------------------------------------------------- loads
        // the tile copies first (lane 0's arrival carries the byte count), then alpha and beta;
        // the other 31 arrivals follow the alpha / beta stores of all lanes
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars[PB_FULL], L::TX);
            const int z = (int)base;
#pragma unroll
            for (int b = 0; b < KB; ++b) {
                tma_load_3d(sm + L::KQ + b * 16384, &tm_k, 64 * b, h, z, &bars[PB_FULL]);
                tma_load_3d(sm + L::KQ + b * 16384 + 8192, &tm_q, 64 * b, h, z, &bars[PB_FULL]);
                tma_load_3d(sm + L::V + b * 8192, &tm_v, 64 * b, h, z, &bars[PB_FULL]);
            }
        }
        float* ab = reinterpret_cast<float*>(sm + L::AB);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = lane + 32 * u;
            const long t = base + i;
            const bool ok = i < nvalid && GUARD(t * p.H + h < p.ab_elems, DBG_GLOBAL_OOB, 1);
            ab[i] = ok ? p.alpha[t * p.H + h] : 1.f;
            ab[64 + i] = ok ? p.beta[t * p.H + h] : 0.f;
        }
        __syncwarp();
        if (lane != 0) mbar_arrive(&bars[PB_FULL]);
        // Warm L2 with the tiles of the CTA that will most likely run next on this SM (CTAs are
        // dispatched in index order as slots free up), so that its loads do not wait on DRAM.
        const int nt = bid + p.ahead;
        if (lane == 0 && nt < p.ntask) {
            const int g2 = nt / p.H, h2 = nt % p.H;
            int z2 = -1;
            if (p.map) {
                const int2 m = p.map[g2];
                if (m.y > 0) z2 = m.x;
            } else {
                z2 = (g2 / p.nchunk_dense) * p.T + (g2 % p.nchunk_dense) * kChunk;
            }
            if (z2 >= 0) {
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    tma_prefetch_3d(&tm_k, 64 * b, h2, z2);
                    tma_prefetch_3d(&tm_q, 64 * b, h2, z2);
                    tma_prefetch_3d(&tm_v, 64 * b, h2, z2);
                }
            }
        }
        // do not leave while the copies are still writing shared memory
        mbar_wait_warp(&bars[PB_FULL], 0, never, 100000000ull);
    } else if (warp == 1) {
        // ---------------------------------------------------------------- TMEM and tensor cores
        tmem_alloc(tmem_slot, L::T_COLS);  // may wait for another CTA on this SM to free TMEM
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[PB_TMEM]);
        tc_fence_after();
        const uint32_t tmem = *tmem_slot;
        if (lane == 0) {
            constexpr uint32_t ID_M1 = idesc_bf16(128, 64, false, false);
            constexpr uint32_t ID_N = idesc_bf16(128, D, false, true);
            const uint32_t s0 = smem_u32(sm);
            const uint64_t dKQ = sdesc(s0 + L::KQ, 16, 1024);           // [K;Q] rows, K-major
            const uint64_t dKb = sdesc(s0 + L::KQ, 16384, 1024);        // K as MN-major B
            const uint64_t dVb = sdesc(s0 + L::V, 8192, 1024);          // V as MN-major B
            const uint64_t dTWN = sdesc(s0 + L::TWN, 16, 1024);         // [T_w; N_b], K-major
            constexpr uint64_t KS = 32 >> 4, MS = 2048 >> 4, BLK = 16384 >> 4;
            bool ok = mbar_wait(&bars[PB_FULL], 0, abort_flag);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int b = 0; b < KB; ++b)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a = dKQ + b * BLK + kk * KS;
                        mma_bf16(tmem + L::T_D1, a, a, ID_M1, (b | kk) != 0);
                    }
                mma_commit(&bars[PB_M1]);
                ok = mbar_wait(&bars[PB_RA1], 0, abort_flag);
            }
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_D3, dTWN + kk * KS, dKb + kk * MS, ID_N, kk != 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_DU, dTWN + kk * KS, dVb + kk * MS, ID_N, kk != 0);
                mma_commit(&bars[PB_M3]);
            }
            if (!ok && !*abort_flag) fail(PB_COUNT);
            // no MMA may still be writing TMEM or arriving on a barrier when the CTA ends
            mma_commit(&bars[PB_FIN]);
            mbar_wait(&bars[PB_FIN], 0, never, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- prep warps
        // Warps 2..9: two per TMEM lane quadrant.  t is the TMEM lane (the row of the 128-row
        // accumulators); hf selects the half of the columns this warp handles.
        const int t = ((warp & 3) << 5) | lane;
        const int wa = t >> 5;
        const int hf = (warp - 2) >> 2;
        const uint32_t lane_base = static_cast<uint32_t>(wa * 32) << 16;
        __nv_bfloat16* AF = reinterpret_cast<__nv_bfloat16*>(sm + L::AF);
        __nv_bfloat16* TF = reinterpret_cast<__nv_bfloat16*>(sm + L::TF);
        __nv_bfloat16* XB = reinterpret_cast<__nv_bfloat16*>(sm + L::XB) + wa * 16 * 24;
        const float* ab = reinterpret_cast<const float*>(sm + L::AB);
        float* sG = scal(PS_G);
        float* sGam = scal(PS_GAM);
        float* sBeta = scal(PS_BETA);
        float* sRk = scal(PS_RK);
        float* sRq = scal(PS_RQ);
        float* sFtw = scal(PS_FTW);
        float* sCarry = scal(PS_CARRY);
        float* sColf = scal(PS_COLF);
        float* rs = p.ws_s + rec * (kRecS / 4);

        // (1) decay and norms
        bool ok = wwait(PB_FULL, 0);
        if (ok && hf == 0) {
            if (t < 64) {
                float gl = lg2(ab[t]);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float x = __shfl_up_sync(0xffffffffu, gl, o);
                    if (lane >= o) gl += x;
                }
                if (t == 31) sCarry[0] = gl;
                float ss = 0.f;
#pragma unroll
                for (int b = 0; b < KB; ++b) ss += row_sumsq(sm + L::KQ + b * 16384, t);
                sRk[t] = p.l2norm ? 1.0f / sqrtf(ss + kNormEps) : 1.0f;
                sBeta[t] = ab[64 + t];
                sG[t] = gl;
            } else {
                const int r = t - 64;
                float ss = 0.f;
#pragma unroll
                for (int b = 0; b < KB; ++b) ss += row_sumsq(sm + L::KQ + b * 16384 + 8192, r);
                sRq[r] = p.l2norm ? 1.0f / sqrtf(ss + kNormEps) : 1.0f;
            }
        }
        named_sync(1, 256);
        if (ok && hf == 0 && t >= 32 && t < 64) sG[t] += sCarry[0];
        named_sync(1, 256);
        const float Glast = sG[nvalid - 1];
        if (ok && hf == 0) {
            if (t < 64) {
                const float G = sG[t], gam = ex2(G);
                sGam[t] = gam;
                sColf[t] = ex2(sG[t | 15] - G);  // decay from token t to the end of its 16-block
                sFtw[t] = sBeta[t] * gam * sRk[t];
                rs[t] = (t < nvalid) ? ex2(Glast - G) * sRk[t] : 0.f;
                if (t == 0) rs[128] = ex2(Glast);
            } else {
                const int r = t - 64;
                rs[64 + r] = p.scale * ex2(sG[r]) * sRq[r];
            }
        }
        named_sync(1, 256);

        // (2) A (rows 0-63 of M1, to shared memory) and P (rows 64-127, to the workspace)
        ok = wwait(PB_TMEM, 0) && ok;
        tc_fence_after();
        const uint32_t tmem = *tmem_slot;
        ok = wwait(PB_M1, 0) && ok;
        tc_fence_after();
        // Gam_ij = 2^(G_i - G_j) for j <= i.  Within the row's own 16-token block it is computed
        // directly; for an earlier block b it is the product 2^(G_i - G_e) 2^(G_e - G_j) through
        // the block's last token e = 16 b + 15.  Both exponents are <= 0 (G does not increase),
        // so neither factor can overflow, and a row needs 20 exponentials instead of 64.
        if (ok) {
            const int i = t & 63, blk = i >> 4;
            const bool arow = t < 64;  // rows of A (strictly lower) or of P (lower, diagonal incl.)
            const float Gi = sG[i];
            const float sc = arow ? sBeta[i] * sRk[i] : p.scale * sRq[i];
            // this warp's columns: blocks 2 hf and 2 hf + 1; the row's own block is among them
            // when blk / 2 == hf (the same for the whole warp)
            float rf[2], dg[16];
#pragma unroll
            for (int k = 0; k < 2; ++k) rf[k] = ex2(Gi - sG[16 * (2 * hf + k) + 15]);
            if ((blk >> 1) == hf) {
#pragma unroll
                for (int u = 0; u < 16; ++u) dg[u] = ex2(Gi - sG[16 * blk + u]);
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) dg[u] = 0.f;
            }
            const int lim = arow ? i : i + 1;  // columns j < lim are kept
            uint8_t* P = p.ws_p + rec * kRecP;
            float d[32];
            tmem_ld32(tmem + L::T_D1 + lane_base + hf * 32, d);
#pragma unroll
            for (int j4 = 0; j4 < 32; j4 += 4) {
                const int j = hf * 32 + j4, cb = j >> 4;
                const float4 rk4 = *reinterpret_cast<const float4*>(sRk + j);
                const float4 cf4 = *reinterpret_cast<const float4*>(sColf + j);
                const float rk[4] = {rk4.x, rk4.y, rk4.z, rk4.w};
                const float cf[4] = {cf4.x, cf4.y, cf4.z, cf4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float f = (cb < blk) ? rf[j4 >> 4] * cf[u] : dg[(j4 & 15) + u];
                    d[j4 + u] = (j + u < lim) ? sc * rk[u] * d[j4 + u] * f : 0.f;
                }
            }
            if (arow) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(AF + i * kLd + hf * 32 + 8 * q) =
                        (q & 1) ? pack8_fma(d + 8 * q) : pack8(d + 8 * q);
            } else {
                store_half_row_mixed(P, i, hf * 4, d);
            }
        }
        named_sync(1, 256);

        // (3) T = (I + A)^-1.  16x16 diagonal blocks by forward substitution (fp32), then the
        // off-diagonal blocks T_ij = -D_i sum_m A_im T_mj by diagonals on mma.sync.
        if (ok && hf == 0 && t < 64) {
            const int b = t >> 4, l = t & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float arow[16];
                const __nv_bfloat16* src = AF + (16 * b + r) * kLd + 16 * b;
                unpack8(*reinterpret_cast<const uint4*>(src), arow);
                unpack8(*reinterpret_cast<const uint4*>(src + 8), arow + 8);
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                for (int m = 0; m < r; m += 2) {
                    acc0 = fmaf(arow[m], x[m], acc0);
                    if (m + 1 < r) acc1 = fmaf(arow[m + 1], x[m + 1], acc1);
                }
                x[r] = (r < l) ? 0.f : (r == l ? 1.f : -(acc0 + acc1));
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) TF[(16 * b + r) * kLd + 16 * b + l] = __float2bfloat16_rn(x[r]);
        }
        named_sync(1, 256);
        {
            const int mrow = (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix row of this lane
            const int mcol = (lane >> 4) * 8;                      // ldmatrix column offset
            const int gid = lane >> 2, tig = lane & 3;
            for (int dd = 1; dd < 4; ++dd) {
                if (ok && hf == 0 && wa < 4 - dd) {
                    const int bi = wa + dd, bj = wa;
                    float cx[2][4] = {};
                    for (int m = bj; m < bi; ++m) {
                        uint32_t a[4], b0, b1, b2, b3;
                        ldsm_x4(smem_u32(AF + (16 * bi + mrow) * kLd + 16 * m + mcol), a[0], a[1], a[2], a[3]);
                        ldsm_x4_t(smem_u32(TF + (16 * m + mrow) * kLd + 16 * bj + mcol), b0, b1, b2, b3);
                        mma16816(cx[0], a, b0, b1);
                        mma16816(cx[1], a, b2, b3);
                    }
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        *reinterpret_cast<uint32_t*>(XB + gid * 24 + 8 * nt + 2 * tig) = pack_bf16(cx[nt][0], cx[nt][1]);
                        *reinterpret_cast<uint32_t*>(XB + (gid + 8) * 24 + 8 * nt + 2 * tig) = pack_bf16(cx[nt][2], cx[nt][3]);
                    }
                    __syncwarp();
                    uint32_t a[4], b0, b1, b2, b3;
                    ldsm_x4(smem_u32(TF + (16 * bi + mrow) * kLd + 16 * bi + mcol), a[0], a[1], a[2], a[3]);
                    ldsm_x4_t(smem_u32(XB + mrow * 24 + mcol), b0, b1, b2, b3);
                    float ct[2][4] = {};
                    mma16816(ct[0], a, b0, b1);
                    mma16816(ct[1], a, b2, b3);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        *reinterpret_cast<uint32_t*>(TF + (16 * bi + gid) * kLd + 16 * bj + 8 * nt + 2 * tig) =
                            pack_bf16(-ct[nt][0], -ct[nt][1]);
                        *reinterpret_cast<uint32_t*>(TF + (16 * bi + gid + 8) * kLd + 16 * bj + 8 * nt + 2 * tig) =
                            pack_bf16(-ct[nt][2], -ct[nt][3]);
                    }
                    __syncwarp();
                }
                named_sync(1, 256);
            }
        }

        // (4) T_w = T diag(beta gamma rk) -> rows 0-63;  N_b = strict(T) diag(beta) -> rows 64-127.
        // The tile overlays A and T, so every thread first takes its T row into registers.
        {
            const int i = t & 63;
            uint4 tr[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) tr[q] = *reinterpret_cast<const uint4*>(TF + i * kLd + hf * 32 + 8 * q);
            named_sync(1, 256);
            if (ok) {
                float x[32];
#pragma unroll
                for (int q = 0; q < 4; ++q) unpack8(tr[q], x + 8 * q);
#pragma unroll
                for (int j4 = 0; j4 < 32; j4 += 4) {
                    const int j = hf * 32 + j4;
                    if (t < 64) {
                        const float4 f4 = *reinterpret_cast<const float4*>(sFtw + j);
                        x[j4 + 0] = (j + 0 <= i) ? x[j4 + 0] * f4.x : 0.f;
                        x[j4 + 1] = (j + 1 <= i) ? x[j4 + 1] * f4.y : 0.f;
                        x[j4 + 2] = (j + 2 <= i) ? x[j4 + 2] * f4.z : 0.f;
                        x[j4 + 3] = (j + 3 <= i) ? x[j4 + 3] * f4.w : 0.f;
                    } else {
                        const float4 b4 = *reinterpret_cast<const float4*>(sBeta + j);
                        x[j4 + 0] = (j + 0 < i) ? x[j4 + 0] * b4.x : 0.f;
                        x[j4 + 1] = (j + 1 < i) ? x[j4 + 1] * b4.y : 0.f;
                        x[j4 + 2] = (j + 2 < i) ? x[j4 + 2] * b4.z : 0.f;
                        x[j4 + 3] = (j + 3 < i) ? x[j4 + 3] * b4.w : 0.f;
                    }
                }
                store_half_row_mixed(sm + L::TWN, t, hf * 4, x);
            }
        }
        fence_proxy_async_smem();
        named_sync(1, 256);
        if (t == 0 && hf == 0) mbar_arrive(&bars[PB_RA1]);

        // (5) -W (lanes 0-63 of the W accumulator) and Ut = beta V + N_b V (lanes 64-127), built
        // as the record's byte images in shared memory that the products no longer read (-W over
        // the T_w / N_b tile, Ut over K and Q), then written out by two bulk copies
        ok = wwait(PB_M3, 0) && ok;
        tc_fence_after();
        static_assert(L::KB * 16384 >= D * 256 && 16384 >= D * 128, "staging space");
        if (ok) {
            if (t < 64) {
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    float w[32];
                    tmem_ld32(tmem + L::T_D3 + lane_base + 64 * b + 32 * hf, w);
#pragma unroll
                    for (int j = 0; j < 32; ++j) w[j] = -w[j];
                    store_half_row_mixed(sm + L::TWN + b * 8192, t, hf * 4, w);
                }
            } else {
                const int i = t - 64;
                const bool valid = i < nvalid;
                const float bi = sBeta[i];
                uint8_t* urec = sm + L::KQ + (size_t)i * 256;
#pragma unroll
                for (int s = 0; s < KB; ++s) {
                    float d[32], vv[32];
                    tmem_ld32(tmem + L::T_DU + lane_base + 64 * s + 32 * hf, d);
                    load_half_row(sm + L::V + s * 8192, i, hf * 4, vv);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 u;
                        u.x = valid ? fmaf(bi, vv[4 * q + 0], d[4 * q + 0]) : 0.f;
                        u.y = valid ? fmaf(bi, vv[4 * q + 1], d[4 * q + 1]) : 0.f;
                        u.z = valid ? fmaf(bi, vv[4 * q + 2], d[4 * q + 2]) : 0.f;
                        u.w = valid ? fmaf(bi, vv[4 * q + 3], d[4 * q + 3]) : 0.f;
                        const int ch = hf * 8 + q;
                        *reinterpret_cast<float4*>(urec + s * 16384 + ((ch ^ (i & 7)) << 4)) = u;
                    }
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_sync(1, 256);
        if (ok && t == 0 && hf == 0) {
            bulk_store(p.ws_w + rec * (size_t)(D * 128), sm + L::TWN, D * 128);
            bulk_store(p.ws_u + rec * (size_t)(D * 256), sm + L::KQ, D * 256);
            bulk_commit();
            bulk_wait_read();  // the CTA's shared memory must outlive the copies' reads
        }
    }
#undef GUARD
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(*tmem_slot, L::T_COLS);
    }
}

// ============================================================================ chain kernel
template <int D>
struct ChainLayout {
    static constexpr int KB = D / 64;
    static constexpr int KQW_BLOCK = 192 * 128;   // per dk block: K rows 0-63, Q 64-127, -W 128-191
    static constexpr int KQW = KB * KQW_BLOCK;
    static constexpr int P = KQW;                 // P, 64 rows (read as 128 rows: then U)
    static constexpr int U = P + 8192;            // Ut image of the 64-column slice: fp32, 64 x 256 B
    static constexpr int SC = U + 16384;          // record scalars
    static constexpr int STAGE = SC + 1024;
    // The CTA's 32 state columns use the first half of 64-column operand tiles; an N = 64 MMA
    // costs the tensor core what an N = 32 one does.
    static constexpr int SB = 2 * STAGE;          // S in bf16: D rows x 64 columns (0-31 used)
    static constexpr int UHL = SB + D * 128;      // [U'_hi (columns 0-31) | U'_lo (32-63)], 64 rows
    static constexpr int UB = UHL + 8192;         // U in bf16, 64 rows (columns 0-31 used)
    static constexpr int BAR = UB + 8192;
    static constexpr int MISC = BAR + 16 * 8;     // tmem base, abort flag, zero word, 2 counters
    static constexpr int BYTES = MISC + 32;
    static constexpr int TX = KB * 16384 + KB * 8192 + 8192 + 16384 + 1024;
    static constexpr uint32_t T_S = 0;            // [K^T U'_hi | K^T U'_lo] of the chunk, 64 columns
    static constexpr uint32_t T_D4 = 64;          // [Q S ; -W S], 2 x 64 columns (0-31 used)
    static constexpr uint32_t T_D6 = 192;         // P U, 2 x 64 columns (0-31 used)
    static constexpr uint32_t T_COLS = 512;
    static_assert(STAGE % 1024 == 0, "stage tiles stay 1024-byte aligned");
    static_assert(BYTES + 1024 <= 232448 - 1024, "shared memory budget");
};
enum {
    CB_FULL0 = 0, CB_FULL1, CB_EMPTY0, CB_EMPTY1,  // input ring
    CB_M4, CB_M5, CB_M6_0, CB_M6_1,                // tensor-core completions
    CB_COUNT
};

struct ChainParams {
    const float* s0;
    __nv_bfloat16* y;
    float* s_final;
    const int32_t* cu_seqlens;
    const int32_t* cb;
    int num_seqs, T, H, DV;
    int nchunk_dense, nrec_chunks;
    const uint8_t* ws_w;
    const uint8_t* ws_p;
    const uint8_t* ws_u;
    const float* ws_s;
    int* status;
    long long y_elems, state_elems;
};

constexpr int kChainThreads = 384;

// Warp roles: 0 loads (TMA for K and Q, bulk copies for the workspace record), 1 owns the TMEM
// allocation and issues the output product, 4..11 are the epilogue warps.  Epilogue warp w reads
// TMEM lanes 32 (w % 4) .. +31 and columns 16 ((w - 4) / 4) .. +15 of the CTA's 32; lanes 0-63
// carry the output rows (Y) and lanes 64-127 the pseudo-value rows (U); all eight hold a
// 16-column strip of S.  There is no separate MMA warp:
// the last epilogue warp to finish a step (found with a shared-memory arrival counter) issues the
// tensor-core products that depend on it, which saves a wake-up on the sequential path.
template <int D>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const ChainParams p) {
    using L = ChainLayout<D>;
    constexpr int KB = L::KB;
    const int nsl = p.DV / kNV;
    const int bid = blockIdx.x;
    const int jsl = bid % nsl;
    const int h = (bid / nsl) % p.H;
    const int n = bid / (nsl * p.H);
    long t0, t1;
    int cbase;
    if (p.cu_seqlens) {
        t0 = p.cu_seqlens[n];
        t1 = p.cu_seqlens[n + 1];
        cbase = p.cb[n];
    } else {
        t0 = (long)n * p.T;
        t1 = t0 + p.T;
        cbase = n * p.nchunk_dense;
    }
    const int len = (int)(t1 - t0);
    int nch = len > 0 ? (len + kChunk - 1) / kChunk : 0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t soff = ((size_t)n * p.H + h) * (size_t)D * p.DV + (size_t)jsl * kNV;

#define GUARD(cond, code, detail) GDN_GUARD(cond, p.status, code, detail)
    if (nch > 0 && (cbase < 0 || cbase + nch > p.nrec_chunks)) {  // inconsistent cu_seqlens
        if (tid == 0) record_status(p.status, GDN_ERR_INVALID_ARG);
        nch = 0;
    }
    if (nch == 0) {  // empty document: the final state is the initial one
        if (p.s_final)
            for (int e = tid; e < D * kNV; e += kChainThreads) {
                const int r = e / kNV, cc = e % kNV;
                const size_t o = soff + (size_t)r * p.DV + cc;
                if (GUARD((long long)o < p.state_elems, DBG_GLOBAL_OOB, 5))
                    p.s_final[o] = p.s0 ? p.s0[o] : 0.f;
            }
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* never = reinterpret_cast<volatile int*>(sm + L::MISC + 8);
    int* arrivals = reinterpret_cast<int*>(sm + L::MISC + 16);  // (A) and (B) completions
    if (tid == 0) {
        mbar_init(&bars[CB_FULL0], 1);
        mbar_init(&bars[CB_FULL1], 1);
        mbar_init(&bars[CB_EMPTY0], 5);  // MMA commit + 4 output warps
        mbar_init(&bars[CB_EMPTY1], 5);
        for (int b = CB_M4; b < CB_COUNT; ++b) mbar_init(&bars[b], 1);
        *abort_flag = 0;
        *never = 0;
        arrivals[0] = 0;
        arrivals[1] = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, L::T_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto fail = [&](int bar, int c) {
        (void)GUARD(false, DBG_WAIT, (long)bar * 65536 + c);
        *abort_flag = 1;
        record_status(p.status, GDN_ERR_TIMEOUT);
    };
    auto wwait = [&](int bar, uint32_t parity, int c) {
        const bool ok = mbar_spin_warp(&bars[bar], parity, abort_flag);
        if (!ok && lane == 0) fail(bar, c);
        return ok;
    };
    constexpr uint32_t kRecW = D * 128, kRecU = D * 256;

    if (warp == 0) {
        // ---------------------------------------------------------------- loads
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            int issued = 0;
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1;
                if (!mbar_wait(&bars[CB_EMPTY0 + s], ((c >> 1) & 1) ^ 1, abort_flag)) {
                    if (!*abort_flag) fail(CB_EMPTY0 + s, c);
                    break;
                }
                uint8_t* st = sm + s * L::STAGE;
                const size_t rec = (size_t)(cbase + c) * p.H + h;
                uint64_t* full = &bars[CB_FULL0 + s];
                mbar_arrive_expect_tx(full, L::TX);
                const int z = (int)(t0 + (long)c * kChunk);
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    tma_load_3d(st + b * L::KQW_BLOCK, &tm_k, 64 * b, h, z, full);
                    tma_load_3d(st + b * L::KQW_BLOCK + 8192, &tm_q, 64 * b, h, z, full);
                    bulk_load(st + b * L::KQW_BLOCK + 16384, p.ws_w + rec * kRecW + b * 8192, 8192, full);
                }
                bulk_load(st + L::P, p.ws_p + rec * kRecP, kRecP, full);
                bulk_load(st + L::U, p.ws_u + rec * kRecU + (size_t)(jsl >> 1) * 16384, 16384, full);
                bulk_load(st + L::SC, p.ws_s + rec * (kRecS / 4), kRecS, full);
                if (c + 2 < nch) {  // warm L2 for the chunk that will reuse this stage
                    const size_t rec2 = rec + 2 * (size_t)p.H;
#pragma unroll
                    for (int b = 0; b < KB; ++b) {
                        tma_prefetch_3d(&tm_k, 64 * b, h, z + 2 * kChunk);
                        tma_prefetch_3d(&tm_q, 64 * b, h, z + 2 * kChunk);
                    }
                    bulk_prefetch_l2(p.ws_w + rec2 * kRecW, kRecW);
                    bulk_prefetch_l2(p.ws_p + rec2 * kRecP, kRecP);
                    bulk_prefetch_l2(p.ws_u + rec2 * kRecU + (size_t)(jsl >> 1) * 16384, 16384);
                    bulk_prefetch_l2(p.ws_s + rec2 * (kRecS / 4), kRecS);
                }
                ++issued;
            }
            // Tail of the ring: do not exit while a copy or a commit-arrive on this CTA's shared
            // memory is still pending.
            for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c) {
                mbar_wait(&bars[CB_FULL0 + (c & 1)], (c >> 1) & 1, never, 100000000ull);
                mbar_wait(&bars[CB_EMPTY0 + (c & 1)], (c >> 1) & 1, abort_flag);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- output product M6
        if (lane == 0) {
            constexpr uint32_t ID_KN = idesc_bf16(128, 64, false, true);  // U_bf16 tile is 64 wide
            constexpr uint64_t KS = 32 >> 4, MS = 2048 >> 4;
            const uint64_t dUB = sdesc(smem_u32(sm + L::UB), 8192, 1024);
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1;
                // U_bf16 of chunk c is complete once M5(c) is (M5 is issued after it is written)
                if (!mbar_wait(&bars[CB_M5], c & 1, abort_flag)) {
                    if (!*abort_flag) fail(CB_M5, c);
                    break;
                }
                tc_fence_after();
                const uint64_t dP = sdesc(smem_u32(sm + s * L::STAGE + L::P), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_D6 + s * 64, dP + kk * KS, dUB + kk * MS, ID_KN, kk != 0);
                mma_commit(&bars[CB_M6_0 + s]);
                mma_commit(&bars[CB_EMPTY0 + s]);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- epilogue warps
        const int qd = warp & 3, hf = (warp - 4) >> 2;
        const int srow = qd * 32 + lane;               // TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
        const uint32_t col = 16 * hf;
        const bool uwarp = qd >= 2;                    // U rows; the others write Y
        float S[16];
        {
            // D = 64: lanes 64-127 of the state product mirror rows 0-63
            const size_t o = soff + (size_t)(srow % D) * p.DV + col;
            const bool in = p.s0 && GUARD((long long)(o + 16) <= p.state_elems, DBG_GLOBAL_OOB, 2);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = in ? *reinterpret_cast<const float4*>(p.s0 + o + 4 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
                S[4 * q] = v.x; S[4 * q + 1] = v.y; S[4 * q + 2] = v.z; S[4 * q + 3] = v.w;
            }
            // the unused halves of the operand tiles feed only unused accumulator columns;
            // zero them once so that they hold finite values
            const uint4 z = make_uint4(0, 0, 0, 0);
            for (int e = tid - 128; e < (D * 128 + 16384) / 16; e += 256)
                reinterpret_cast<uint4*>(sm + L::SB)[e] = z;
            fence_proxy_async_smem();
            named_sync(1, 256);
        }
        float gprev = 1.f;
        bool ok = true;

        constexpr uint32_t ID_KN = idesc_bf16(128, 64, false, true);
        constexpr uint32_t ID_M5 = idesc_bf16(128, 64, true, true);  // B = [U'_hi | U'_lo]
        constexpr uint64_t KS = 32 >> 4, MS = 2048 >> 4, BLK = L::KQW_BLOCK >> 4;
        static_assert(L::SB + D * 128 + 16384 == L::UB + 8192, "tiles zeroed at start");
        // M4: [Q; -W] S_bf16  ->  Q S (lanes 0-63), -W S (lanes 64-127)
        auto issue_m4 = [&](int c) {
            const int s = c & 1;
            const uint64_t dQW = sdesc(smem_u32(sm + s * L::STAGE + 8192), 16, 1024);
            const uint64_t dSB = sdesc(smem_u32(sm + L::SB), D * 128, 1024);
            const uint32_t d4 = tmem + L::T_D4 + s * 64;
#pragma unroll
            for (int b = 0; b < KB; ++b)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(d4, dQW + b * BLK + kk * KS, dSB + (b * 4 + kk) * MS, ID_KN, (b | kk) != 0);
            mma_commit(&bars[CB_M4]);
        };
        // M5: K^T [U'_hi | U'_lo] (U' = diag(Gam_C,. rk) U in two bf16 terms, side by side in one
        // 64-column tile).  The output product M6 is issued by warp 1 once M5 is done, so that it
        // does not delay M5's completion.
        auto issue_m56 = [&](int c) {
            const int s = c & 1;
            const uint64_t dKt = sdesc(smem_u32(sm + s * L::STAGE), D == 128 ? L::KQW_BLOCK : 0, 1024);
            const uint64_t dUHL = sdesc(smem_u32(sm + L::UHL), 8192, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + L::T_S, dKt + kk * MS, dUHL + kk * MS, ID_M5, kk != 0);
            mma_commit(&bars[CB_M5]);
        };
        // Arrival of this warp at the end of a step; the last of `n` arrivals for chunk c issues
        // the dependent products.  The warp's shared-memory and TMEM accesses are ordered before
        // the counter update (proxy and tcgen05 fences, then a CTA-scope fence), and the issuing
        // thread orders the counter read before its tcgen05 operations the same way.
        auto arrive = [&](int which, int n, int c) {
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                const int old = atomicAdd(arrivals + which, 1);
                if (old == n * c + n - 1) {
                    __threadfence_block();
                    tc_fence_after();
                    if (which == 0) issue_m4(c); else issue_m56(c);
                }
            }
            __syncwarp();
        };

        auto y_epilogue = [&](int cy) {
            const int s = cy & 1;
            ok = wwait(CB_M6_0 + s, (cy >> 1) & 1, cy) && ok;
            tc_fence_after();
            if (ok) {
                const uint8_t* st = sm + s * L::STAGE;
                const int nv = min(kChunk, len - cy * kChunk);
                float a[16], b[16];
                tmem_ld16x2(tmem + L::T_D4 + s * 64 + lane_base + col, tmem + L::T_D6 + s * 64 + lane_base + col, a, b);
                const float ys = reinterpret_cast<const float*>(st + L::SC)[64 + srow];
                const size_t yoff = ((size_t)(t0 + (long)cy * kChunk + srow) * p.H + h) * p.DV + jsl * kNV + col;
                if (srow < nv && GUARD((long long)(yoff + 16) <= p.y_elems, DBG_GLOBAL_OOB, 3)) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) a[j] = fmaf(ys, a[j], b[j]);
                    uint4* dst = reinterpret_cast<uint4*>(p.y + yoff);
#pragma unroll
                    for (int q = 0; q < 2; ++q) dst[q] = pack8(a + 8 * q);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CB_EMPTY0 + s]);
        };

        for (int c = 0; c < nch; ++c) {
            const int s = c & 1;
            const uint8_t* st = sm + s * L::STAGE;
            // (A) S_c = gamma_C S_{c-1} + K^T U'  ->  bf16 operand rows
            ok = wwait(CB_FULL0 + s, (c >> 1) & 1, c) && ok;
            if (c >= 1) {
                ok = wwait(CB_M5, (c - 1) & 1, c) && ok;
                tc_fence_after();
                if (ok) {
                    float d[16], e[16];
                    tmem_ld16x2(tmem + L::T_S + lane_base + col, tmem + L::T_S + lane_base + 32 + col, d, e);
#pragma unroll
                    for (int j = 0; j < 16; ++j) S[j] = fmaf(gprev, S[j], d[j] + e[j]);
                }
            }
            if (ok && srow < D) {
                *reinterpret_cast<uint4*>(sm + L::SB + swz(srow, 2 * hf)) = pack8(S);
                *reinterpret_cast<uint4*>(sm + L::SB + swz(srow, 2 * hf + 1)) = pack8_fma(S + 8);
            }
            gprev = reinterpret_cast<const float*>(st + L::SC)[128];
            // M4 of this chunk may overwrite the output accumulators of chunk c - 2: the output
            // warps read them in iteration c - 1, before this arrival
            arrive(0, 8, c);

            if (uwarp) {
                // (B) U = Ut + (-W S) -> U'_hi, U'_lo (scaled for the state update), U_bf16.
                // M6 of the previous chunk (issued by another thread, so not covered by this
                // chunk's M4 commit) must have finished reading U_bf16.
                ok = wwait(CB_M4, c & 1, c) && ok;
                if (c >= 1) ok = wwait(CB_M6_0 + ((c - 1) & 1), ((c - 1) >> 1) & 1, c) && ok;
                tc_fence_after();
                if (ok) {
                    const int i = srow - 64;
                    const float us = reinterpret_cast<const float*>(st + L::SC)[i];
                    float d[16];
                    tmem_ld16(tmem + L::T_D4 + s * 64 + lane_base + col, d);
                    const uint8_t* urow = st + L::U + i * 256;
                    const int ch0 = 8 * (jsl & 1) + 4 * hf;  // first 4-float chunk of these columns
                    uint32_t phi[8], plo[8], pub[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 ut = *reinterpret_cast<const float4*>(urow + (((ch0 + q) ^ (i & 7)) << 4));
                        const float u[4] = {ut.x + d[4 * q], ut.y + d[4 * q + 1], ut.z + d[4 * q + 2], ut.w + d[4 * q + 3]};
#pragma unroll
                        for (int e = 0; e < 4; e += 2) {
                            // U' = hi + lo with hi = U' truncated to bf16 and lo = the exact fp32
                            // rest, itself truncated: |U' - hi - lo| < 2^-14 |U'|.  Bit operations
                            // only, no conversion instructions.
                            const uint32_t b0 = __float_as_uint(u[e] * us), b1 = __float_as_uint(u[e + 1] * us);
                            const float l0 = __uint_as_float(b0) - __uint_as_float(b0 & 0xffff0000u);
                            const float l1 = __uint_as_float(b1) - __uint_as_float(b1 & 0xffff0000u);
                            phi[2 * q + e / 2] = __byte_perm(b0, b1, 0x7632);
                            plo[2 * q + e / 2] = __byte_perm(__float_as_uint(l0), __float_as_uint(l1), 0x7632);
                            pub[2 * q + e / 2] = pack_bf16(u[e], u[e + 1]);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint4 vh = make_uint4(phi[4 * q], phi[4 * q + 1], phi[4 * q + 2], phi[4 * q + 3]);
                        const uint4 vl = make_uint4(plo[4 * q], plo[4 * q + 1], plo[4 * q + 2], plo[4 * q + 3]);
                        const uint4 vb = make_uint4(pub[4 * q], pub[4 * q + 1], pub[4 * q + 2], pub[4 * q + 3]);
                        *reinterpret_cast<uint4*>(sm + L::UHL + swz(i, 2 * hf + q)) = vh;
                        *reinterpret_cast<uint4*>(sm + L::UHL + swz(i, 4 + 2 * hf + q)) = vl;
                        *reinterpret_cast<uint4*>(sm + L::UB + swz(i, 2 * hf + q)) = vb;
                    }
                }
                arrive(1, 4, c);
            } else if (c >= 1) {
                // (C) outputs of the previous chunk, while this chunk's M4 runs
                y_epilogue(c - 1);
            }
        }
        // the final state and the outputs of the last chunk
        ok = wwait(CB_M5, (nch - 1) & 1, nch) && ok;
        tc_fence_after();
        if (ok) {
            float d[16], e[16];
            tmem_ld16x2(tmem + L::T_S + lane_base + col, tmem + L::T_S + lane_base + 32 + col, d, e);
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(gprev, S[j], d[j] + e[j]);
            const size_t o = soff + (size_t)srow * p.DV + col;
            if (p.s_final && srow < D && GUARD((long long)(o + 16) <= p.state_elems, DBG_GLOBAL_OOB, 4)) {
                float4* dst = reinterpret_cast<float4*>(p.s_final + o);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_float4(S[4 * q], S[4 * q + 1], S[4 * q + 2], S[4 * q + 3]);
            }
        }
        if (!uwarp) y_epilogue(nch - 1);
        tc_fence_before();
    }
#undef GUARD
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        if (*abort_flag) {  // a wait gave up: let products already issued drain first
            const long long t = clock64();
            while (clock64() - t < 400000) {}
        }
        tc_fence_after();
        tmem_dealloc(tmem, L::T_COLS);
    }
}

// ---------------------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 3-D map over a [tokens, H, d] bf16 array: box = 64 (d) x 1 (head) x 64 (tokens), 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, long tokens, int H, int d) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of the [tokens, H, d] bf16 token tensors; nullptr arguments are skipped.
bool make_maps(const PrefillArgs& a, int D, CUtensorMap* mq, CUtensorMap* mk, CUtensorMap* mv) {
    const long tokens = a.cu_seqlens ? (long)a.T : (long)a.num_seqs * a.T;
    return (!mq || make_map(mq, a.q, tokens, a.H, D)) && (!mk || make_map(mk, a.k, tokens, a.H, D)) &&
           (!mv || make_map(mv, a.v, tokens, a.H, D));
}

// The state-independent phase: chunk map (packed documents) and the prep kernel.
template <int D>
cudaError_t launch_prep(const PrefillArgs& a, cudaStream_t st) {
    const bool varlen = a.cu_seqlens != nullptr;
    const long tokens = varlen ? (long)a.T : (long)a.num_seqs * a.T;
    const PrefillWorkspace w = prefill_workspace(a.num_seqs, a.T, a.H, D, varlen);
    if (a.ws == nullptr || a.ws_bytes < w.total) return cudaErrorInvalidValue;
    uint8_t* ws = static_cast<uint8_t*>(a.ws);
    int32_t* cb = reinterpret_cast<int32_t*>(ws + w.off_cb);
    int2* map = reinterpret_cast<int2*>(ws + w.off_map);
    CUtensorMap mq, mk, mv;
    if (!make_maps(a, D, &mq, &mk, &mv)) return cudaErrorInvalidValue;
    const int nchunk_dense = (a.T + kChunk - 1) / kChunk;
    cudaError_t e;
    if (varlen) {
        chunk_base_kernel<<<1, 1024, 0, st>>>(a.cu_seqlens, a.num_seqs, w.nrec_chunks, cb, map);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    int dev = 0, nsm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int ntask = w.nrec_chunks * a.H;
    PrepParams pp{a.alpha, a.beta, varlen ? map : nullptr, a.num_seqs, a.T, a.H,
                  nchunk_dense, ntask, 2 * nsm, a.scale, a.l2norm, ws + w.off_w, ws + w.off_p,
                  ws + w.off_u, reinterpret_cast<float*>(ws + w.off_s), a.status,
                  (long long)tokens * a.H};
    const int smem1 = PrepLayout<D>::BYTES + 1024;
    if ((e = cudaFuncSetAttribute(prep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem1)) != cudaSuccess)
        return e;
    prep_kernel<D><<<(unsigned)ntask, kPrepThreads, smem1, st>>>(mq, mk, mv, pp);
    return cudaGetLastError();
}

// The sequential phase: the chain kernel over the workspace records.
template <int D>
cudaError_t launch_chain(const PrefillArgs& a, cudaStream_t st) {
    const bool varlen = a.cu_seqlens != nullptr;
    const long tokens = varlen ? (long)a.T : (long)a.num_seqs * a.T;
    const PrefillWorkspace w = prefill_workspace(a.num_seqs, a.T, a.H, D, varlen);
    if (a.ws == nullptr || a.ws_bytes < w.total) return cudaErrorInvalidValue;
    uint8_t* ws = static_cast<uint8_t*>(a.ws);
    int32_t* cb = reinterpret_cast<int32_t*>(ws + w.off_cb);
    CUtensorMap mq, mk;
    if (!make_maps(a, D, &mq, &mk, nullptr)) return cudaErrorInvalidValue;
    const int nchunk_dense = (a.T + kChunk - 1) / kChunk;
    ChainParams cp{a.s0, static_cast<__nv_bfloat16*>(a.y), a.s_final, a.cu_seqlens,
                   varlen ? cb : nullptr, a.num_seqs, a.T, a.H, a.dv, nchunk_dense,
                   w.nrec_chunks, ws + w.off_w, ws + w.off_p, ws + w.off_u,
                   reinterpret_cast<const float*>(ws + w.off_s), a.status,
                   (long long)tokens * a.H * a.dv, (long long)a.num_seqs * a.H * a.dk * a.dv};
    const int smem2 = ChainLayout<D>::BYTES + 1024;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(chain_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem2)) != cudaSuccess)
        return e;
    const unsigned grid = (unsigned)a.num_seqs * a.H * (a.dv / kNV);
    chain_kernel<D><<<grid, kChainThreads, smem2, st>>>(mq, mk, cp);
    return cudaGetLastError();
}

}  // namespace

PrefillWorkspace prefill_workspace(int num_seqs, int T, int H, int d, bool varlen) {
    PrefillWorkspace w{};
    const long nrec = varlen ? ((long)T + 63L * num_seqs) / kChunk
                             : (long)num_seqs * ((T + kChunk - 1) / kChunk);
    w.nrec_chunks = (int)nrec;
    const size_t R = (size_t)nrec * H;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    size_t off = 0;
    w.off_cb = off;
    off += up(varlen ? ((size_t)num_seqs + 1) * 4 : 0);
    w.off_map = off;
    off += up(varlen ? (size_t)nrec * 8 : 0);
    w.off_w = off;
    off += up(R * (size_t)d * 128);
    w.off_p = off;
    off += up(R * kRecP);
    w.off_u = off;
    off += up(R * (size_t)d * 256);
    w.off_s = off;
    off += up(R * kRecS);
    w.total = off;
    return w;
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st) {
    // bf16 inputs run the tensor-core kernels; fp32 inputs the exact-fp32 token loop.
    if (a.dtype != GDN_BF16) return launch_prefill_seq(a, st);
    cudaError_t e = launch_prefill_phase(a, 0, st);
    return e != cudaSuccess ? e : launch_prefill_phase(a, 1, st);
}

cudaError_t launch_prefill_phase(const PrefillArgs& a, int phase, cudaStream_t st) {
    if (a.dtype != GDN_BF16) return cudaErrorInvalidValue;
    if (phase == 0) return a.dk == 128 ? launch_prep<128>(a, st) : launch_prep<64>(a, st);
    return a.dk == 128 ? launch_chain<128>(a, st) : launch_chain<64>(a, st);
}

}  // namespace gdn
