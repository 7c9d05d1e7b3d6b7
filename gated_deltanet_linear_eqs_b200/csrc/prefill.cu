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
//                 A and P, the 64x64 triangular inverse, W and Ut, and X = -W K_prev^T (the
//                 chunk's -W against the previous chunk's keys), written to a workspace record
//                 as ready-made tensor-core operand tiles
//   chain kernel  one CTA per (document, head, 32-column slice of dv) walks its chunks in order
//                 with the fp32 state in registers.  U_c = Ut_c - W_c S^c is formed from the
//                 state one chunk back plus X_c U'_{c-1}, so that the state update runs a chunk
//                 behind the pseudo-value recursion instead of inside it.
// Only the chain kernel is sequential, and it does the state-dependent work alone.
//
// Workspace record of (chunk record g, head h), r = g * H + h:
//   W  [r][dk/64][64 tokens][128 B]  -W, bf16, 128-byte swizzled rows (K-major MMA operand)
//   P  [r][64 tokens][128 B]          P, bf16, 128-byte swizzled rows
//   U  [r][dv/32][64 tokens][128 B]   Ut, fp32, 32-column slices, 16-byte chunk q of row i at
//                                     position q ^ (i % 8)
//   X  [r][64 tokens][128 B]          -W K_prev^T (bf16, 128-byte swizzled rows): W of this chunk
//                                     times the K tile of the previous chunk of the document
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
constexpr uint32_t kRecX = 8192;

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
// Sum of squares of one half (columns 32 half .. +31) of a swizzled bf16 row of 64 elements.
__device__ __forceinline__ float row_sumsq_half(const uint8_t* tile, int row, int half) {
    float s[8] = {};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float x[8];
        unpack8(*reinterpret_cast<const uint4*>(tile + swz(row, 4 * half + c)), x);
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
// Then, for every record g < nrec, map[g] = (first token, valid tokens + 65536 if the chunk is
// not the first of its document) ((0, 0) past the last record), so that a prep CTA finds its
// chunk with one load.
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
            const int c = g - (in_smem ? scb[lo] : cb[lo]);
            const int t0 = cu[lo] + c * kChunk;
            m = make_int2(t0, min(kChunk, cu[lo + 1] - t0) + (c > 0 ? 65536 : 0));
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
    static constexpr int KP = V + KB * 8192;          // K tile of the previous chunk, then X
    static constexpr int AF = KP + KB * 8192;         // A, bf16 64 x kLd
    static constexpr int TF = AF + 64 * kLd * 2;      // T, bf16 64 x kLd
    static constexpr int TWN = AF;                    // 128 rows: T_w (0-63), N_b (64-127), written
                                                      // over A and T once T is in registers
    static constexpr int XB = TF + 64 * kLd * 2;      // 4 warps x 16 x 24 bf16
    static constexpr int AB = XB + 4 * 16 * 24 * 2;   // alpha[64], beta[64]
    static constexpr int SC = AB + 512;               // scalar arrays, 64 floats each
    static constexpr int BAR = SC + 8 * 256;
    static constexpr int MISC = BAR + 8 * 8;          // tmem base, abort flag, zero word
    // the X product reads 128 rows from the last -W block: 8 KB past it must be allocated
    static constexpr int BYTES = MISC + 16 > TWN + (KB + 1) * 8192 ? MISC + 16 : TWN + (KB + 1) * 8192;
    static constexpr int TX = KB * 16384 + KB * 8192;  // + KB * 8192 with the previous K tile
    static constexpr uint32_t T_D1 = 0;               // [K K^T | Q K^T] (64 columns), then
    static constexpr uint32_t T_D3 = 0;               // W (D columns, lanes 0-63), then X
    static constexpr uint32_t T_DU = D;               // N_b V (D columns, lanes 64-127)
    static constexpr uint32_t T_COLS = 2 * D;
    static_assert(TWN % 1024 == 0 && TF + 64 * kLd * 2 >= TWN + 16384, "T_w / N_b tile");
    static_assert(2 * (BYTES + 1024 + 1024) <= 233472, "two prep CTAs per SM");
};
enum { PS_G = 0, PS_GAM, PS_BETA, PS_RK, PS_RQ, PS_FTW, PS_UNUSED, PS_COLF };
enum { PB_FULL = 0, PB_TMEM, PB_M1, PB_RA1, PB_M3, PB_RW, PB_MX, PB_FIN, PB_COUNT };

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
    uint8_t* ws_x;
    int* status;
    long long ab_elems;
    const float* A_log;         // gated form: alpha, beta hold the logits of eqs. (9)-(10)
    const float* b_alpha;
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
    bool has_prev;  // the chunk has a predecessor in its document: X is computed
    if (p.map) {
        const int2 m = p.map[g];
        nvalid = m.y & 0xffff;
        if (nvalid <= 0) return;  // grid sized for the worst case
        base = m.x;
        has_prev = (m.y >> 16) != 0;
    } else {
        const int n = g / p.nchunk_dense, c = g % p.nchunk_dense;
        base = (long)n * p.T + (long)c * kChunk;
        nvalid = min(kChunk, p.T - c * kChunk);
        has_prev = c > 0;
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
        // the tile copies first (lane 0's arrival carries the byte count), then log2(alpha) and
        // beta; the other 31 arrivals follow the stores of all lanes
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars[PB_FULL], L::TX + (has_prev ? KB * 8192 : 0));
            const int z = (int)base;
#pragma unroll
            for (int b = 0; b < KB; ++b) {
                tma_load_3d(sm + L::KQ + b * 16384, &tm_k, 64 * b, h, z, &bars[PB_FULL]);
                tma_load_3d(sm + L::KQ + b * 16384 + 8192, &tm_q, 64 * b, h, z, &bars[PB_FULL]);
                tma_load_3d(sm + L::V + b * 8192, &tm_v, 64 * b, h, z, &bars[PB_FULL]);
                if (has_prev)
                    tma_load_3d(sm + L::KP + b * 8192, &tm_k, 64 * b, h, z - kChunk, &bars[PB_FULL]);
            }
        }
        float* ab = reinterpret_cast<float*>(sm + L::AB);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = lane + 32 * u;
            const long t = base + i;
            const bool ok = i < nvalid && GUARD(t * p.H + h < p.ab_elems, DBG_GLOBAL_OOB, 1);
            float lg = 0.f, bt = 0.f;  // rows past the end: alpha = 1, beta = 0
            if (ok) {
                const float av = p.alpha[t * p.H + h], bv = p.beta[t * p.H + h];
                if (p.A_log) {
                    lg = gate_log_decay(av, p.A_log[h], p.b_alpha[h]) * kLog2e;
                    bt = gate_sigmoid(bv);
                } else {
                    lg = lg2(av);
                    bt = bv;
                }
            }
            ab[i] = lg;
            ab[64 + i] = bt;
        }
        __syncwarp();
        if (lane != 0) mbar_arrive(&bars[PB_FULL]);
        // Warm L2 with the tiles of the CTA that will most likely run next on this SM (CTAs are
        // dispatched in index order as slots free up), so that its loads do not wait on DRAM.
        // The same CTA's alpha and beta go in too (one line per token and head), or its loader
        // would wait on DRAM for them.
        const int nt = bid + p.ahead;
        if (nt < p.ntask) {
            const int g2 = nt / p.H, h2 = nt % p.H;
            int z2 = -1, nv2 = 0;
            if (p.map) {
                const int2 m = p.map[g2];
                if ((m.y & 0xffff) > 0) { z2 = m.x; nv2 = m.y & 0xffff; }
            } else {
                const int c2 = g2 % p.nchunk_dense;
                z2 = (g2 / p.nchunk_dense) * p.T + c2 * kChunk;
                nv2 = min(kChunk, p.T - c2 * kChunk);
            }
            if (z2 >= 0) {
                if (lane == 0) {
#pragma unroll
                    for (int b = 0; b < KB; ++b) {
                        tma_prefetch_3d(&tm_k, 64 * b, h2, z2);
                        tma_prefetch_3d(&tm_q, 64 * b, h2, z2);
                        tma_prefetch_3d(&tm_v, 64 * b, h2, z2);
                    }
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int i = lane + 32 * u;
                    const long long e = ((long long)z2 + i) * p.H + h2;
                    if (i < nv2 && e < p.ab_elems) {
                        prefetch_l2(p.alpha + e);
                        prefetch_l2(p.beta + e);
                    }
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
            if (ok && has_prev) {
                // X = -W K_prev^T from the -W image (rows 0-63 of each 64-column block; the
                // 64 rows after it are read too and give unused accumulator rows)
                ok = mbar_wait(&bars[PB_RW], 0, abort_flag);
                if (ok) {
                    tc_fence_after();
                    const uint64_t dWI = sdesc(s0 + L::TWN, 16, 1024);
                    const uint64_t dKP = sdesc(s0 + L::KP, 16, 1024);
#pragma unroll
                    for (int b = 0; b < KB; ++b)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16(tmem + L::T_D3, dWI + b * (8192 >> 4) + kk * KS,
                                     dKP + b * (8192 >> 4) + kk * KS, ID_M1, (b | kk) != 0);
                    mma_commit(&bars[PB_MX]);
                }
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
        float* sColf = scal(PS_COLF);
        float* rs = p.ws_s + rec * (kRecS / 4);

        // (1) decay and norms.  Row t of [K; Q] is summed by both warps of its lane quadrant (hf:
        // the first or the second half of each 64-column block); warp 8 scans log2(alpha) over
        // the chunk, two tokens per lane.
        float* sPart = reinterpret_cast<float*>(sm + L::XB);  // free until the T merges
        bool ok = wwait(PB_FULL, 0);
        float ss = 0.f;
        if (ok) {
            const uint8_t* rows = sm + L::KQ + (t < 64 ? 0 : 8192);
#pragma unroll
            for (int b = 0; b < KB; ++b) ss += row_sumsq_half(rows + b * 16384, t & 63, hf);
            if (hf == 1) sPart[t] = ss;
            if (warp == 8) {
                const float a0 = ab[2 * lane], a1 = ab[2 * lane + 1];
                float incl = a0 + a1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float x = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += x;
                }
                sG[2 * lane] = incl - a1;
                sG[2 * lane + 1] = incl;
                sBeta[2 * lane] = ab[64 + 2 * lane];
                sBeta[2 * lane + 1] = ab[65 + 2 * lane];
            }
        }
        named_sync(1, 256);
        const float Glast = sG[nvalid - 1];
        if (ok && hf == 0) {
            const float rn = p.l2norm ? 1.0f / sqrtf(ss + sPart[t] + kNormEps) : 1.0f;
            if (t < 64) {
                const float G = sG[t], gam = ex2(G);
                sRk[t] = rn;
                sGam[t] = gam;
                sColf[t] = ex2(sG[t | 15] - G);  // decay from token t to the end of its 16-block
                sFtw[t] = sBeta[t] * gam * rn;
                rs[t] = (t < nvalid) ? ex2(Glast - G) * rn : 0.f;
                if (t == 0) rs[128] = ex2(Glast);
            } else {
                const int r = t - 64;
                sRq[r] = rn;
                rs[64 + r] = p.scale * ex2(sG[r]) * rn;
            }
        }
        named_sync(1, 256);

        // (2) A (rows 0-63 of M1, to shared memory) and P (rows 64-127, to the workspace)
        // Gam_ij = 2^(G_i - G_j) for j <= i.  Within the row's own 16-token block it is computed
        // directly; for an earlier block b it is the product 2^(G_i - G_e) 2^(G_e - G_j) through
        // the block's last token e = 16 b + 15.  Both exponents are <= 0 (G does not increase),
        // so neither factor can overflow, and a row needs 20 exponentials instead of 64.  They
        // are taken while the products run.
        const int i = t & 63, blk = i >> 4;
        const bool arow = t < 64;  // rows of A (strictly lower) or of P (lower, diagonal incl.)
        // this warp's columns: blocks 2 hf and 2 hf + 1; the row's own block is among them when
        // blk / 2 == hf (the same for the whole warp)
        float rf[2], dg[16];
        {
            const float Gi = sG[i];
#pragma unroll
            for (int k = 0; k < 2; ++k) rf[k] = ex2(Gi - sG[16 * (2 * hf + k) + 15]);
            if ((blk >> 1) == hf) {
#pragma unroll
                for (int u = 0; u < 16; ++u) dg[u] = ex2(Gi - sG[16 * blk + u]);
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) dg[u] = 0.f;
            }
        }
        ok = wwait(PB_TMEM, 0) && ok;
        tc_fence_after();
        const uint32_t tmem = *tmem_slot;
        ok = wwait(PB_M1, 0) && ok;
        tc_fence_after();
        if (ok) {
            const float sc = arow ? sBeta[i] * sRk[i] : p.scale * sRq[i];
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
                // 32-column slice (2 s + hf) of Ut: 64 rows x 128 bytes
                uint8_t* urec = sm + L::KQ + (size_t)i * 128;
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
                        *reinterpret_cast<float4*>(urec + (2 * s + hf) * 8192 + ((q ^ (i & 7)) << 4)) = u;
                    }
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_sync(1, 256);
        if (ok && t == 0 && hf == 0) {
            if (has_prev) mbar_arrive(&bars[PB_RW]);  // the -W image is ready for X
            bulk_store(p.ws_w + rec * (size_t)(D * 128), sm + L::TWN, D * 128);
            bulk_store(p.ws_u + rec * (size_t)(D * 256), sm + L::KQ, D * 256);
            bulk_commit();
        }
        if (has_prev) {
            // (6) X = -W K_prev^T (lanes 0-63) -> bf16 image over the previous K tile
            ok = wwait(PB_MX, 0) && ok;
            tc_fence_after();
            if (ok && t < 64) {
                float x[32];
                tmem_ld32(tmem + L::T_D3 + lane_base + 32 * hf, x);
                store_half_row_mixed(sm + L::KP, t, hf * 4, x);
            }
            tc_fence_before();
            fence_proxy_async_smem();
            named_sync(1, 256);
            if (ok && t == 0 && hf == 0) {
                bulk_store(p.ws_x + rec * (size_t)8192, sm + L::KP, 8192);
                bulk_commit();
            }
        }
        if (t == 0 && hf == 0) bulk_wait_read();  // shared memory must outlive the copies' reads
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
// Per chunk c of a document, with S^c the state at the chunk's start (S^0 = s0), gamma_c the
// chunk's total decay and U'_c = diag(rk Gam_C / gamma) U_c:
//   S^{c+1} = gamma_c S^c + K_c^T U'_c
//   U_c     = Ut_c - W_c S^c
//           = Ut_c + gamma_{c-1} (-W_c S^{c-1}) + X_c U'_{c-1}     (c >= 1, X_c = -W_c K_{c-1}^T)
//   Y_c     = diag(scale gamma rq) Q_c S^c + P_c U_c
// In the second form U_c needs the state one chunk back, and the step from U_{c-1} to U_c is a
// single 64-token product X_c U'_{c-1}.  So the sequential loop per chunk is
//   (B) pseudo-value epilogue -> M4b = X U' (4 MMAs) -> (B)
// and the state update (M5 and its readout (A)) and the product -W S (M4a) run a chunk behind it:
//   M4a(j)   = [Q_{j-1} ; -W_j] S^{max(j-1,0)}_bf16                 -> D4a[j & 1]
//   M4b(c+1) = [P_c ; X_{c+1}] [U'_hi | U'_lo | U_bf16 | 0]_c        -> D4b[c & 1]
//              rows 64-127, columns 0-63: X_{c+1} U'_c; rows 0-63, columns 64-95: P_c U_c
//   M5(c)    = K_c^T [U'_hi | U'_lo]_c                              -> D5[c & 1]
//   Y_c      = ysc (rows 0-63 of D4a[(c+1) & 1]) + (rows 0-63, columns 64-95 of D4b[c & 1])
// Issuing a tensor-core instruction holds the issuing thread for about as long as the tensor
// pipe takes to execute it, so the products are issued by two threads of their own (one for
// M4a, one for M4b and M5) that wait on the epilogue warps' arrivals; the epilogue warps never
// issue.
template <int D>
struct ChainLayout {
    static constexpr int KB = D / 64;
    // Each operand has a ring of two slots of its own, released by its last reader, so that the
    // copy for chunk c + 2 starts as soon as chunk c no longer needs that operand.
    static constexpr int QWR = 0;                   // slot j: per dk block [Q_{j-1} | -W_j], 16 KB
    static constexpr int PXR = QWR + 2 * KB * 16384; // slot u: [P_u | X_{u+1}], 16 KB
    static constexpr int KR = PXR + 32768;          // slot: K_c, KB x 8 KB
    static constexpr int SB = KR + 2 * KB * 8192;   // 2 buffers: S^c in bf16, D rows x 64 cols
    static constexpr int UU = SB + 2 * D * 128;     // 2 buffers: [U'_hi | U'_lo] then [U_bf16 | 0]
    static constexpr int BAR = UU + 2 * 16384;
    static constexpr int MISC = BAR + 32 * 8;       // tmem base, abort flag, zero word
    static constexpr int BYTES = MISC + 16;
    static constexpr uint32_t T_D4A = 0;            // 2 x 64 columns
    static constexpr uint32_t T_D4B = 128;          // 2 x 128 columns
    static constexpr uint32_t T_D5 = 384;           // 2 x 64 columns
    static constexpr uint32_t T_COLS = 512;
    static_assert(SB % 1024 == 0 && UU % 1024 == 0 && KR % 1024 == 0, "tile alignment");
    static_assert(BYTES + 1024 <= 232448, "shared memory budget");
};
// ring barriers (full / empty per slot), then per-step arrivals and tensor-core completions
enum {
    CB_QWF = 0, CB_QWE = 2, CB_PXF = 4, CB_PXE = 6, CB_KF = 8, CB_KE = 10,  // 12-15 unused
    CB_AD = 16, CB_BD = 18, CB_YD = 20, CB_M4A = 22, CB_M4B = 24, CB_M5 = 26,
    CB_FIN = 28,  // one per issuer: the commit that covers every product it issued
    CB_COUNT = 30
};
static_assert(CB_COUNT <= 32, "the barrier area holds 32 barriers");

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
    const uint8_t* ws_x;
    int* status;
    long long y_elems, state_elems;
};

constexpr int kChainThreads = 512;

// Warp roles: 0 loads the [Q; -W] and [P; X] rings, 1 owns the TMEM allocation and loads the
// K ring (the Ut slices and scalars go straight from global memory into the registers of the
// warps that use them, one chunk ahead); 2, 3, 4, 5, 8, 9, 14, 15 hold the state (16 columns each: rows
// 32 (w % 4) .. +31, columns 0-15 for w < 8, 16-31 otherwise) for the readout (A), warps 4, 5,
// 8, 9 also write Y; 6, 7, 10, 11 run the pseudo-value epilogue (B) on rows 64-127 (16 columns
// each); 12 issues M4a, 13 issues M4b and M5.  Warp w reads TMEM lanes 32 (w % 4) .. +31.
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
    if (tid == 0) {
        for (int b = 0; b < CB_COUNT; ++b) {
            int cnt = 1;
            if (b == CB_AD || b == CB_AD + 1) cnt = 8;
            if (b == CB_BD || b == CB_BD + 1 || b == CB_YD || b == CB_YD + 1) cnt = 4;
            mbar_init(&bars[b], cnt);
        }
        *abort_flag = 0;
        *never = 0;
        fence_mbar_init();
    }
    // the unused columns of the 64-column operand tiles feed only unused accumulator columns;
    // zero them (and the rest of those tiles) once so that they hold finite values
    for (int e = tid; e < (2 * D * 128 + 2 * 16384) / 16; e += kChainThreads)
        reinterpret_cast<uint4*>(sm + L::SB)[e] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
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
        const bool ok = mbar_wait_warp(&bars[bar], parity, abort_flag);
        if (!ok && lane == 0) fail(bar, c);
        return ok;
    };
    // single-thread wait for use `u` of a two-buffer barrier pair: its completion (or, with
    // `empty`, the completion of use u - 2, which frees the slot)
    auto slot_wait = [&](int bar0, int u, bool empty) {
        const uint32_t par = ((u >> 1) & 1) ^ (empty ? 1u : 0u);
        if (mbar_wait(&bars[bar0 + (u & 1)], par, abort_flag)) return true;
        if (!*abort_flag) fail(bar0 + (u & 1), u);
        return false;
    };
    auto spin_done = [&](int bar0, int u) {
        if (mbar_spin(&bars[bar0 + (u & 1)], (u >> 1) & 1, abort_flag)) return true;
        if (!*abort_flag) fail(bar0 + (u & 1), u);
        return false;
    };
    constexpr uint32_t kRecW = D * 128, kRecU = D * 256;
    auto recof = [&](int c) { return (size_t)(cbase + c) * p.H + h; };
    auto zof = [&](int c) { return (int)(t0 + (long)c * kChunk); };
    constexpr uint32_t ID_KN = idesc_bf16(128, 64, false, true);
    constexpr uint32_t ID_KN128 = idesc_bf16(128, 128, false, true);
    constexpr uint32_t ID_M5 = idesc_bf16(128, 64, true, true);
    constexpr uint64_t KS = 32 >> 4, MS = 2048 >> 4;

    if (warp == 0) {
        // ---------------------------------------------------------------- loads: [Q; -W], [P; X]
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            int nq = 0, npx = 0;  // uses issued
            for (int j = 0; j <= nch; ++j) {
                // slot j of the [Q; -W] ring: Q of chunk j - 1, -W of chunk j
                if (!slot_wait(CB_QWE, j, true)) break;
                uint64_t* full = &bars[CB_QWF + (j & 1)];
                mbar_arrive_expect_tx(full, (j >= 1 ? KB * 8192 : 0) + (j < nch ? KB * 8192 : 0));
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    uint8_t* blk = sm + L::QWR + ((j & 1) * KB + b) * 16384;
                    if (j >= 1) tma_load_3d(blk, &tm_q, 64 * b, h, zof(j - 1), full);
                    if (j < nch) bulk_load(blk + 8192, p.ws_w + recof(j) * kRecW + b * 8192, 8192, full);
                }
                ++nq;
                // use j of the [P; X] ring: P of chunk j, X of chunk j + 1 (the last has none)
                if (j < nch) {
                    if (!slot_wait(CB_PXE, j, true)) break;
                    uint64_t* pf = &bars[CB_PXF + (j & 1)];
                    uint8_t* slot = sm + L::PXR + (j & 1) * 16384;
                    mbar_arrive_expect_tx(pf, kRecP + (j + 1 < nch ? kRecX : 0));
                    bulk_load(slot, p.ws_p + recof(j) * kRecP, kRecP, pf);
                    if (j + 1 < nch) bulk_load(slot + 8192, p.ws_x + recof(j + 1) * kRecX, kRecX, pf);
                    ++npx;
                }
                if (j + 2 < nch) {  // warm L2 for the use that will follow in this slot
#pragma unroll
                    for (int b = 0; b < KB; ++b) tma_prefetch_3d(&tm_q, 64 * b, h, zof(j + 1));
                    bulk_prefetch_l2(p.ws_w + recof(j + 2) * kRecW, kRecW);
                    bulk_prefetch_l2(p.ws_p + recof(j + 2) * kRecP, kRecP);
                    if (j + 3 < nch) bulk_prefetch_l2(p.ws_x + recof(j + 3) * kRecX, kRecX);
                }
            }
            // do not exit while a copy or a commit-arrive on this CTA's shared memory is pending
            for (int u = nq - 2 < 0 ? 0 : nq - 2; u < nq; ++u) {
                mbar_wait(&bars[CB_QWF + (u & 1)], (u >> 1) & 1, never, 100000000ull);
                mbar_wait(&bars[CB_QWE + (u & 1)], (u >> 1) & 1, abort_flag);
            }
            for (int u = npx - 2 < 0 ? 0 : npx - 2; u < npx; ++u) {
                mbar_wait(&bars[CB_PXF + (u & 1)], (u >> 1) & 1, never, 100000000ull);
                mbar_wait(&bars[CB_PXE + (u & 1)], (u >> 1) & 1, abort_flag);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- loads: K; L2 warming
        // (the Ut slice and the scalars are read from global memory by the warps that use them,
        // one chunk ahead; here they are only prefetched into L2 two chunks ahead)
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            int nl = 0;
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1;
                if (!slot_wait(CB_KE, c, true)) break;
                uint64_t* kf = &bars[CB_KF + s];
                mbar_arrive_expect_tx(kf, KB * 8192);
#pragma unroll
                for (int b = 0; b < KB; ++b)
                    tma_load_3d(sm + L::KR + (s * KB + b) * 8192, &tm_k, 64 * b, h, zof(c), kf);
                ++nl;
                if (c + 2 < nch) {
                    const size_t rec2 = recof(c + 2);
#pragma unroll
                    for (int b = 0; b < KB; ++b) tma_prefetch_3d(&tm_k, 64 * b, h, zof(c + 2));
                    bulk_prefetch_l2(p.ws_u + rec2 * kRecU + (size_t)jsl * 8192, 8192);
                    bulk_prefetch_l2(p.ws_s + rec2 * (kRecS / 4), kRecS);
                }
            }
            for (int u = nl - 2 < 0 ? 0 : nl - 2; u < nl; ++u) {
                mbar_wait(&bars[CB_KF + (u & 1)], (u >> 1) & 1, never, 100000000ull);
                mbar_wait(&bars[CB_KE + (u & 1)], (u >> 1) & 1, abort_flag);
            }
        }
        __syncwarp();
    } else if (warp == 12) {
        // ---------------------------------------------------------------- issue M4a
        // M4a(j) reads S^{max(j-1,0)} (written by the readout of that step, which also implies
        // that the readers of D4a[j & 1] from step j - 2 are done) and slot j of the [Q; -W] ring
        if (lane == 0) {
            for (int j = 0; j <= nch; ++j) {
                // the copy normally landed long before the readout ends: check it first, so that
                // the readout's arrival is the last wait before the issue
                if (!spin_done(CB_QWF, j) || (j != 1 && !spin_done(CB_AD, j >= 1 ? j - 1 : 0))) break;
                tc_fence_after();
                const int sbuf = (j >= 1 ? j - 1 : 0) & 1;
                const uint64_t dA = sdesc(smem_u32(sm + L::QWR + (j & 1) * KB * 16384), 16, 1024);
                const uint64_t dSB = sdesc(smem_u32(sm + L::SB + sbuf * D * 128), D * 128, 1024);
#pragma unroll
                for (int b = 0; b < KB; ++b)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + L::T_D4A + (j & 1) * 64, dA + b * (16384 >> 4) + kk * KS,
                                 dSB + (b * 4 + kk) * MS, ID_KN, (b | kk) != 0);
                mma_commit(&bars[CB_M4A + (j & 1)]);
                mma_commit(&bars[CB_QWE + (j & 1)]);
            }
            // no product of this thread may still be writing TMEM or arriving on a barrier when
            // the CTA ends, also when a wait above gave up
            mma_commit(&bars[CB_FIN]);
            mbar_wait(&bars[CB_FIN], 0, never, 100000000ull);
        }
        __syncwarp();
    } else if (warp == 13) {
        // ---------------------------------------------------------------- issue M4b and M5
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1;
                // U'_c and U_c are written; the [P; X] slot c has landed; the output warps have
                // read D4b[c & 1] from chunk c - 2
                // (the copy and the output reads normally completed long before the epilogue ends:
                // checked first, so that the epilogue's arrival is the last wait before the issue)
                if (!spin_done(CB_PXF, c) || (c >= 2 && !spin_done(CB_YD, c - 2)) || !spin_done(CB_BD, c)) break;
                tc_fence_after();
                const uint64_t dPX = sdesc(smem_u32(sm + L::PXR + s * 16384), 16, 1024);
                const uint64_t dUU = sdesc(smem_u32(sm + L::UU + s * 16384), 8192, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_D4B + s * 128, dPX + kk * KS, dUU + kk * MS, ID_KN128, kk != 0);
                mma_commit(&bars[CB_M4B + s]);
                mma_commit(&bars[CB_PXE + s]);
                if (!spin_done(CB_KF, c)) break;
                tc_fence_after();
                const uint64_t dKt = sdesc(smem_u32(sm + L::KR + s * KB * 8192), D == 128 ? 8192 : 0, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_D5 + s * 64, dKt + kk * MS, dUU + kk * MS, ID_M5, kk != 0);
                mma_commit(&bars[CB_M5 + s]);
                mma_commit(&bars[CB_KE + s]);
            }
            mma_commit(&bars[CB_FIN + 1]);  // as for the other issuer
            mbar_wait(&bars[CB_FIN + 1], 0, never, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue warps
        const int qd = warp & 3;
        const int srow = qd * 32 + lane;               // TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
        const bool uwarp = warp == 6 || warp == 7 || warp == 10 || warp == 11;
        const bool ywarp = warp == 4 || warp == 5 || warp == 8 || warp == 9;
        const int hf = warp >= 8 ? 1 : 0;              // column half (16 columns) of the warp
        bool ok = true;
        // end of a step: order this warp's shared-memory writes (for the tensor cores) and TMEM
        // reads before the arrival
        auto signal = [&](int bar) {
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[bar]);
        };

        if (!uwarp) {
            // ------------------------------------------------ (A): state readout, and Y
            const int col0 = 16 * hf;
            float S[16], pu[16];
            {
                const size_t o = soff + (size_t)(srow % D) * p.DV + col0;  // D = 64: mirror rows
                const bool in = p.s0 && GUARD((long long)(o + 16) <= p.state_elems, DBG_GLOBAL_OOB, 2);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (in) v = *reinterpret_cast<const float4*>(p.s0 + o + 4 * q);
                    S[4 * q] = v.x; S[4 * q + 1] = v.y; S[4 * q + 2] = v.z; S[4 * q + 3] = v.w;
                }
            }
            // gamma of the previous chunk; the output scale of the previous chunk's rows.  Chunk
            // a's values are loaded at the top of step a and first used at step a + 1.
            float gprev = 1.f, ysprev = 0.f;
            for (int a = 0; a <= nch; ++a) {
                float g_a = 1.f, ys_a = 0.f;
                if (a < nch) {
                    const float* sc = p.ws_s + recof(a) * (kRecS / 4);
                    g_a = __ldg(sc + 128);
                    if (ywarp) ys_a = __ldg(sc + 64 + srow);
                }
                if (a >= 1) {
                    ok = wwait(CB_M5 + ((a - 1) & 1), ((a - 1) >> 1) & 1, a) && ok;
                    tc_fence_after();
                    if (ok) {
                        const uint32_t t5 = tmem + L::T_D5 + ((a - 1) & 1) * 64 + lane_base + col0;
                        float d[16], e[16];
                        tmem_ld16x2(t5, t5 + 32, d, e);
#pragma unroll
                        for (int j = 0; j < 16; ++j) S[j] = fmaf(gprev, S[j], d[j] + e[j]);
                    }
                }
                if (a < nch) {
                    // S^a -> bf16 operand rows (columns col0 .. col0 + 15 of the 64-wide tile)
                    if (ok && srow < D) {
                        uint8_t* sb = sm + L::SB + (a & 1) * D * 128;
                        *reinterpret_cast<uint4*>(sb + swz(srow, col0 / 8)) = pack8(S);
                        *reinterpret_cast<uint4*>(sb + swz(srow, col0 / 8 + 1)) = pack8_fma(S + 8);
                    }
                    signal(CB_AD + (a & 1));
                    gprev = g_a;
                } else if (ok && p.s_final && srow < D) {
                    const size_t o = soff + (size_t)srow * p.DV + col0;
                    if (GUARD((long long)(o + 16) <= p.state_elems, DBG_GLOBAL_OOB, 4)) {
                        float4* dst = reinterpret_cast<float4*>(p.s_final + o);
#pragma unroll
                        for (int q = 0; q < 4; ++q) dst[q] = make_float4(S[4 * q], S[4 * q + 1], S[4 * q + 2], S[4 * q + 3]);
                    }
                }
                if (ywarp && a >= 1) {
                    // Y_{a-1} = ysc (Q_{a-1} S^{a-1}) + P_{a-1} U_{a-1}: rows 0-63 of M4a(a), M4b(a).
                    // P_{a-1} U_{a-1} (M4b(a), complete before M5(a-1) is) goes into registers at
                    // once, releasing the accumulator; both are read after the state image is out,
                    // which the next product waits for.
                    const int cy = a - 1;
                    ok = wwait(CB_M4B + (cy & 1), (cy >> 1) & 1, cy) && ok;
                    tc_fence_after();
                    if (ok) tmem_ld16(tmem + L::T_D4B + (cy & 1) * 128 + 64 + lane_base + col0, pu);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[CB_YD + (cy & 1)]);
                    ok = wwait(CB_M4A + (a & 1), (a >> 1) & 1, a) && ok;
                    tc_fence_after();
                    if (ok) {
                        const int nv = min(kChunk, len - cy * kChunk);
                        float qs[16];
                        tmem_ld16(tmem + L::T_D4A + (a & 1) * 64 + lane_base + col0, qs);
                        const size_t yoff = ((size_t)(t0 + (long)cy * kChunk + srow) * p.H + h) * p.DV + jsl * kNV + col0;
                        if (srow < nv && GUARD((long long)(yoff + 16) <= p.y_elems, DBG_GLOBAL_OOB, 3)) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) qs[j] = fmaf(ysprev, qs[j], pu[j]);
                            uint4* dst = reinterpret_cast<uint4*>(p.y + yoff);
                            dst[0] = pack8(qs);
                            dst[1] = pack8(qs + 8);
                        }
                    }
                    tc_fence_before();
                }
                ysprev = ys_a;
            }
        } else {
            // ------------------------------------------------ (B): pseudo-values, rows 64-127
            const int col0 = 16 * hf;
            const int i = srow - 64;
            float gprev = 1.f;
            // this row's Ut values (16-byte chunk q of row i at position q ^ (i % 8)) and
            // scalars, loaded from the workspace record one chunk before they are used
            auto load_u = [&](int c, float4* u4, float& usv, float& gn) {
                const size_t rec = recof(c);
                const float* scg = p.ws_s + rec * (kRecS / 4);
                usv = __ldg(scg + i);
                gn = __ldg(scg + 128);
                const uint8_t* urow = p.ws_u + rec * kRecU + (size_t)jsl * 8192 + (size_t)i * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    u4[q] = __ldg(reinterpret_cast<const float4*>(urow + (((4 * hf + q) ^ (i & 7)) << 4)));
            };
            float4 utq[4];
            float us = 0.f, gnext = 1.f;
            load_u(0, utq, us, gnext);
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1;
                float4 nutq[4] = {};
                float nus = 0.f, ngn = 1.f;
                if (c + 1 < nch) load_u(c + 1, nutq, nus, ngn);
                ok = wwait(CB_M4A + s, (c >> 1) & 1, c) && ok;
                if (c >= 1) ok = wwait(CB_M4B + ((c - 1) & 1), ((c - 1) >> 1) & 1, c) && ok;
                tc_fence_after();
                if (ok) {
                    float d[16], e[16], f[16];
                    if (c >= 1) {
                        const uint32_t t4 = tmem + L::T_D4B + ((c - 1) & 1) * 128 + lane_base + col0;
                        tmem_ld16x3(tmem + L::T_D4A + s * 64 + lane_base + col0, t4, t4 + 32, d, e, f);
                    } else {
                        tmem_ld16(tmem + L::T_D4A + s * 64 + lane_base + col0, d);
#pragma unroll
                        for (int j = 0; j < 16; ++j) e[j] = f[j] = 0.f;
                    }
                    uint32_t phi[8], plo[8], pub[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 ut = utq[q];
                        const float utv[4] = {ut.x, ut.y, ut.z, ut.w};
                        float u[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int j = 4 * q + e2;
                            u[e2] = fmaf(gprev, d[j], utv[e2] + (e[j] + f[j]));
                        }
#pragma unroll
                        for (int e2 = 0; e2 < 4; e2 += 2) {
                            // U' = hi + lo with hi = U' truncated to bf16 and lo = the exact fp32
                            // rest, itself truncated: |U' - hi - lo| < 2^-14 |U'|
                            const uint32_t b0 = __float_as_uint(u[e2] * us), b1 = __float_as_uint(u[e2 + 1] * us);
                            const float l0 = __uint_as_float(b0) - __uint_as_float(b0 & 0xffff0000u);
                            const float l1 = __uint_as_float(b1) - __uint_as_float(b1 & 0xffff0000u);
                            phi[2 * q + e2 / 2] = __byte_perm(b0, b1, 0x7632);
                            plo[2 * q + e2 / 2] = __byte_perm(__float_as_uint(l0), __float_as_uint(l1), 0x7632);
                            pub[2 * q + e2 / 2] = pack_bf16(u[e2], u[e2 + 1]);
                        }
                    }
                    uint8_t* uhl = sm + L::UU + s * 16384;
                    uint8_t* ub = uhl + 8192;
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        *reinterpret_cast<uint4*>(uhl + swz(i, 2 * hf + q)) = make_uint4(phi[4 * q], phi[4 * q + 1], phi[4 * q + 2], phi[4 * q + 3]);
                        *reinterpret_cast<uint4*>(uhl + swz(i, 4 + 2 * hf + q)) = make_uint4(plo[4 * q], plo[4 * q + 1], plo[4 * q + 2], plo[4 * q + 3]);
                        *reinterpret_cast<uint4*>(ub + swz(i, 2 * hf + q)) = make_uint4(pub[4 * q], pub[4 * q + 1], pub[4 * q + 2], pub[4 * q + 3]);
                    }
                }
                gprev = gnext;
                us = nus;
                gnext = ngn;
#pragma unroll
                for (int q = 0; q < 4; ++q) utq[q] = nutq[q];
                signal(CB_BD + s);
            }
        }
        tc_fence_before();
    }
#undef GUARD
    __syncwarp();
    __syncthreads();
    // every product has completed (the issuers' final commits) and every copy has landed (the
    // loaders' final waits), whether or not a wait gave up: TMEM can be released
    if (warp == 1) {
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
                  ws + w.off_u, reinterpret_cast<float*>(ws + w.off_s), ws + w.off_x, a.status,
                  (long long)tokens * a.H, a.A_log, a.b_alpha};
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
                   reinterpret_cast<const float*>(ws + w.off_s), ws + w.off_x, a.status,
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
    w.off_x = off;
    off += up(R * kRecX);
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
