// prefill.cu -- chunked (64-token) gated-delta-rule forward on the sm_100a tensor cores.
//
// Method: eqs. (1)-(4) of the Qwen3.8-Flash-Next summary (picx.dev, "Theoretical foundations")
// with L2-normalised q and k ("Methodology", "1. GDN Hybrid Token Mixing"), evaluated chunk by
// chunk in the WY/UT form (the chunkwise gated delta rule of Yang, Kautz & Hatamizadeh 2024).
// For a chunk of C = 64 tokens starting from state S (dk x dv), with G = inclusive cumsum of
// log2(alpha), gamma = 2^G, Gam_ij = 2^(G_i - G_j):
//
//   A   = strictly-lower( diag(beta) (Kh Kh^T * Gam) ),   T = (I + A)^-1
//   W   = T diag(beta gamma) Kh             U = diag(beta) V + strict(T) diag(beta) V - W S
//   Y   = scale ( diag(gamma) Qh S + (Qh Kh^T * Gam * lower-incl) U )
//   S' = gamma_C S + Kh^T diag(Gam_C,.) U
//
// Kh = diag(rk) K, Qh = diag(rq) Q are the normalised rows; the norms are applied as fp32 row or
// column scales so that the MMA operands K, Q, V stay the exact bf16 inputs.
//
// One CTA owns one chain (sequence or document, head, 64-column slice of dv).  Warp roles:
//   warp 0       TMA producer: K, Q, V tiles (128B swizzle) + alpha/beta, 2-stage ring, L2
//                prefetch two chunks ahead
//   warp 1       tcgen05.mma issuer (one lane) with a non-blocking scheduler; TMEM owner
//   warps 4..7   prep warpgroup: the state-independent part of chunk c+1 (decay, norms, A and
//                P, the 64x64 triangular inverse on warp-level mma.sync, T_w, N_b, -W)
//   warps 8..11  chain warpgroup: the state-dependent part of chunk c (S -> bf16 operand and
//                gamma_C S, U epilogue) and the output epilogue of chunk c-1
// MMAs per chunk (M = 128, accumulators in TMEM, bf16 operands):
//   M1  [K;Q] K^T                 -> K K^T (lanes 0-63), Q K^T (lanes 64-127)
//   M3  T_w K        (T_w = T diag(beta gamma rk))            -> W
//   M4  [0;N_b] V + [Q;-W] S_bf16 -> Q S (rows 0-63), N_b V - W S (rows 64-127)   [2 buffers]
//   M5  S += K^T U'_hi + K^T U'_lo   (U' = diag(Gam_C,. rk) U in two bf16 terms, so the state
//                                      update keeps ~16 mantissa bits)
//   M6  P U_bf16     (P = scale diag(rq) (Q K^T * Gam) diag(rk), causal)          [2 buffers]
#include <mutex>

// The prefill kernel always carries its bounds guards (shared-memory rows, TMEM columns, global
// extents), each recording the failing index in the device status words and skipping the access.
// A build of the first version of this kernel without them raised an illegal-address error on
// B200 that no guarded run has ever shown (every guard passes); until that is explained, only
// guarded builds of the kernel run.
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
constexpr int kThreads = 384;
constexpr int kWarpA = 4;  // prep warpgroup: warps 4..7
constexpr int kWarpB = 8;  // chain warpgroup: warps 8..11
constexpr int kNV = 64;    // dv columns per CTA
constexpr int kStages = 2;
constexpr int kLd = 72;    // bf16 row stride (elements) of the A / T scratch: 144-byte rows

template <int DK>
struct Layout {
    static constexpr int KB = DK / 64;            // 64-wide dk blocks
    static constexpr int KQW_BLOCK = 192 * 128;   // per dk block: rows 0-63 K, 64-127 Q, 128-191 W
    static constexpr int KQW = KB * KQW_BLOCK;
    static constexpr int VT = kChunk * kNV * 2;   // V slice: 64 tokens x 64 dv
    static constexpr int STAGE = KQW + VT;
    static constexpr int TW = kStages * STAGE;           // 64 rows (read as 128: then P0)
    static constexpr int P0 = TW + 8192;                 // P, two buffers by chunk parity
    static constexpr int AV = P0 + 2 * 8192;             // 128 rows: 0-63 zero, 64-127 N_b
    static constexpr int SB = AV + 16384;                // S in bf16: DK rows x 64 dv
    static constexpr int UHI = SB + DK * 128;
    static constexpr int ULO = UHI + 8192;
    static constexpr int UB = ULO + 8192;
    static constexpr int AF = UB + 8192;                 // A, bf16 64 x kLd
    static constexpr int TF = AF + 64 * kLd * 2;         // T, bf16 64 x kLd
    static constexpr int XB = TF + 64 * kLd * 2;         // 4 warps x 16 x 24 bf16
    static constexpr int AB = XB + 4 * 16 * 24 * 2;      // per stage alpha[64], beta[64]
    static constexpr int SC = AB + kStages * 512;        // scalars: 2 buffers x 9 x 64 floats
    static constexpr int BAR = SC + 2 * 9 * 256;         // mbarriers
    static constexpr int MISC = BAR + 32 * 8;            // tmem base, abort, exit flags
    static constexpr int BYTES = MISC + 64;
    static constexpr int TX = 2 * KB * 8192 + VT;        // TMA bytes per stage
    static constexpr uint32_t T_S = 0;                   // state, 64 columns
    static constexpr uint32_t T_D1 = 64;                 // [KK^T | QK^T], 64 columns
    static constexpr uint32_t T_D3 = 128;                // W, DK columns
    static constexpr uint32_t T_D4 = 256;                // 2 x 64 columns
    static constexpr uint32_t T_D6 = 384;                // 2 x 64 columns
    static constexpr uint32_t T_COLS = 512;
    static_assert(BYTES + 1024 <= 232448 - 1024, "shared memory budget");
};

// scalar arrays (64 floats each) inside one scalar buffer
enum { SC_G = 0, SC_GAM, SC_BETA, SC_RK, SC_RQ, SC_USC, SC_YSC, SC_FTW, SC_CARRY, SC_SLOTS };
// barriers
enum {
    B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1,  // input ring
    B_M1, B_M3, B_M4, B_M56, B_FIN,            // tensor-core completions (tcgen05.commit)
    B_RA1, B_RAD, B_SCAL,                      // prep warpgroup -> others
    B_RB4, B_RB5, B_YDONE,                     // chain warpgroup -> others
    B_COUNT
};

struct Params {
    const float* alpha;
    const float* beta;
    const float* s0;
    __nv_bfloat16* y;
    float* s_final;
    const int32_t* cu_seqlens;
    int num_seqs, T, H, DV;
    float scale;
    int l2norm;
    int* status;
    long long ab_elems, y_elems, state_elems;  // extents, used by the bounds guards
};

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
// 32 floats -> 4 swizzled 16-byte chunks (chunk index c0..c0+3) of a 128-byte bf16 row
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

template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using L = Layout<DK>;
    const int nsl = p.DV / kNV;
    const int bid = blockIdx.x;
    const int jsl = bid % nsl;
    const int h = (bid / nsl) % p.H;
    const int n = bid / (nsl * p.H);
    long t0, t1;
    if (p.cu_seqlens) {
        t0 = p.cu_seqlens[n];
        t1 = p.cu_seqlens[n + 1];
    } else {
        t0 = (long)n * p.T;
        t1 = t0 + p.T;
    }
    const int len = (int)(t1 - t0);
    const int nchunks = len > 0 ? (len + kChunk - 1) / kChunk : 0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t soff = ((size_t)n * p.H + h) * (size_t)DK * p.DV + (size_t)jsl * kNV;

#define GUARD(cond, code, detail) GDN_GUARD(cond, p.status, code, detail)
    if (nchunks == 0) {  // empty document: the final state is the initial one
        if (p.s_final)
            for (int e = tid; e < DK * kNV; e += kThreads) {
                const int r = e / kNV, c = e % kNV;
                const size_t o = soff + (size_t)r * p.DV + c;
                if (GUARD((long long)o < p.state_elems, DBG_GLOBAL_OOB, 5))
                    p.s_final[o] = p.s0 ? p.s0[o] : 0.f;
            }
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* exit_a = reinterpret_cast<volatile int*>(sm + L::MISC + 8);
    volatile int* exit_b = reinterpret_cast<volatile int*>(sm + L::MISC + 12);

    if (tid == 0) {
        mbar_init(&bars[B_FULL0], 32);
        mbar_init(&bars[B_FULL1], 32);
        for (int b = B_EMPTY0; b < B_COUNT; ++b) mbar_init(&bars[b], 1);
        *abort_flag = 0;
        *exit_a = 0;
        *exit_b = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, L::T_COLS);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto fail = [&](int bar, int c) {
        (void)GUARD(false, DBG_WAIT, (long)bar * 65536 + c);
        *abort_flag = 1;
        record_status(p.status, GDN_ERR_TIMEOUT);
    };
    auto smem_ok = [&](const void* ptr, int bytes, int tag) {
        const long off = (long)((const uint8_t*)ptr - sm);
        return GUARD(off >= 0 && off + bytes <= L::BYTES, DBG_SMEM_OOB, tag * 1000000L + off);
    };
    (void)smem_ok;
    // full-warp wait; on failure the warp records it and continues without doing the work
    auto wwait = [&](int bar, uint32_t parity, int c) {
        const bool ok = mbar_wait_warp(&bars[bar], parity, abort_flag);
        if (!ok && lane == 0) fail(bar, c);
        return ok;
    };
    auto stage_of = [&](int c) { return sm + (c & 1) * L::STAGE; };
    auto scal = [&](int c, int which) { return reinterpret_cast<float*>(sm + L::SC + (c & 1) * (SC_SLOTS * 256) + which * 256); };

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            if (!wwait(B_EMPTY0 + s, ((c >> 1) & 1) ^ 1, c)) break;
            uint8_t* stage = stage_of(c);
            float* ab = reinterpret_cast<float*>(sm + L::AB + s * 512);
            const long base = t0 + (long)c * kChunk;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = lane + 32 * u;
                const long t = base + i;
                const bool ok = t < t1 && GUARD(t * p.H + h < p.ab_elems, DBG_GLOBAL_OOB, 1);
                ab[i] = ok ? p.alpha[t * p.H + h] : 1.f;
                ab[64 + i] = ok ? p.beta[t * p.H + h] : 0.f;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[B_FULL0 + s], L::TX);
                const int z = (int)base;
#pragma unroll
                for (int b = 0; b < L::KB; ++b) {
                    tma_load_3d(stage + b * L::KQW_BLOCK, &tm_k, 64 * b, h, z, &bars[B_FULL0 + s]);
                    tma_load_3d(stage + b * L::KQW_BLOCK + 8192, &tm_q, 64 * b, h, z, &bars[B_FULL0 + s]);
                }
                tma_load_3d(stage + L::KQW, &tm_v, jsl * kNV, h, z, &bars[B_FULL0 + s]);
                if (c + 2 < nchunks) {  // warm L2 for the chunk that will reuse this stage
                    const int z2 = z + 2 * kChunk;
#pragma unroll
                    for (int b = 0; b < L::KB; ++b) {
                        tma_prefetch_3d(&tm_k, 64 * b, h, z2);
                        tma_prefetch_3d(&tm_q, 64 * b, h, z2);
                    }
                    tma_prefetch_3d(&tm_v, jsl * kNV, h, z2);
                }
            } else {
                mbar_arrive(&bars[B_FULL0 + s]);
            }
            ++issued;
        }
        // Tail of the ring: do not exit while a TMA write or a tensor-core commit-arrive on
        // this CTA's shared memory is still pending.
        for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c) {
            mbar_wait_warp(&bars[B_FULL0 + (c & 1)], (c >> 1) & 1, abort_flag, 100000000ull);
            mbar_wait_warp(&bars[B_EMPTY0 + (c & 1)], (c >> 1) & 1, abort_flag);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_M1 = idesc_bf16(128, 64, false, false);
            constexpr uint32_t ID_M3 = idesc_bf16(128, DK, false, true);
            constexpr uint32_t ID_KN = idesc_bf16(128, kNV, false, true);
            constexpr uint32_t ID_M5 = idesc_bf16(128, kNV, true, true);
            const uint32_t lbo_k = (DK == 128) ? L::KQW_BLOCK : 0;  // DK=64: rows 64-127 repeat 0-63
            // Descriptors of every operand, built once; a K step only adds its byte offset / 16
            // to the start-address field (all addresses stay far below 2^18).
            // stage 0 descriptors; stage 1 is the same plus STAGE / 16 in the address field
            const uint32_t st0 = smem_u32(sm);
            const uint64_t dK0 = sdesc(st0, 16, 1024);                // K-major K / [K;Q] rows
            const uint64_t dM3b0 = sdesc(st0, L::KQW_BLOCK, 1024);    // K as MN-major B (N = dk)
            const uint64_t dV0 = sdesc(st0 + L::KQW, 8192, 1024);     // V as MN-major B
            const uint64_t dQW0 = sdesc(st0 + 8192, 16, 1024);        // [Q;-W] rows, K-major A
            const uint64_t dM5a0 = sdesc(st0, lbo_k, 1024);           // K^T as MN-major A
            constexpr uint64_t SST = L::STAGE >> 4;
            const uint64_t dTW = sdesc(smem_u32(sm + L::TW), 16, 1024);
            const uint64_t dAV = sdesc(smem_u32(sm + L::AV), 16, 1024);
            const uint64_t dSB = sdesc(smem_u32(sm + L::SB), DK * 128, 1024);
            const uint64_t dUHI = sdesc(smem_u32(sm + L::UHI), 8192, 1024);
            const uint64_t dULO = sdesc(smem_u32(sm + L::ULO), 8192, 1024);
            const uint64_t dUB = sdesc(smem_u32(sm + L::UB), 8192, 1024);
            const uint64_t dP0 = sdesc(smem_u32(sm + L::P0), 16, 1024);
            constexpr uint64_t PST = 8192 >> 4;
            constexpr uint64_t KS = 32 >> 4;     // K-major: +32 bytes per 16-element K step
            constexpr uint64_t MS = 2048 >> 4;   // MN-major: +2048 bytes per 16-row K step
            constexpr uint64_t BLK = L::KQW_BLOCK >> 4;
            int c1 = 0, c3 = 0, c4 = 0, c5 = 0;
            long long t_last = clock64();
            int idle = 0;
            while (c5 < nchunks) {
                bool did = true;
                if (c5 < c4 && mbar_test(&bars[B_RB5], c5 & 1)) {
                    tc_fence_after();
                    const int s2 = c5 & 1;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + L::T_S, dM5a0 + s2 * SST + kk * MS, dUHI + kk * MS, ID_M5, 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + L::T_S, dM5a0 + s2 * SST + kk * MS, dULO + kk * MS, ID_M5, 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + L::T_D6 + s2 * 64, dP0 + s2 * PST + kk * KS, dUB + kk * MS, ID_KN, kk != 0);
                    mma_commit(&bars[B_M56]);
                    mma_commit(&bars[B_EMPTY0 + s2]);
                    ++c5;
                } else if (c4 < c3 && mbar_test(&bars[B_RAD], c4 & 1) &&
                           mbar_test(&bars[B_RB4], c4 & 1)) {
                    tc_fence_after();
                    const int s2 = c4 & 1;
                    const uint32_t d4 = tmem + L::T_D4 + s2 * 64;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(d4, dAV + kk * KS, dV0 + s2 * SST + kk * MS, ID_KN, kk != 0);
#pragma unroll
                    for (int b = 0; b < L::KB; ++b)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16(d4, dQW0 + s2 * SST + b * BLK + kk * KS, dSB + (b * 4 + kk) * MS, ID_KN, 1);
                    mma_commit(&bars[B_M4]);
                    ++c4;
                } else if (c3 < c1 && mbar_test(&bars[B_RA1], c3 & 1)) {
                    tc_fence_after();
                    const int s2 = c3 & 1;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + L::T_D3, dTW + kk * KS, dM3b0 + s2 * SST + kk * MS, ID_M3, kk != 0);
                    mma_commit(&bars[B_M3]);
                    ++c3;
                } else if (c1 < nchunks && c1 <= c3 &&
                           mbar_test(&bars[B_FULL0 + (c1 & 1)], (c1 >> 1) & 1)) {
                    tc_fence_after();
                    const int s2 = c1 & 1;
#pragma unroll
                    for (int b = 0; b < L::KB; ++b)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t a = dK0 + s2 * SST + b * BLK + kk * KS;
                            mma_bf16(tmem + L::T_D1, a, a, ID_M1, (b | kk) != 0);
                        }
                    mma_commit(&bars[B_M1]);
                    ++c1;
                } else {
                    did = false;
                }
                if (!did) __nanosleep(32);  // leave the issue slots to the warpgroups
                if (did) {
                    idle = 0;
                } else if (++idle >= 64) {  // about 2 s of cycles without progress: give up
                    idle = 0;
                    const long long now = clock64();
                    if (*abort_flag) break;
                    if (t_last == 0) t_last = now;
                    if (now - t_last > 4000000000ll) {
                        fail(B_COUNT, c5);
                        break;
                    }
                    continue;
                }
                if (did) t_last = 0;
            }
            // no MMA may still be writing TMEM when the warpgroups leave
            mma_commit(&bars[B_FIN]);
            mbar_wait(&bars[B_FIN], 0, abort_flag, 100000000ull);
        }
        __syncwarp();
    } else if (warp >= kWarpA && warp < kWarpB) {
        // ================================================================ prep warpgroup
        const int t = tid - kWarpA * 32;   // 0..127 == TMEM lane
        const int wa = t >> 5;
        const uint32_t lane_base = static_cast<uint32_t>(wa * 32) << 16;
        __nv_bfloat16* AF = reinterpret_cast<__nv_bfloat16*>(sm + L::AF);
        __nv_bfloat16* TF = reinterpret_cast<__nv_bfloat16*>(sm + L::TF);
        __nv_bfloat16* XB = reinterpret_cast<__nv_bfloat16*>(sm + L::XB) + wa * 16 * 24;
        for (int c = 0; c < nchunks; ++c) {
            bool ok = true;
            uint8_t* stage = stage_of(c);
            const float* ab = reinterpret_cast<const float*>(sm + L::AB + (c & 1) * 512);
            const int nvalid = min(kChunk, len - c * kChunk);
            float* sG = scal(c, SC_G);
            float* sGam = scal(c, SC_GAM);
            float* sBeta = scal(c, SC_BETA);
            float* sRk = scal(c, SC_RK);
            float* sRq = scal(c, SC_RQ);
            float* sUsc = scal(c, SC_USC);
            float* sYsc = scal(c, SC_YSC);
            float* sCarry = scal(c, SC_CARRY);

            // (1) decay and norms -> scalar buffer of this chunk's parity
            if (c >= 2) ok = wwait(B_YDONE, (c - 2) & 1, c) && ok;  // buffer free again
            ok = wwait(B_FULL0 + (c & 1), (c >> 1) & 1, c) && ok;
            if (ok) {
                if (t < 64) {
                    float g = lg2(ab[t]);
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float x = __shfl_up_sync(0xffffffffu, g, o);
                        if (lane >= o) g += x;
                    }
                    if (t == 31) sCarry[0] = g;
                    float ss = 0.f;
#pragma unroll
                    for (int b = 0; b < L::KB; ++b) ss += row_sumsq(stage + b * L::KQW_BLOCK, t);
                    sRk[t] = p.l2norm ? 1.0f / sqrtf(ss + kNormEps) : 1.0f;
                    sBeta[t] = ab[64 + t];
                    sG[t] = g;
                } else {
                    const int r = t - 64;
                    float ss = 0.f;
#pragma unroll
                    for (int b = 0; b < L::KB; ++b) ss += row_sumsq(stage + b * L::KQW_BLOCK + 8192, r);
                    sRq[r] = p.l2norm ? 1.0f / sqrtf(ss + kNormEps) : 1.0f;
                }
            }
            named_sync(1, 128);
            if (ok && t >= 32 && t < 64) sG[t] += sCarry[0];
            named_sync(1, 128);
            const float Glast = sG[nvalid - 1];
            if (ok) {
                if (t < 64) {
                    const float G = sG[t], gam = ex2(G);
                    sGam[t] = gam;
                    sUsc[t] = (t < nvalid) ? ex2(Glast - G) * sRk[t] : 0.f;
                    scal(c, SC_FTW)[t] = sBeta[t] * gam * sRk[t];
                } else {
                    const int r = t - 64;
                    sYsc[r] = p.scale * ex2(sG[r]) * sRq[r];
                }
            }
            named_sync(1, 128);
            if (t == 0) mbar_arrive(&bars[B_SCAL]);

            // (2) A (rows 0-63) and P (rows 64-127) from M1
            ok = wwait(B_M1, c & 1, c) && ok;
            if (c >= 1) ok = wwait(B_M4, (c - 1) & 1, c) && ok;  // AV and P[c&1] free again
            tc_fence_after();
            if (ok) {
                if (t < 64) {
                    const int i = t;
                    const float Gi = sG[i], bi = sBeta[i] * sRk[i];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float d[32];
                        tmem_ld32(tmem + L::T_D1 + lane_base + half * 32, d);
#pragma unroll
                        for (int j4 = 0; j4 < 32; j4 += 4) {
                            const int j = half * 32 + j4;
                            const float4 rk4 = *reinterpret_cast<const float4*>(sRk + j);
                            const float4 g4 = *reinterpret_cast<const float4*>(sG + j);
                            d[j4 + 0] = (j + 0 < i) ? bi * rk4.x * d[j4 + 0] * ex2(Gi - g4.x) : 0.f;
                            d[j4 + 1] = (j + 1 < i) ? bi * rk4.y * d[j4 + 1] * ex2(Gi - g4.y) : 0.f;
                            d[j4 + 2] = (j + 2 < i) ? bi * rk4.z * d[j4 + 2] * ex2(Gi - g4.z) : 0.f;
                            d[j4 + 3] = (j + 3 < i) ? bi * rk4.w * d[j4 + 3] * ex2(Gi - g4.w) : 0.f;
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<uint4*>(AF + i * kLd + half * 32 + 8 * q) = pack8(d + 8 * q);
                    }
                } else {
                    const int r = t - 64;
                    const float Gr = sG[r], pr = p.scale * sRq[r];
                    uint8_t* P = sm + L::P0 + (c & 1) * 8192;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float d[32];
                        tmem_ld32(tmem + L::T_D1 + lane_base + half * 32, d);
#pragma unroll
                        for (int j4 = 0; j4 < 32; j4 += 4) {
                            const int j = half * 32 + j4;
                            const float4 rk4 = *reinterpret_cast<const float4*>(sRk + j);
                            const float4 g4 = *reinterpret_cast<const float4*>(sG + j);
                            d[j4 + 0] = (j + 0 <= r) ? pr * rk4.x * d[j4 + 0] * ex2(Gr - g4.x) : 0.f;
                            d[j4 + 1] = (j + 1 <= r) ? pr * rk4.y * d[j4 + 1] * ex2(Gr - g4.y) : 0.f;
                            d[j4 + 2] = (j + 2 <= r) ? pr * rk4.z * d[j4 + 2] * ex2(Gr - g4.z) : 0.f;
                            d[j4 + 3] = (j + 3 <= r) ? pr * rk4.w * d[j4 + 3] * ex2(Gr - g4.w) : 0.f;
                        }
                        if (smem_ok(P + r * 128, 128, 15)) store_half_row(P, r, half * 4, d);
                    }
                }
            }
            named_sync(1, 128);

            // (3) T = (I + A)^-1.  16x16 diagonal blocks by forward substitution (fp32), then the
            // off-diagonal blocks T_ij = -D_i sum_m A_im T_mj by diagonals on mma.sync.
            if (ok && t < 64) {
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
            named_sync(1, 128);
            {
                const int mrow = (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix row of this lane
                const int mcol = (lane >> 4) * 8;                      // ldmatrix column offset
                const int gid = lane >> 2, tig = lane & 3;
                for (int dd = 1; dd < 4; ++dd) {
                    if (ok && wa < 4 - dd) {
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
                    named_sync(1, 128);
                }
            }

            // (4) T_w = T diag(beta gamma rk) -> TW;  N_b = strict(T) diag(beta) -> AV rows 64-127
            if (ok) {
                const int i = t & 63;
                const __nv_bfloat16* trow = TF + i * kLd;
                uint8_t* dst = (t < 64) ? sm + L::TW : sm + L::AV;
                const int drow = (t < 64) ? i : 64 + i;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float x[32];
#pragma unroll
                    for (int q = 0; q < 4; ++q) unpack8(*reinterpret_cast<const uint4*>(trow + half * 32 + 8 * q), x + 8 * q);
#pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = half * 32 + j4;
                        const float4 b4 = *reinterpret_cast<const float4*>(sBeta + j);
                        if (t < 64) {
                            const float4 f4 = *reinterpret_cast<const float4*>(scal(c, SC_FTW) + j);
                            x[j4 + 0] = (j + 0 <= i) ? x[j4 + 0] * f4.x : 0.f;
                            x[j4 + 1] = (j + 1 <= i) ? x[j4 + 1] * f4.y : 0.f;
                            x[j4 + 2] = (j + 2 <= i) ? x[j4 + 2] * f4.z : 0.f;
                            x[j4 + 3] = (j + 3 <= i) ? x[j4 + 3] * f4.w : 0.f;
                        } else {
                            x[j4 + 0] = (j + 0 < i) ? x[j4 + 0] * b4.x : 0.f;
                            x[j4 + 1] = (j + 1 < i) ? x[j4 + 1] * b4.y : 0.f;
                            x[j4 + 2] = (j + 2 < i) ? x[j4 + 2] * b4.z : 0.f;
                            x[j4 + 3] = (j + 3 < i) ? x[j4 + 3] * b4.w : 0.f;
                        }
                    }
                    if (smem_ok(dst + drow * 128, 128, 16)) store_half_row(dst, drow, half * 4, x);
                }
            }
            fence_proxy_async_smem();
            named_sync(1, 128);
            if (t == 0) mbar_arrive(&bars[B_RA1]);

            // (5) -W -> the W rows of this chunk's stage
            ok = wwait(B_M3, c & 1, c) && ok;
            tc_fence_after();
            if (ok && t < 64) {
#pragma unroll
                for (int b = 0; b < L::KB; ++b)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float w[32];
                        tmem_ld32(tmem + L::T_D3 + lane_base + 64 * b + 32 * half, w);
#pragma unroll
                        for (int j = 0; j < 32; ++j) w[j] = -w[j];
                        uint8_t* wt = stage + b * L::KQW_BLOCK + 16384;
                        if (smem_ok(wt + t * 128, 128, 20)) store_half_row(wt, t, half * 4, w);
                    }
            }
            fence_proxy_async_smem();
            if (t == 0) *exit_a = *abort_flag;
            named_sync(1, 128);
            if (t == 0) mbar_arrive(&bars[B_RAD]);
            if (*exit_a) break;
            named_sync(1, 128);  // exit_a is read by all before it is written again
        }
    } else if (warp >= kWarpB) {
        // ================================================================ chain warpgroup
        const int t = tid - kWarpB * 32;   // 0..127 == TMEM lane
        const int wb = t >> 5;
        const uint32_t lane_base = static_cast<uint32_t>(wb * 32) << 16;
        const int srow = t % DK;  // state row of this lane (DK=64: lanes 64-127 mirror 0-63)

        // Y of chunk cy: rows 0-63 (lanes 0-63) of D4 (Q S) scaled, plus D6 (P U)
        auto y_epilogue = [&](int cy) {
            if (t >= 64) return;
            const int nv = min(kChunk, len - cy * kChunk);
            const float ys = scal(cy, SC_YSC)[t];
            const size_t yoff = ((size_t)(t0 + (long)cy * kChunk + t) * p.H + h) * p.DV + jsl * kNV;
            const bool store = t < nv && GUARD((long long)(yoff + kNV) <= p.y_elems, DBG_GLOBAL_OOB, 3);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float a[32], b[32];
                tmem_ld32(tmem + L::T_D4 + (cy & 1) * 64 + lane_base + 32 * half, a);
                tmem_ld32(tmem + L::T_D6 + (cy & 1) * 64 + lane_base + 32 * half, b);
                if (store) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) a[j] = fmaf(ys, a[j], b[j]);
                    uint4* dst = reinterpret_cast<uint4*>(p.y + yoff + 32 * half);
#pragma unroll
                    for (int q = 0; q < 4; ++q) dst[q] = pack8(a + 8 * q);
                }
            }
        };

        {   // zero the top half of AV; load the initial state into TMEM
            uint4 z = make_uint4(0, 0, 0, 0);
            uint4* av = reinterpret_cast<uint4*>(sm + L::AV);
            for (int e = t; e < 8192 / 16; e += 128) av[e] = z;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float sv[32];
                const size_t o = soff + (size_t)srow * p.DV + half * 32;
                const bool in = p.s0 && GUARD((long long)(o + 32) <= p.state_elems, DBG_GLOBAL_OOB, 2);
#pragma unroll
                for (int cc = 0; cc < 32; ++cc) sv[cc] = in ? p.s0[o + cc] : 0.f;
                tmem_st32(tmem + L::T_S + lane_base + half * 32, sv);
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_sync(2, 128);

        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int nvalid = min(kChunk, len - c * kChunk);
            uint8_t* stage = stage_of(c);

            // (1) S_c -> bf16 operand; TMEM S <- gamma_C S_c
            ok = wwait(B_SCAL, c & 1, c) && ok;
            if (c >= 1) ok = wwait(B_M56, (c - 1) & 1, c) && ok;
            tc_fence_after();
            if (ok) {
                const float gC = scal(c, SC_GAM)[nvalid - 1];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float sv[32];
                    tmem_ld32(tmem + L::T_S + lane_base + 32 * half, sv);
                    if (t < DK && smem_ok(sm + L::SB + t * 128, 128, 23)) store_half_row(sm + L::SB, t, half * 4, sv);
#pragma unroll
                    for (int j = 0; j < 32; ++j) sv[j] *= gC;
                    tmem_st32(tmem + L::T_S + lane_base + 32 * half, sv);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            named_sync(2, 128);
            if (t == 0) mbar_arrive(&bars[B_RB4]);

            // (2) outputs of the previous chunk (lanes 0-63), while M4 of this chunk runs
            if (c >= 1 && t < 64) {
                if (ok) y_epilogue(c - 1);
                named_sync(3, 64);
                if (t == 0) mbar_arrive(&bars[B_YDONE]);
            }

            // (3) U (rows 64-127 of M4) -> U'_hi, U'_lo, U_bf16
            ok = wwait(B_M4, c & 1, c) && ok;
            tc_fence_after();
            if (ok && t >= 64) {
                const int i = t - 64;
                const float bi = scal(c, SC_BETA)[i], us = scal(c, SC_USC)[i];
                const bool valid = i < nvalid;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float dv[32], vv[32];
                    tmem_ld32(tmem + L::T_D4 + (c & 1) * 64 + lane_base + 32 * half, dv);
                    if (smem_ok(stage + L::KQW + i * 128, 128, 28)) load_half_row(stage + L::KQW, i, half * 4, vv);
                    uint32_t phi[16], plo[16], pub[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const float u0 = valid ? fmaf(bi, vv[j], dv[j]) : 0.f;
                        const float u1 = valid ? fmaf(bi, vv[j + 1], dv[j + 1]) : 0.f;
                        const float p0 = u0 * us, p1 = u1 * us;
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                        const float2 hf = __bfloat1622float2(h2);
                        const __nv_bfloat162 l2 = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(u0, u1);
                        phi[j / 2] = *reinterpret_cast<const uint32_t*>(&h2);
                        plo[j / 2] = *reinterpret_cast<const uint32_t*>(&l2);
                        pub[j / 2] = *reinterpret_cast<const uint32_t*>(&b2);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int ch = half * 4 + q;
                        *reinterpret_cast<uint4*>(sm + L::UHI + swz(i, ch)) = make_uint4(phi[4 * q], phi[4 * q + 1], phi[4 * q + 2], phi[4 * q + 3]);
                        *reinterpret_cast<uint4*>(sm + L::ULO + swz(i, ch)) = make_uint4(plo[4 * q], plo[4 * q + 1], plo[4 * q + 2], plo[4 * q + 3]);
                        *reinterpret_cast<uint4*>(sm + L::UB + swz(i, ch)) = make_uint4(pub[4 * q], pub[4 * q + 1], pub[4 * q + 2], pub[4 * q + 3]);
                    }
                }
            }
            fence_proxy_async_smem();
            if (t == 0) *exit_b = *abort_flag;
            named_sync(2, 128);
            if (t == 0) mbar_arrive(&bars[B_RB5]);
            if (*exit_b) break;
            named_sync(2, 128);  // exit_b is read by all before it is written again
        }
        // outputs of the last chunk and the final state
        if (!*exit_b) {
            ok = wwait(B_M56, (nchunks - 1) & 1, nchunks) && ok;
            tc_fence_after();
            if (ok) {
                y_epilogue(nchunks - 1);
                if (p.s_final) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float sv[32];
                        tmem_ld32(tmem + L::T_S + lane_base + 32 * half, sv);
                        const size_t o = soff + (size_t)t * p.DV + 32 * half;
                        if (t < DK && GUARD((long long)(o + 32) <= p.state_elems, DBG_GLOBAL_OOB, 4)) {
                            float4* dst = reinterpret_cast<float4*>(p.s_final + o);
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                dst[q] = make_float4(sv[4 * q], sv[4 * q + 1], sv[4 * q + 2], sv[4 * q + 3]);
                        }
                    }
                }
            }
        }
        tc_fence_before();
    }
#undef GUARD
    __syncwarp();
    __syncthreads();
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

template <int DK>
cudaError_t launch_dk(const PrefillArgs& a, cudaStream_t st) {
    using L = Layout<DK>;
    const long tokens = a.cu_seqlens ? (long)a.T : (long)a.num_seqs * a.T;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, tokens, a.H, a.dk) || !make_map(&mk, a.k, tokens, a.H, a.dk) ||
        !make_map(&mv, a.v, tokens, a.H, a.dv))
        return cudaErrorInvalidValue;
    Params p{a.alpha, a.beta, a.s0, static_cast<__nv_bfloat16*>(a.y), a.s_final, a.cu_seqlens,
             a.num_seqs, a.T, a.H, a.dv, a.scale, a.l2norm, a.status,
             (long long)tokens * a.H, (long long)tokens * a.H * a.dv,
             (long long)a.num_seqs * a.H * a.dk * a.dv};
    const int smem = L::BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<DK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)a.num_seqs * a.H * (a.dv / kNV);
    prefill_kernel<DK><<<grid, kThreads, smem, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st) {
    // bf16 inputs run the tensor-core kernel; fp32 inputs the exact-fp32 token loop.
    if (a.dtype != GDN_BF16) return launch_prefill_seq(a, st);
    return a.dk == 128 ? launch_dk<128>(a, st) : launch_dk<64>(a, st);
}

}  // namespace gdn
