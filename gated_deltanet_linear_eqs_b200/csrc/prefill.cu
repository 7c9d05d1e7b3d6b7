// prefill.cu -- chunked (64-token) gated-delta-rule forward on the sm_100a tensor cores.
//
// Method: eqs. (1)-(4) of the Qwen3.8-Flash-Next summary (picx.dev, "Theoretical foundations")
// with L2-normalised q and k ("Methodology", "1. GDN Hybrid Token Mixing"), evaluated chunk by
// chunk in the WY/UT form (the chunkwise gated delta rule of Yang, Kautz & Hatamizadeh 2024).
// For a chunk of C = 64 tokens starting from state S (dk x dv), with g = ln(alpha),
// G = inclusive cumsum(g), gamma = exp(G), Gam_ij = exp(G_i - G_j):
//
//   A   = strictly-lower( diag(beta) (Kh Kh^T * Gam) ),   T = (I + A)^-1
//   W   = T diag(beta gamma) Kh             U = diag(beta) V + strict(T) diag(beta) V - W S
//   Y   = scale ( diag(gamma) Qh S + (Qh Kh^T * Gam * lower-incl) U )
//   S' = gamma_C S + Kh^T diag(Gam_C,.) U
//
// Kh = diag(rk) K, Qh = diag(rq) Q are the normalised rows; the norms are applied as fp32 row or
// column scales so that the MMA operands K, Q, V stay the exact bf16 inputs.
//
// One CTA owns one chain (sequence or document, head, 64-column slice of dv) and walks its chunks
// in order.  Roles:
//   warp 0      TMA producer: K, Q, V tiles (128B-swizzled) + alpha/beta, 2-stage ring
//   warp 1      tcgen05.mma issuer (one lane); TMEM allocator
//   warps 4..7  one warpgroup for all CUDA-core work: norms, decay, A and P, the 64x64
//               triangular inverse, operand conversion to bf16, TMEM <-> SMEM traffic, y stores
// MMAs per chunk (all M = 128, accumulators in TMEM):
//   M1  [K;Q] K^T                 -> K K^T (lanes 0-63), Q K^T (lanes 64-127)
//   M3  T_w K        (T_w = T diag(beta gamma rk))            -> W
//   M4  [0;N_b] V + [Q;-W] S_bf16 -> Q S (rows 0-63), N_b V - W S (rows 64-127)
//   M5  S += K^T U'_hi + K^T U'_lo   (U' = diag(Gam_C,. rk) U split into two bf16 terms, so the
//                                      state update keeps ~16 mantissa bits)
//   M6  P U_bf16     (P = scale diag(rq) (Q K^T * Gam) diag(rk), causal)
#include <mutex>

// The prefill kernel always carries its bounds guards (shared-memory rows, TMEM columns, global
// extents), each recording the failing index in the device status words and skipping the access.
// A build of this kernel without them raised an illegal-address error on B200 that no guarded
// run has ever shown (every guard passes); until that is explained, only the guarded kernel runs.
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
constexpr int kThreads = 256;
constexpr int kWGBase = 128;  // first thread of the compute warpgroup (warps 4..7)
constexpr int kNV = 64;       // dv columns per CTA
constexpr int kStages = 2;
constexpr int kAPad = 68;     // fp32 row stride (floats) of the A / T scratch

template <int DK>
struct Layout {
    static constexpr int KB = DK / 64;            // 64-wide dk blocks
    static constexpr int KQW_BLOCK = 192 * 128;   // per dk block: rows 0-63 K, 64-127 Q, 128-191 W
    static constexpr int KQW = KB * KQW_BLOCK;
    static constexpr int VT = kChunk * kNV * 2;   // V slice: 64 tokens x 64 dv (one atom column)
    static constexpr int STAGE = KQW + VT;
    static constexpr int AV = kStages * STAGE;           // 128 rows x 64: rows 0-63 zero, 64-127 N_b
    static constexpr int TW = AV + 16384;                // 64 rows x 64 (read as 128 rows)
    static constexpr int SB = TW + 8192;                 // S in bf16: DK rows x 64 dv
    static constexpr int P = SB + DK * 128;              // 64 rows x 64 (read as 128 rows)
    static constexpr int UHI = P + 8192;
    static constexpr int ULO = UHI + 8192;
    static constexpr int UB = ULO + 8192;
    static constexpr int AF = UB + 8192;                 // fp32 A, 64 x kAPad
    static constexpr int TF = AF + 64 * kAPad * 4;       // fp32 T, 64 x kAPad
    static constexpr int XB = TF + 64 * kAPad * 4;       // fp32 3 x 16 x 16
    static constexpr int AB = XB + 3 * 256 * 4;          // per stage alpha[64], beta[64]
    static constexpr int SC = AB + kStages * 512;        // scalar arrays, 8 x 64 floats
    static constexpr int BAR = SC + 8 * 256;             // mbarriers
    static constexpr int MISC = BAR + 16 * 8;            // tmem base, abort flag, scan carry
    static constexpr int BYTES = MISC + 64;
    static constexpr int TX = 2 * KB * 8192 + VT;        // TMA bytes per stage
    // TMEM columns
    static constexpr uint32_t T_S = 0;
    static constexpr uint32_t T_D1 = kNV;
    static constexpr uint32_t T_D3 = T_D1 + 64;
    static constexpr uint32_t T_D4 = T_D3 + DK;
    static constexpr uint32_t T_D6 = T_D4 + kNV;
    static constexpr uint32_t T_COLS = 512;
    static_assert(T_D6 + kNV <= T_COLS, "TMEM budget");
    static_assert(BYTES + 1024 <= 232448, "shared memory budget");
};

// scalar array slots (each 64 floats)
enum { SC_G = 0, SC_GAM, SC_BETA, SC_RK, SC_RQ, SC_USC, SC_YSC, SC_CARRY };
// barrier slots
enum { B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_M1, B_M3, B_M4, B_M56, B_R3, B_R4, B_R5, B_FIN };

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
    long long ab_elems, y_elems, state_elems;  // extents, used by the debug-build guards
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
}

// Write 64 floats as one 128-byte swizzled bf16 row.
__device__ __forceinline__ void store_row_bf16(uint8_t* tile, int row, const float* x) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = pack_bf16(x[8 * c + 0], x[8 * c + 1]);
        u.y = pack_bf16(x[8 * c + 2], x[8 * c + 3]);
        u.z = pack_bf16(x[8 * c + 4], x[8 * c + 5]);
        u.w = pack_bf16(x[8 * c + 6], x[8 * c + 7]);
        *reinterpret_cast<uint4*>(tile + swz(row, c)) = u;
    }
}
// Read one 128-byte swizzled bf16 row as 64 floats.
__device__ __forceinline__ void load_row_bf16(const uint8_t* tile, int row, float* x) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(tile + swz(row, c));
        float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), d = unpack_bf16(u.z), e = unpack_bf16(u.w);
        x[8 * c + 0] = a.x; x[8 * c + 1] = a.y; x[8 * c + 2] = b.x; x[8 * c + 3] = b.y;
        x[8 * c + 4] = d.x; x[8 * c + 5] = d.y; x[8 * c + 6] = e.x; x[8 * c + 7] = e.y;
    }
}
// Sum of squares of one swizzled bf16 row of 64 elements.
__device__ __forceinline__ float row_sumsq(const uint8_t* tile, int row) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(tile + swz(row, c));
        float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), d = unpack_bf16(u.z), e = unpack_bf16(u.w);
        s = fmaf(a.x, a.x, s); s = fmaf(a.y, a.y, s); s = fmaf(b.x, b.x, s); s = fmaf(b.y, b.y, s);
        s = fmaf(d.x, d.x, s); s = fmaf(d.y, d.y, s); s = fmaf(e.x, e.x, s); s = fmaf(e.y, e.y, s);
    }
    return s;
}

template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using L = Layout<DK>;
    constexpr int NSL = 128 / kNV;  // upper bound of slices; actual = DV / kNV
    (void)NSL;
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

    if (nchunks == 0) {  // empty document: the final state is the initial one
        if (p.s_final)
            for (int e = tid; e < DK * kNV; e += kThreads) {
                const int r = e / kNV, c = e % kNV;
                p.s_final[soff + (size_t)r * p.DV + c] = p.s0 ? p.s0[soff + (size_t)r * p.DV + c] : 0.f;
            }
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    float* sc = reinterpret_cast<float*>(sm + L::SC);

    if (tid == 0) {
        mbar_init(&bars[B_FULL0], 32);
        mbar_init(&bars[B_FULL1], 32);
        mbar_init(&bars[B_EMPTY0], 1);
        mbar_init(&bars[B_EMPTY1], 1);
        for (int b = B_M1; b <= B_FIN; ++b) mbar_init(&bars[b], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, L::T_COLS);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto fail = [&]() {
        *abort_flag = 1;
        record_status(p.status, GDN_ERR_TIMEOUT);
    };
#define GUARD(cond, code, detail) GDN_GUARD(cond, p.status, code, detail)
    // shared-memory byte range [off, off + bytes) inside the layout
    auto smem_ok = [&](const void* ptr, int bytes, int tag) {
        const long off = (long)((const uint8_t*)ptr - sm);
        return GUARD(off >= 0 && off + bytes <= L::BYTES, DBG_SMEM_OOB, tag * 1000000L + off);
    };
    auto saddr_ok = [&](uint32_t addr, int bytes, int tag) {
        const long off = (long)addr - (long)smem_u32(sm);
        return GUARD(off >= 0 && off + bytes <= L::BYTES && (off & 15) == 0, DBG_SMEM_OOB,
                     tag * 1000000L + off);
    };
    auto tcol_ok = [&](uint32_t col, int width, int tag) {
        return GUARD(col + width <= L::T_COLS, DBG_TMEM_OOB, tag * 1000000L + col);
    };
    auto wait_fail = [&](int bar, int c) {
        (void)GUARD(false, DBG_WAIT, (long)bar * 65536 + c);
        fail();
    };
    (void)smem_ok; (void)saddr_ok; (void)tcol_ok;
    // Warpgroup wait: every warp polls, then the four warps meet at the named barrier and all
    // take the same decision from the shared abort flag, so a timeout in one warp can never
    // leave the others blocked at a later bar.sync.
    auto wg_wait = [&](int bar, uint32_t parity, int c) {
        if (!mbar_wait_warp(&bars[bar], parity, abort_flag)) wait_fail(bar, c);
        named_sync(1, 128);
        return *abort_flag == 0;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint32_t ph = (c >> 1) & 1;
            if (!mbar_wait_warp(&bars[B_EMPTY0 + s], ph ^ 1, abort_flag)) { wait_fail(B_EMPTY0 + s, c); break; }
            uint8_t* stage = sm + s * L::STAGE;
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
                (void)smem_ok(stage, L::STAGE, 2);
#pragma unroll
                for (int b = 0; b < L::KB; ++b) {
                    tma_load_3d(stage + b * L::KQW_BLOCK, &tm_k, 64 * b, h, z, &bars[B_FULL0 + s]);
                    tma_load_3d(stage + b * L::KQW_BLOCK + 8192, &tm_q, 64 * b, h, z, &bars[B_FULL0 + s]);
                }
                tma_load_3d(stage + L::KQW, &tm_v, jsl * kNV, h, z, &bars[B_FULL0 + s]);
            } else {
                mbar_arrive(&bars[B_FULL0 + s]);
            }
            ++issued;
        }
        // Tail of the ring: the CTA must not exit while an asynchronous write to its shared
        // memory is still pending -- neither a TMA load (full barrier) nor the tensor core's
        // commit-arrive that releases a stage (empty barrier), which nobody else waits for
        // on the last two chunks.
        for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c) {
            mbar_wait_warp(&bars[B_FULL0 + (c & 1)], (c >> 1) & 1, abort_flag, 100000000ull);
            mbar_wait_warp(&bars[B_EMPTY0 + (c & 1)], (c >> 1) & 1, abort_flag);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_M1 = idesc_bf16(128, 64, false, false);
            constexpr uint32_t ID_M3 = idesc_bf16(128, DK, false, true);
            constexpr uint32_t ID_KN = idesc_bf16(128, kNV, false, true);  // K-major A, MN-major B
            constexpr uint32_t ID_M5 = idesc_bf16(128, kNV, true, true);
            const uint32_t lbo_k = (DK == 128) ? L::KQW_BLOCK : 0;  // DK=64: rows 64-127 repeat 0-63
            bool ok = true;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int s = c & 1;
                const uint32_t ph = (c >> 1) & 1, cp = c & 1;
                const uint32_t st = smem_u32(sm + s * L::STAGE);
                if (!mbar_wait(&bars[B_FULL0 + s], ph, abort_flag)) { wait_fail(B_FULL0 + s, c); break; }
                tc_fence_after();
                // M1: [K;Q] K^T
                for (int b = 0; b < L::KB; ++b)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t a = st + b * L::KQW_BLOCK + kk * 32;
                        mma_bf16(tmem + L::T_D1, sdesc(a, 16, 1024), sdesc(a, 16, 1024), ID_M1,
                                 (b | kk) != 0);
                    }
                mma_commit(&bars[B_M1]);
                // M3: T_w K  (B = K as an MN-major operand, N = dk)
                if (!mbar_wait(&bars[B_R3], cp, abort_flag)) { wait_fail(B_R3, c); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_D3, sdesc(smem_u32(sm + L::TW) + kk * 32, 16, 1024),
                             sdesc(st + kk * 2048, L::KQW_BLOCK, 1024), ID_M3, kk != 0);
                mma_commit(&bars[B_M3]);
                // M4: [0;N_b] V + [Q;-W] S
                if (!mbar_wait(&bars[B_R4], cp, abort_flag)) { wait_fail(B_R4, c); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_D4, sdesc(smem_u32(sm + L::AV) + kk * 32, 16, 1024),
                             sdesc(st + L::KQW + kk * 2048, 8192, 1024), ID_KN, kk != 0);
                for (int b = 0; b < L::KB; ++b)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + L::T_D4,
                                 sdesc(st + b * L::KQW_BLOCK + 8192 + kk * 32, 16, 1024),
                                 sdesc(smem_u32(sm + L::SB) + (b * 4 + kk) * 2048, DK * 128, 1024),
                                 ID_KN, 1);
                mma_commit(&bars[B_M4]);
                // M5: S += K^T (U_hi + U_lo);  M6: P U
                if (!mbar_wait(&bars[B_R5], cp, abort_flag)) { wait_fail(B_R5, c); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_S, sdesc(st + kk * 2048, lbo_k, 1024),
                             sdesc(smem_u32(sm + L::UHI) + kk * 2048, 8192, 1024), ID_M5, 1);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_S, sdesc(st + kk * 2048, lbo_k, 1024),
                             sdesc(smem_u32(sm + L::ULO) + kk * 2048, 8192, 1024), ID_M5, 1);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + L::T_D6, sdesc(smem_u32(sm + L::P) + kk * 32, 16, 1024),
                             sdesc(smem_u32(sm + L::UB) + kk * 2048, 8192, 1024), ID_KN, kk != 0);
                mma_commit(&bars[B_M56]);
                mma_commit(&bars[B_EMPTY0 + s]);
            }
            // make sure no MMA is still writing TMEM before the warpgroups leave
            mma_commit(&bars[B_FIN]);
            mbar_wait(&bars[B_FIN], 0, abort_flag, 100000000ull);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ compute warpgroup
        const int t = tid - kWGBase;         // 0..127 == TMEM lane
        const int wq = t >> 5;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        float* sG = sc + SC_G * 64;
        float* sGam = sc + SC_GAM * 64;
        float* sBeta = sc + SC_BETA * 64;
        float* sRk = sc + SC_RK * 64;
        float* sRq = sc + SC_RQ * 64;
        float* sUsc = sc + SC_USC * 64;
        float* sYsc = sc + SC_YSC * 64;
        float* sCarry = sc + SC_CARRY * 64;
        float* AF = reinterpret_cast<float*>(sm + L::AF);
        float* TF = reinterpret_cast<float*>(sm + L::TF);
        float* XB = reinterpret_cast<float*>(sm + L::XB);
        const int srow = t % DK;  // state row handled by this thread (DK=64: lanes 64-127 mirror 0-63)

        // zero the top half of AV; load the initial state into TMEM
        {
            uint4 z = make_uint4(0, 0, 0, 0);
            uint4* av = reinterpret_cast<uint4*>(sm + L::AV);
            for (int e = t; e < 8192 / 16; e += 128) av[e] = z;
            float sv[32];
#pragma unroll
            for (int half = 0; half < kNV / 32; ++half) {
                const bool in = p.s0 && GUARD((long long)(soff + (size_t)srow * p.DV + half * 32 + 32) <= p.state_elems, DBG_GLOBAL_OOB, 2);
#pragma unroll
                for (int cc = 0; cc < 32; ++cc)
                    sv[cc] = in ? p.s0[soff + (size_t)srow * p.DV + half * 32 + cc] : 0.f;
                if (tcol_ok(L::T_S + half * 32, 32, 1)) tmem_st32(tmem + L::T_S + lane_base + half * 32, sv);
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_sync(1, 128);

        bool ok = true;
        float yacc[kNV];
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint32_t ph = (c >> 1) & 1, cp = c & 1;
            uint8_t* stage = sm + s * L::STAGE;
            const float* ab = reinterpret_cast<const float*>(sm + L::AB + s * 512);
            const int nvalid = min(kChunk, len - c * kChunk);

            // (2) decay, norms
            if (!wg_wait(B_FULL0 + s, ph, c)) { ok = false; break; }
            if (t < 64) {
                const float a = ab[t];
                float g = logf(a);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float x = __shfl_up_sync(0xffffffffu, g, o);
                    if (lane >= o) g += x;
                }
                if (t == 31) sCarry[0] = g;
                float ss = 0.f;
#pragma unroll
                for (int b = 0; b < L::KB; ++b) if (smem_ok(stage + b * L::KQW_BLOCK + (t) * 128, 128, 11)) ss += row_sumsq(stage + b * L::KQW_BLOCK, t);
                sRk[t] = p.l2norm ? 1.0f / sqrtf(ss + kNormEps) : 1.0f;
                sBeta[t] = ab[64 + t];
                sG[t] = g;  // warp 1 of the group adds the carry below
            } else {
                const int r = t - 64;
                float ss = 0.f;
#pragma unroll
                for (int b = 0; b < L::KB; ++b) if (smem_ok(stage + b * L::KQW_BLOCK + 8192 + (r) * 128, 128, 12)) ss += row_sumsq(stage + b * L::KQW_BLOCK + 8192, r);
                sRq[r] = p.l2norm ? 1.0f / sqrtf(ss + kNormEps) : 1.0f;
            }
            named_sync(1, 128);
            if (t >= 32 && t < 64) sG[t] += sCarry[0];
            named_sync(1, 128);
            const float Glast = sG[nvalid - 1];
            if (t < 64) {
                const float G = sG[t];
                sGam[t] = expf(G);
                sUsc[t] = (t < nvalid) ? expf(Glast - G) * sRk[t] : 0.f;
            } else {
                const int r = t - 64;
                sYsc[r] = p.scale * expf(sG[r]) * sRq[r];
            }

            // (3) A (rows 0-63) and P (rows 64-127) from M1
            if (!wg_wait(B_M1, cp, c)) { ok = false; break; }
            tc_fence_after();
            {
                float d[64];
                if (tcol_ok(L::T_D1, 32, 13)) tmem_ld32(tmem + L::T_D1 + lane_base, d);
                if (tcol_ok(L::T_D1 + 32, 32, 14)) tmem_ld32(tmem + L::T_D1 + lane_base + 32, d + 32);
                named_sync(1, 128);  // sGam/sUsc/sYsc visible
                if (t < 64) {
                    const int i = t;
                    const float Gi = sG[i], bi = sBeta[i] * sRk[i];
                    float* arow = AF + i * kAPad;
#pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        float4 o;
                        o.x = (j + 0 < i) ? bi * sRk[j + 0] * d[j + 0] * expf(Gi - sG[j + 0]) : 0.f;
                        o.y = (j + 1 < i) ? bi * sRk[j + 1] * d[j + 1] * expf(Gi - sG[j + 1]) : 0.f;
                        o.z = (j + 2 < i) ? bi * sRk[j + 2] * d[j + 2] * expf(Gi - sG[j + 2]) : 0.f;
                        o.w = (j + 3 < i) ? bi * sRk[j + 3] * d[j + 3] * expf(Gi - sG[j + 3]) : 0.f;
                        *reinterpret_cast<float4*>(arow + j) = o;
                    }
                } else {
                    const int r = t - 64;
                    const float Gr = sG[r], pr = p.scale * sRq[r];
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        d[j] = (j <= r) ? pr * sRk[j] * d[j] * expf(Gr - sG[j]) : 0.f;
                    if (smem_ok(sm + L::P + (r) * 128, 128, 15)) store_row_bf16(sm + L::P, r, d);
                }
            }
            named_sync(1, 128);

            // (4) T = (I + A)^-1: 16x16 diagonal blocks by substitution, then block products
            if (t < 64) {
                const int b = t >> 4, l = t & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < r; ++m) acc = fmaf(AF[(16 * b + r) * kAPad + 16 * b + m], x[m], acc);
                    x[r] = (r < l) ? 0.f : (r == l ? 1.f : -acc);
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) TF[(16 * b + r) * kAPad + 16 * b + l] = x[r];
            }
            named_sync(1, 128);
            for (int dd = 1; dd < 4; ++dd) {
                const int nout = (4 - dd) * 256;
                for (int e = t; e < nout; e += 128) {
                    const int blk = e >> 8, w = e & 255, rr = w >> 4, cc = w & 15;
                    const int bi = blk + dd, bj = blk;
                    float acc = 0.f;
                    for (int m = bj; m < bi; ++m)
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            acc = fmaf(AF[(16 * bi + rr) * kAPad + 16 * m + k],
                                       TF[(16 * m + k) * kAPad + 16 * bj + cc], acc);
                    XB[blk * 256 + rr * 16 + cc] = acc;
                }
                named_sync(1, 128);
                for (int e = t; e < nout; e += 128) {
                    const int blk = e >> 8, w = e & 255, rr = w >> 4, cc = w & 15;
                    const int bi = blk + dd, bj = blk;
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        acc = fmaf(TF[(16 * bi + rr) * kAPad + 16 * bi + k], XB[blk * 256 + k * 16 + cc], acc);
                    TF[(16 * bi + rr) * kAPad + 16 * bj + cc] = -acc;
                }
                named_sync(1, 128);
            }

            // (5) T_w = T diag(beta gamma rk) -> TW;  N_b = strict(T) diag(beta) -> AV rows 64-127
            {
                float x[64];
                if (t < 64) {
                    const int i = t;
                    const float* trow = TF + i * kAPad;
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        x[j] = (j <= i) ? trow[j] * sBeta[j] * sGam[j] * sRk[j] : 0.f;
                    if (smem_ok(sm + L::TW + (i) * 128, 128, 16)) store_row_bf16(sm + L::TW, i, x);
                } else {
                    const int i = t - 64;
                    const float* trow = TF + i * kAPad;
#pragma unroll
                    for (int j = 0; j < 64; ++j) x[j] = (j < i) ? trow[j] * sBeta[j] : 0.f;
                    if (smem_ok(sm + L::AV + (64 + i) * 128, 128, 17)) store_row_bf16(sm + L::AV, 64 + i, x);
                }
            }
            fence_proxy_async_smem();
            named_sync(1, 128);
            if (t == 0) mbar_arrive(&bars[B_R3]);

            // (6) -W -> W rows of the stage; S_c -> bf16 operand; TMEM S <- gamma_C S_c
            if (!wg_wait(B_M3, cp, c)) { ok = false; break; }
            tc_fence_after();
            if (t < 64) {
#pragma unroll
                for (int b = 0; b < L::KB; ++b) {
                    float w[64];
                    if (tcol_ok(L::T_D3 + 64 * b, 32, 18)) tmem_ld32(tmem + L::T_D3 + lane_base + 64 * b, w);
                    if (tcol_ok(L::T_D3 + 64 * b + 32, 32, 19)) tmem_ld32(tmem + L::T_D3 + lane_base + 64 * b + 32, w + 32);
#pragma unroll
                    for (int j = 0; j < 64; ++j) w[j] = -w[j];
                    if (smem_ok(stage + b * L::KQW_BLOCK + 16384 + (t) * 128, 128, 20)) store_row_bf16(stage + b * L::KQW_BLOCK + 16384, t, w);
                }
            } else {
                // lanes 64-127 must still take part in the warp-collective loads above
                (void)0;
            }
            if (c > 0) {
                if (!wg_wait(B_M56, (c - 1) & 1, c)) { ok = false; break; }
                tc_fence_after();
            }
            {
                const float gC = expf(Glast);
                float sv[64];
                if (tcol_ok(L::T_S, 32, 21)) tmem_ld32(tmem + L::T_S + lane_base, sv);
                if (tcol_ok(L::T_S + 32, 32, 22)) tmem_ld32(tmem + L::T_S + lane_base + 32, sv + 32);
                if (t < DK && smem_ok(sm + L::SB + (t) * 128, 128, 23)) store_row_bf16(sm + L::SB, t, sv);
#pragma unroll
                for (int j = 0; j < 64; ++j) sv[j] *= gC;
                if (tcol_ok(L::T_S, 32, 24)) tmem_st32(tmem + L::T_S + lane_base, sv);
                if (tcol_ok(L::T_S + 32, 32, 25)) tmem_st32(tmem + L::T_S + lane_base + 32, sv + 32);
            }
            tc_fence_before();
            fence_proxy_async_smem();
            named_sync(1, 128);
            if (t == 0) mbar_arrive(&bars[B_R4]);

            // (7) U (rows 64-127 of M4) -> U'_hi, U'_lo, U_bf16;  rows 0-63: y partial
            if (!wg_wait(B_M4, cp, c)) { ok = false; break; }
            tc_fence_after();
            {
                float dv[64];
                if (tcol_ok(L::T_D4, 32, 26)) tmem_ld32(tmem + L::T_D4 + lane_base, dv);
                if (tcol_ok(L::T_D4 + 32, 32, 27)) tmem_ld32(tmem + L::T_D4 + lane_base + 32, dv + 32);
                if (t >= 64) {
                    const int i = t - 64;
                    float vv[64];
                    if (smem_ok(stage + L::KQW + (i) * 128, 128, 28)) load_row_bf16(stage + L::KQW, i, vv);
                    const float bi = sBeta[i], us = sUsc[i];
                    const bool valid = i < nvalid;
                    float hi[64], lo[64];
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const float u = valid ? fmaf(bi, vv[j], dv[j]) : 0.f;
                        const float up = u * us;
                        const float h16 = __bfloat162float(__float2bfloat16_rn(up));
                        hi[j] = h16;
                        lo[j] = up - h16;
                        vv[j] = u;
                    }
                    if (smem_ok(sm + L::UHI + (i) * 128, 128, 29)) store_row_bf16(sm + L::UHI, i, hi);
                    if (smem_ok(sm + L::ULO + (i) * 128, 128, 30)) store_row_bf16(sm + L::ULO, i, lo);
                    if (smem_ok(sm + L::UB + (i) * 128, 128, 31)) store_row_bf16(sm + L::UB, i, vv);
                } else {
                    const float ys = sYsc[t];
#pragma unroll
                    for (int j = 0; j < 64; ++j) yacc[j] = ys * dv[j];
                }
            }
            fence_proxy_async_smem();
            named_sync(1, 128);
            if (t == 0) mbar_arrive(&bars[B_R5]);

            // (8) y = y partial + P U
            if (!wg_wait(B_M56, cp, c)) { ok = false; break; }
            tc_fence_after();
            {
                float d6[64];
                if (tcol_ok(L::T_D6, 32, 32)) tmem_ld32(tmem + L::T_D6 + lane_base, d6);
                if (tcol_ok(L::T_D6 + 32, 32, 33)) tmem_ld32(tmem + L::T_D6 + lane_base + 32, d6 + 32);
                const size_t yoff = ((size_t)(t0 + (long)c * kChunk + t) * p.H + h) * p.DV + jsl * kNV;
                if (t < nvalid && GUARD((long long)(yoff + kNV) <= p.y_elems, DBG_GLOBAL_OOB, 3)) {
                    __nv_bfloat16* yrow = p.y + yoff;
#pragma unroll
                    for (int q8 = 0; q8 < 8; ++q8) {
                        uint4 u;
                        u.x = pack_bf16(yacc[8 * q8 + 0] + d6[8 * q8 + 0], yacc[8 * q8 + 1] + d6[8 * q8 + 1]);
                        u.y = pack_bf16(yacc[8 * q8 + 2] + d6[8 * q8 + 2], yacc[8 * q8 + 3] + d6[8 * q8 + 3]);
                        u.z = pack_bf16(yacc[8 * q8 + 4] + d6[8 * q8 + 4], yacc[8 * q8 + 5] + d6[8 * q8 + 5]);
                        u.w = pack_bf16(yacc[8 * q8 + 6] + d6[8 * q8 + 6], yacc[8 * q8 + 7] + d6[8 * q8 + 7]);
                        *reinterpret_cast<uint4*>(yrow + 8 * q8) = u;
                    }
                }
            }
        }
        // final state
        if (ok && p.s_final) {
            if (wg_wait(B_M56, (nchunks - 1) & 1, nchunks)) {
                tc_fence_after();
                float sv[64];
                if (tcol_ok(L::T_S, 32, 34)) tmem_ld32(tmem + L::T_S + lane_base, sv);
                if (tcol_ok(L::T_S + 32, 32, 35)) tmem_ld32(tmem + L::T_S + lane_base + 32, sv + 32);
                if (t < DK && GUARD((long long)(soff + (size_t)t * p.DV + kNV) <= p.state_elems, DBG_GLOBAL_OOB, 4)) {
                    float* dst = p.s_final + soff + (size_t)t * p.DV;
#pragma unroll
                    for (int j = 0; j < 64; j += 4)
                        *reinterpret_cast<float4*>(dst + j) = make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
                }
            }
        }
        tc_fence_before();
    }
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
