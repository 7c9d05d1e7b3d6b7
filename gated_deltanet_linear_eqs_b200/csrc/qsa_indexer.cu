// qsa_indexer.cu -- the block indexer of Qwen Sparse Attention (Qwen3.8-Flash-Next summary,
// picx.dev, "Methodology", "2. Qwen Sparse Attention (QSA)", eq. (13); the bud-325 wiki entry,
// "Key claims": 4 indexer query heads, 1 shared key head, head dim 128, a budget of 512 blocks).
//
//   k^_b   = RMSNorm(AvgPool(k_{4b .. 4b+3}))                 per document, complete blocks only
//   I[t,b] = sum_{h<4} ReLU(q[t,h] . k^_b)                     for blocks complete at or before t
//   sel[t] = the budget highest-scoring visible blocks (ties to the lower index), sorted, -1 padded
//
// Kernels, in stream order:
//   qsa_base_kernel   one CTA: per document its first key block and its first 32-token query tile
//   qsa_pool_kernel   one warp per key block: mean of its 4 rows, RMS norm with the gain, bf16 k^
//   qsa_score_kernel  one CTA per 32-token query tile of a document: the 32 tokens x 4 heads are
//                     the 128 rows of a tcgen05 product (K = 128) against tiles of 128 key blocks,
//                     loaded by TMA into a two-slot ring and accumulated in two TMEM buffers; the
//                     epilogue takes ReLU, sums the 4 heads of each token (the heads are adjacent
//                     TMEM lanes, so a reduce-scatter over lane pairs) and stores the visible scores
//   qsa_select_kernel one CTA per query token: radix selection of the budget-th largest score over
//                     the token's visible blocks (4 passes of 8 bits on the scores' bit patterns,
//                     which order like the non-negative scores; the row staged once in shared
//                     memory), then an ordered compaction
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kR = 4;          // tokens per key block
constexpr int kD = 128;        // head dim
constexpr int kTileTok = 32;   // query tokens per score CTA: 32 x 4 heads = 128 rows
constexpr int kNB = 128;       // key blocks per product tile
constexpr float kEps = 1e-6f;

// ============================================================================ bases
// block_base[n] = sum_{m<n} floor(len_m / 4), tile_base[n] = sum_{m<n} ceil(len_m / 32); a
// document longer than max_len is recorded in the status word (its rows are then skipped).
__global__ void __launch_bounds__(1024) qsa_base_kernel(const int32_t* __restrict__ cu, int n,
                                                         int max_len, int32_t* __restrict__ block_base,
                                                         int32_t* __restrict__ tile_base,
                                                         int* status) {
    __shared__ int2 wsum[32];
    __shared__ int2 carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = make_int2(0, 0);
    __syncthreads();
    for (int base = 0; base < n; base += 1024) {
        const int i = base + tid;
        int2 v = make_int2(0, 0);
        if (i < n) {
            const int len = cu[i + 1] - cu[i];
            if (len > max_len) record_status(status, GDN_ERR_INVALID_ARG);
            v = len > 0 ? make_int2(len / kR, (len + kTileTok - 1) / kTileTok) : make_int2(0, 0);
        }
        int2 x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int yx = __shfl_up_sync(0xffffffffu, x.x, o), yy = __shfl_up_sync(0xffffffffu, x.y, o);
            if (lane >= o) { x.x += yx; x.y += yy; }
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int2 s = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int yx = __shfl_up_sync(0xffffffffu, s.x, o), yy = __shfl_up_sync(0xffffffffu, s.y, o);
                if (lane >= o) { s.x += yx; s.y += yy; }
            }
            wsum[lane] = s;
        }
        __syncthreads();
        const int2 pre = warp > 0 ? wsum[warp - 1] : make_int2(0, 0);
        const int2 incl = make_int2(carry.x + pre.x + x.x, carry.y + pre.y + x.y);
        if (i < n) {
            block_base[i] = incl.x - v.x;
            tile_base[i] = incl.y - v.y;
        }
        __syncthreads();
        if (tid == 1023) carry = incl;
        __syncthreads();
    }
    if (tid == 0) {
        block_base[n] = carry.x;
        tile_base[n] = carry.y;
    }
}

// the last index m in [0, n) with base[m] <= x (base non-decreasing, base[0] = 0 <= x)
__device__ __forceinline__ int last_le(const int32_t* base, int n, int x) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(base + mid) <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ============================================================================ pooled keys
// One warp per key block; lane l holds dims 4 l .. 4 l + 3 (8 bytes of bf16 per row).
__global__ void __launch_bounds__(256) qsa_pool_kernel(const __nv_bfloat16* __restrict__ k,
                                                        const float* __restrict__ g,
                                                        const int32_t* __restrict__ cu, int n,
                                                        const int32_t* __restrict__ block_base,
                                                        __nv_bfloat16* __restrict__ khat, int nb_cap) {
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int total = __ldg(block_base + n);
    if (b >= total || b >= nb_cap) return;
    const int m = last_le(block_base, n, b);
    const long t0 = (long)__ldg(cu + m) + (long)kR * (b - __ldg(block_base + m));
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < kR; ++r) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(k + (t0 + r) * kD + 4 * lane));
        acc[0] += __uint_as_float(u.x << 16);
        acc[1] += __uint_as_float(u.x & 0xffff0000u);
        acc[2] += __uint_as_float(u.y << 16);
        acc[3] += __uint_as_float(u.y & 0xffff0000u);
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[e] *= 1.f / kR;
        ss = fmaf(acc[e], acc[e], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss * (1.f / kD) + kEps);
    const float4 gv = __ldg(reinterpret_cast<const float4*>(g + 4 * lane));
    const __nv_bfloat162 lo = __floats2bfloat162_rn(gv.x * acc[0] * inv, gv.y * acc[1] * inv);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(gv.z * acc[2] * inv, gv.w * acc[3] * inv);
    *reinterpret_cast<uint2*>(khat + (size_t)b * kD + 4 * lane) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}

// ============================================================================ scores
struct ScoreLayout {
    static constexpr int A = 0;                  // 2 x (128 rows x 128 B): dims 0-63, 64-127
    static constexpr int B = 32768;              // 2 slots x 2 x (128 rows x 128 B)
    static constexpr int BAR = B + 2 * 32768;
    static constexpr int MISC = BAR + 16 * 8;    // tmem base, abort flag, zero word
    static constexpr int BYTES = MISC + 16;
    static constexpr uint32_t T_COLS = 256;      // two 128-column accumulators
};
enum { QB_A = 0, QB_BF = 1, QB_BE = 3, QB_AF = 5, QB_AE = 7, QB_FIN = 9, QB_COUNT = 10 };
// warp 0 loads, warp 1 TMEM + tensor cores, 2..9 epilogue (two per TMEM lane quadrant, each
// taking half of a tile's columns)
constexpr int kScoreThreads = 320;

struct ScoreParams {
    const int32_t* cu;
    const int32_t* block_base;
    const int32_t* tile_base;
    int n, ld;
    float* scores;
    int* status;
};

__global__ void __launch_bounds__(kScoreThreads, 2)
qsa_score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kh,
                 const ScoreParams p) {
    using L = ScoreLayout;
    const int total = __ldg(p.tile_base + p.n);
    if ((int)blockIdx.x >= total) return;
    // later tiles of a document see more blocks: they are dispatched first
    const int tile = total - 1 - (int)blockIdx.x;
    const int m = last_le(p.tile_base, p.n, tile);
    const int start = __ldg(p.cu + m), len = __ldg(p.cu + m + 1) - start;
    const int i0 = (tile - __ldg(p.tile_base + m)) * kTileTok;
    const int ntok = min(kTileTok, len - i0);
    const int nvis_last = (i0 + ntok) / kR;  // blocks visible to the tile's last token
    if (len / kR > p.ld || nvis_last <= 0) return;  // too long (recorded by qsa_base_kernel) or nothing visible
    const int NT = (nvis_last + kNB - 1) / kNB;
    const int kb0 = __ldg(p.block_base + m);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* never = reinterpret_cast<volatile int*>(sm + L::MISC + 8);
    if (tid == 0) {
        for (int b = 0; b < QB_COUNT; ++b) mbar_init(&bars[b], (b == QB_AE || b == QB_AE + 1) ? 8 : 1);
        *abort_flag = 0;
        *never = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, L::T_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() {
        *abort_flag = 1;
        record_status(p.status, GDN_ERR_TIMEOUT);
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- loads
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_kh);
            mbar_arrive_expect_tx(&bars[QB_A], 32768);
            tma_load_3d(sm + L::A, &tm_q, 0, 0, start + i0, &bars[QB_A]);
            tma_load_3d(sm + L::A + 16384, &tm_q, 64, 0, start + i0, &bars[QB_A]);
            int issued = 0;
            for (int nt = 0; nt < NT; ++nt) {
                const int s = nt & 1;
                if (nt >= 2 && !mbar_wait(&bars[QB_BE + s], ((nt >> 1) - 1) & 1, abort_flag)) {
                    if (!*abort_flag) fail();
                    break;
                }
                mbar_arrive_expect_tx(&bars[QB_BF + s], 32768);
                uint8_t* dst = sm + L::B + s * 32768;
                tma_load_3d(dst, &tm_kh, 0, 0, kb0 + kNB * nt, &bars[QB_BF + s]);
                tma_load_3d(dst + 16384, &tm_kh, 64, 0, kb0 + kNB * nt, &bars[QB_BF + s]);
                ++issued;
            }
            // do not leave while a copy is still writing shared memory
            mbar_wait(&bars[QB_A], 0, never, 100000000ull);
            for (int u = issued - 2 < 0 ? 0 : issued - 2; u < issued; ++u)
                mbar_wait(&bars[QB_BF + (u & 1)], (u >> 1) & 1, never, 100000000ull);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- tensor cores
        if (lane == 0) {
            constexpr uint32_t ID = idesc_bf16(128, kNB, false, false);
            const uint64_t dA = sdesc(smem_u32(sm + L::A), 16, 1024);
            constexpr uint64_t KS = 32 >> 4, BLK = 16384 >> 4;
            bool ok = mbar_wait(&bars[QB_A], 0, abort_flag);
            for (int nt = 0; ok && nt < NT; ++nt) {
                const int s = nt & 1;
                ok = mbar_wait(&bars[QB_BF + s], (nt >> 1) & 1, abort_flag) &&
                     (nt < 2 || mbar_wait(&bars[QB_AE + s], ((nt >> 1) - 1) & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                const uint64_t dB = sdesc(smem_u32(sm + L::B + s * 32768), 16, 1024);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + s * kNB, dA + kb * BLK + kk * KS, dB + kb * BLK + kk * KS, ID,
                                 (kb | kk) != 0);
                mma_commit(&bars[QB_BE + s]);
                mma_commit(&bars[QB_AF + s]);
            }
            if (!ok && !*abort_flag) fail();
            // every product has completed before the CTA ends
            mma_commit(&bars[QB_FIN]);
            mbar_wait(&bars[QB_FIN], 0, never, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        // row = 32 q + lane of the accumulator: token 8 q + lane / 4, head lane % 4; this warp
        // takes the 32-column chunks 2 hc and 2 hc + 1 of every tile
        const int q = warp & 3, h = lane & 3, hc = (warp - 2) >> 2;
        const int tl = 8 * q + (lane >> 2);
        const bool row_ok = tl < ntok;
        const int i = i0 + tl;
        const int nvis = (i + 1) / kR;
        float* srow = p.scores + (size_t)(start + i) * p.ld;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        for (int nt = 0; nt < NT; ++nt) {
            const int s = nt & 1;
            if (!mbar_wait_warp(&bars[QB_AF + s], (nt >> 1) & 1, abort_flag)) {
                if (lane == 0 && !*abort_flag) fail();
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int c = 2 * hc; c < 2 * hc + 2; ++c) {
                float v[32];
                tmem_ld32(tmem + s * kNB + 32 * c + lane_base, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.f);
                // heads h and h ^ 2: keep 16 columns, hand the other 16 to the partner
                float part[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float keep = (h & 2) ? v[16 + j] : v[j];
                    const float give = (h & 2) ? v[j] : v[16 + j];
                    part[j] = keep + __shfl_xor_sync(0xffffffffu, give, 2);
                }
                // heads h and h ^ 1: keep 8 of those 16
                float fin[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float keep = (h & 1) ? part[8 + j] : part[j];
                    const float give = (h & 1) ? part[j] : part[8 + j];
                    fin[j] = keep + __shfl_xor_sync(0xffffffffu, give, 1);
                }
                // fin holds the 4-head sums of columns 8 h .. 8 h + 7 of this 32-column chunk
                const int col = kNB * nt + 32 * c + 8 * h;
                if (row_ok && col < nvis)
                    *reinterpret_cast<float4*>(srow + col) = make_float4(fin[0], fin[1], fin[2], fin[3]);
                if (row_ok && col + 4 < nvis)
                    *reinterpret_cast<float4*>(srow + col + 4) = make_float4(fin[4], fin[5], fin[6], fin[7]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[QB_AE + s]);
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::T_COLS);
    }
}

// ============================================================================ selection
constexpr int kSelThreads = 256;
constexpr int kSelSmemKeys = 12288;  // rows of up to this many blocks are staged in shared memory

// exclusive prefix sum of x over the block; *total receives the sum
__device__ __forceinline__ int block_excl_sum(int x, int* sh, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int v = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) sh[warp] = v;
    __syncthreads();
    int pre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        if (w < warp) pre += sh[w];
        tot += sh[w];
    }
    __syncthreads();
    *total = tot;
    return pre + v - x;
}

// scores' bit patterns order like the scores (all >= 0); the sign bit of a -0 is dropped
__device__ __forceinline__ uint32_t score_key(float s) { return __float_as_uint(s) & 0x7fffffffu; }

// One CTA per query token.  The row's keys are read once into shared memory (when they fit);
// each of the 4 radix passes builds a 256-bin histogram of one byte of the keys that match the
// bytes chosen so far, and a suffix sum over the bins (one bin per thread) picks the byte of
// the budget-th largest key.
template <bool kStage>
__global__ void __launch_bounds__(kSelThreads) qsa_select_kernel(const float* __restrict__ scores,
                                                                 int ld, const int32_t* __restrict__ cu,
                                                                 int n, int budget, int32_t* __restrict__ sel) {
    extern __shared__ uint32_t skeys[];
    __shared__ int hist[256];
    __shared__ int sh[kSelThreads / 32];
    __shared__ uint32_t s_prefix;
    __shared__ int s_need;
    const long t = blockIdx.x;
    const int tid = threadIdx.x;
    const int m = last_le(cu, n, (int)t);
    const int i = (int)t - __ldg(cu + m);
    const int nvis = min((i + 1) / kR, ld);
    int32_t* out = sel + t * budget;
    if (nvis <= budget) {
        for (int j = tid; j < budget; j += kSelThreads) out[j] = j < nvis ? j : -1;
        return;
    }
    const float* row = scores + t * ld;
    auto key_at = [&](int b) -> uint32_t {
        return kStage ? skeys[b] : score_key(__ldg(row + b));
    };
    if (kStage) {
        for (int b = tid; b < nvis; b += kSelThreads) skeys[b] = score_key(__ldg(row + b));
    }
    uint32_t prefix = 0, mask = 0;
    int need = budget;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        hist[tid] = 0;  // kSelThreads == 256 bins
        __syncthreads();
        for (int b = tid; b < nvis; b += kSelThreads) {
            const uint32_t key = key_at(b);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
        }
        __syncthreads();
        // suffix sum: above = number of matching keys whose byte is larger than bin 255 - tid
        const int d = 255 - tid, hd = hist[d];
        int total;
        const int above = block_excl_sum(hd, sh, &total);
        if (above < need && above + hd >= need) {
            s_prefix = prefix | ((uint32_t)d << shift);
            s_need = need - above;
        }
        __syncthreads();
        prefix = s_prefix;
        need = s_need;
        mask |= 255u << shift;
    }
    // prefix is the budget-th largest key; `need` of the keys equal to it are taken, lowest
    // block first.  Ordered compaction over contiguous per-thread ranges.
    const int per = (nvis + kSelThreads - 1) / kSelThreads;
    const int b0 = min(nvis, tid * per), b1 = min(nvis, b0 + per);
    int gt = 0, eq = 0;
    for (int b = b0; b < b1; ++b) {
        const uint32_t key = key_at(b);
        gt += key > prefix;
        eq += key == prefix;
    }
    int tot_gt, tot_eq;
    const int gt_before = block_excl_sum(gt, sh, &tot_gt);
    const int eq_before = block_excl_sum(eq, sh, &tot_eq);
    int pos = gt_before + min(eq_before, need), eq_rank = eq_before;
    for (int b = b0; b < b1; ++b) {
        const uint32_t key = key_at(b);
        bool take = key > prefix;
        if (key == prefix) take = eq_rank++ < need;
        if (take && pos < budget) out[pos++] = b;
    }
}

// ---------------------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn qsa_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 3-D bf16 map over [rows, mid, 128]: box 64 (dims) x mid x box_rows, 128-byte swizzle; reads past
// the last row fill with zeros
bool qsa_map(CUtensorMap* mp, const void* base, long rows, int mid, int box_rows) {
    EncodeTiledFn enc = qsa_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)mid, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)mid * kD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)mid, (cuuint32_t)box_rows};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t qsa_workspace_bytes(int num_seqs) { return ((size_t)(num_seqs + 1) * 4 + 255) & ~size_t(255); }

cudaError_t launch_qsa_scores(const QsaArgs& a, cudaStream_t st) {
    if (a.ws == nullptr || a.ws_bytes < qsa_workspace_bytes(a.num_seqs)) return cudaErrorInvalidValue;
    int32_t* tile_base = static_cast<int32_t*>(a.ws);
    qsa_base_kernel<<<1, 1024, 0, st>>>(a.cu_seqlens, a.num_seqs, a.max_doc_len, a.block_base,
                                        tile_base, a.status);
    cudaError_t e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int nb_cap = a.T / kR;
    if (nb_cap == 0) return cudaSuccess;  // no complete block anywhere: no score is visible
    qsa_pool_kernel<<<(unsigned)((nb_cap + 7) / 8), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(a.k), a.g, a.cu_seqlens, a.num_seqs, a.block_base,
        static_cast<__nv_bfloat16*>(a.k_hat), nb_cap);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CUtensorMap mq, mk;
    if (!qsa_map(&mq, a.q, a.T, 4, kTileTok) || !qsa_map(&mk, a.k_hat, nb_cap, 1, kNB))
        return cudaErrorInvalidValue;
    ScoreParams sp{a.cu_seqlens, a.block_base, tile_base, a.num_seqs, a.ld, a.scores, a.status};
    const int smem = ScoreLayout::BYTES + 1024;
    if ((e = cudaFuncSetAttribute(qsa_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
        return e;
    // tiles: sum over documents of ceil(len / 32) <= T / 32 + num_seqs
    const long grid = (long)a.T / kTileTok + a.num_seqs + 1;
    qsa_score_kernel<<<(unsigned)grid, kScoreThreads, smem, st>>>(mq, mk, sp);
    return cudaGetLastError();
}

cudaError_t launch_qsa_select(const QsaArgs& a, cudaStream_t st) {
    if (a.T == 0) return cudaSuccess;
    if (a.ld <= kSelSmemKeys) {
        const int smem = a.ld * 4;
        cudaError_t e;
        if (smem > 48 * 1024 &&
            (e = cudaFuncSetAttribute(qsa_select_kernel<true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
            return e;
        qsa_select_kernel<true><<<(unsigned)a.T, kSelThreads, smem, st>>>(
            a.scores, a.ld, a.cu_seqlens, a.num_seqs, a.budget, a.sel);
    } else {
        qsa_select_kernel<false><<<(unsigned)a.T, kSelThreads, 0, st>>>(
            a.scores, a.ld, a.cu_seqlens, a.num_seqs, a.budget, a.sel);
    }
    return cudaGetLastError();
}

}  // namespace gdn
