// gated_norm.cu -- the bracket of eq. (11) of the Qwen3.8-Flash-Next summary (picx.dev,
// "Methodology", "1. GDN Hybrid Token Mixing"):
//
//     o = sigmoid(z) * RMSNorm(y),   RMSNorm(y) = (1 + w) * y / sqrt(mean(y^2) + eps)
//
// per row of dv values (one head of one token; "zero-centred" read as the gain 1 + w), and its
// reverse mode
//
//     n = y r,  s = sigmoid(z):   dz = do (1 + w) n s (1 - s),   dn = do s (1 + w),
//     dy = r (dn - n mean(dn n)),  dw = sum over rows of do s n.
//
// Both are streaming passes (read y, z [, do], write o [, dy, dz]); nothing is reused, so the
// bound is HBM.  The reads are staged through shared memory by bulk copies so that many of them
// are in flight independently of the registers: one persistent CTA per SM, one producer warp
// that copies tiles of consecutive rows (8 KB of each input tensor per tile) into a ring of
// stages (six in the forward, five in the backward), and consumer warps (16 in the forward, 8 in
// the backward) that normalise the rows of a stage (a row of 16 bytes per lane, row sums by
// shuffles) and write the outputs straight to global memory with streaming stores.
// Every wait is bounded: a wait that gives up records GDN_ERR_TIMEOUT and the CTA unwinds.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gdn {

namespace {

// consumer warps: 16 in the forward (two inputs, one output: more warps keep more of the output
// stores in flight), 8 in the backward (three inputs, two outputs and the dw partials)
template <bool BWD>
constexpr int consumers() { return BWD ? 8 : 16; }
template <bool BWD>
constexpr int norm_threads() { return 32 * (consumers<BWD>() + 1); }  // + the producer warp
constexpr int kTileBytes = 8192;                   // per input tensor per tile

// sigmoid(x) = 1 / (1 + e^-x) with the fast exponential and divide intrinsics (the outputs are
// rounded to the rows' dtype afterwards)
__device__ __forceinline__ float fast_sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

// sum over the LPR lanes that share a row (LPR a power of two, <= 32)
template <int LPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// 16 bytes of a row in shared memory -> fp32 values; fp32 values -> 16 bytes of a row in global
// memory (streaming store)
__device__ __forceinline__ void ld16(const uint8_t* p, float* x, __nv_bfloat16) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[2 * j] = __uint_as_float(w[j] << 16);
        x[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
}
__device__ __forceinline__ void ld16(const uint8_t* p, float* x, float) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
__device__ __forceinline__ void st16(__nv_bfloat16* p, const float* x) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    __stcs(reinterpret_cast<uint4*>(p), make_uint4(w[0], w[1], w[2], w[3]));
}
__device__ __forceinline__ void st16(float* p, const float* x) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
}

template <int DV, typename T, bool BWD>
struct NormCfg {
    static constexpr int ROWB = DV * (int)sizeof(T);     // bytes per row
    static constexpr int VPL = 16 / (int)sizeof(T);      // values per lane
    static constexpr int LPR = DV / VPL;                 // lanes per row
    static constexpr int RPW = 32 / LPR;                 // rows per warp instruction
    static constexpr int R = kTileBytes / ROWB;          // rows per tile
    static constexpr int NT = BWD ? 3 : 2;               // input tensors
    static constexpr int STAGES = BWD ? 5 : 6;          // the fastest in a sweep of 3 .. 12
    static constexpr int STAGE = NT * kTileBytes;
    static constexpr int BAR = STAGES * STAGE;           // full[STAGES], empty[STAGES]
    static constexpr int MISC = BAR + 2 * STAGES * 8;    // abort flag
    static constexpr int NC = consumers<BWD>();           // consumer warps
    static constexpr int DWS = MISC + 16;                // dw partials: NC x DV floats
    static constexpr int BYTES = DWS + (BWD ? NC * DV * 4 : 0) + 1024;
    static_assert(R % (NC * RPW) == 0, "rows of a tile split evenly over the warps");
};

template <int DV, typename T, bool BWD>
__global__ void __launch_bounds__(norm_threads<BWD>(), 1)
gated_norm_kernel(const T* __restrict__ y, const T* __restrict__ z, const T* __restrict__ d_o,
                  const float* __restrict__ w, T* __restrict__ o, T* __restrict__ dy,
                  T* __restrict__ dz, float* __restrict__ dw, long long rows, float eps,
                  int* __restrict__ status) {
    using C = NormCfg<DV, T, BWD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::BAR);
    uint64_t* empty = full + C::STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::MISC);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long ntiles = (rows + C::R - 1) / C::R;
    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], C::NC);
        }
        *abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (warp == C::NC) {
        // ------------------------------------------------------------ producer (one lane)
        if (lane == 0) {
            int it = 0;
            for (long long tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x, ++it) {
                const int s = it % C::STAGES;
                if (it >= C::STAGES &&
                    !sm100::mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1, abort_flag))
                    break;
                const long long r0 = tile * C::R;
                const uint32_t bytes = (uint32_t)((rows - r0 < C::R ? rows - r0 : C::R) * C::ROWB);
                sm100::mbar_arrive_expect_tx(&full[s], bytes * C::NT);
                uint8_t* dst = sm + s * C::STAGE;
                sm100::bulk_load(dst, reinterpret_cast<const uint8_t*>(y) + r0 * C::ROWB, bytes, &full[s]);
                sm100::bulk_load(dst + kTileBytes, reinterpret_cast<const uint8_t*>(z) + r0 * C::ROWB, bytes,
                                 &full[s]);
                if (BWD)
                    sm100::bulk_load(dst + 2 * kTileBytes, reinterpret_cast<const uint8_t*>(d_o) + r0 * C::ROWB,
                                     bytes, &full[s]);
            }
            // copies still in flight land before the CTA may end (bounded)
            for (int k = (it > C::STAGES ? it - C::STAGES : 0); k < it; ++k) {
                int never = 0;
                sm100::mbar_wait(&full[k % C::STAGES], (k / C::STAGES) & 1, &never, 100000000ull);
            }
        }
        return;
    }
    // ---------------------------------------------------------------- consumers
    const int col = (lane % C::LPR) * C::VPL;
    float g[C::VPL], acc[C::VPL];  // the gain 1 + w of this lane's columns; its dw partial
#pragma unroll
    for (int j = 0; j < C::VPL; ++j) {
        g[j] = 1.f + w[col + j];
        acc[j] = 0.f;
    }
    int it = 0;
    for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int s = it % C::STAGES;
        if (!sm100::mbar_wait_warp(&full[s], (it / C::STAGES) & 1, abort_flag)) {
            if (lane == 0 && atomicExch(const_cast<int*>(abort_flag), 1) == 0) record_status(status, GDN_ERR_TIMEOUT);
            break;
        }
        const uint8_t* st = sm + s * C::STAGE;
        const long long r0 = tile * C::R;
#pragma unroll
        for (int k = 0; k < C::R / (C::NC * C::RPW); ++k) {
            const int rr = (k * C::NC + warp) * C::RPW + lane / C::LPR;  // row within the tile
            const long long row = r0 + rr;
            float yv[C::VPL], zv[C::VPL];
            ld16(st + rr * C::ROWB + col * (int)sizeof(T), yv, T());
            ld16(st + kTileBytes + rr * C::ROWB + col * (int)sizeof(T), zv, T());
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < C::VPL; ++j) ss = fmaf(yv[j], yv[j], ss);
            const float r = rsqrtf(row_sum<C::LPR>(ss) * (1.0f / DV) + eps);
            if constexpr (!BWD) {
                float ov[C::VPL];
#pragma unroll
                for (int j = 0; j < C::VPL; ++j) ov[j] = g[j] * yv[j] * r * fast_sigmoid(zv[j]);
                if (row < rows) st16(o + row * DV + col, ov);
            } else {
                float dv[C::VPL];
                ld16(st + 2 * kTileBytes + rr * C::ROWB + col * (int)sizeof(T), dv, T());
                float n[C::VPL], sg[C::VPL], ds[C::VPL], dn[C::VPL];
                float m = 0.f;
#pragma unroll
                for (int j = 0; j < C::VPL; ++j) {
                    n[j] = yv[j] * r;
                    sg[j] = fast_sigmoid(zv[j]);
                    ds[j] = dv[j] * sg[j];
                    dn[j] = ds[j] * g[j];
                    m = fmaf(dn[j], n[j], m);
                }
                m = row_sum<C::LPR>(m) * (1.0f / DV);
                float gy[C::VPL], gz[C::VPL];
#pragma unroll
                for (int j = 0; j < C::VPL; ++j) {
                    gy[j] = r * (dn[j] - n[j] * m);
                    gz[j] = dn[j] * n[j] * (1.f - sg[j]);
                }
                if (row < rows) {  // rows past the end of the tensor add nothing
#pragma unroll
                    for (int j = 0; j < C::VPL; ++j) acc[j] = fmaf(ds[j], n[j], acc[j]);
                    st16(dy + row * DV + col, gy);
                    st16(dz + row * DV + col, gz);
                }
            }
        }
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&empty[s]);
    }
    if constexpr (BWD) {
        // dw: the lanes that share columns (the RPW rows of a warp instruction), then the warps
        float* dws = reinterpret_cast<float*>(sm + C::DWS);
#pragma unroll
        for (int o2 = C::LPR; o2 < 32; o2 <<= 1)
#pragma unroll
            for (int j = 0; j < C::VPL; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o2);
        if (lane < C::LPR)
#pragma unroll
            for (int j = 0; j < C::VPL; ++j) dws[warp * DV + col + j] = acc[j];
        asm volatile("bar.sync 1, %0;" ::"r"(32 * C::NC) : "memory");  // the consumer warps
        for (int c = tid; c < DV; c += 32 * C::NC) {
            float t = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < C::NC; ++k2) t += dws[k2 * DV + c];
            atomicAdd(dw + c, t);
        }
    }
}

// One CTA per SM (its shared memory holds the ring), at most one per tile.
template <int DV, typename T, bool BWD>
cudaError_t launch(const GatedNormArgs& a, cudaStream_t st) {
    using C = NormCfg<DV, T, BWD>;
    int dev = 0, nsm = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const long long ntiles = (a.rows + C::R - 1) / C::R;
    const unsigned grid = (unsigned)(ntiles < nsm ? ntiles : nsm);
    if ((e = cudaFuncSetAttribute(gated_norm_kernel<DV, T, BWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  C::BYTES)) != cudaSuccess)
        return e;
    if (BWD && (e = cudaMemsetAsync(a.dw, 0, sizeof(float) * DV, st)) != cudaSuccess) return e;
    gated_norm_kernel<DV, T, BWD><<<grid, norm_threads<BWD>(), C::BYTES, st>>>(
        static_cast<const T*>(a.y), static_cast<const T*>(a.z), static_cast<const T*>(a.d_o), a.w,
        static_cast<T*>(a.o), static_cast<T*>(a.dy), static_cast<T*>(a.dz), a.dw, a.rows, a.eps,
        a.status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gated_norm(const GatedNormArgs& a, cudaStream_t st) {
    if (a.rows == 0) return cudaSuccess;
    if (a.dtype == GDN_BF16)
        return a.dv == 128 ? launch<128, __nv_bfloat16, false>(a, st) : launch<64, __nv_bfloat16, false>(a, st);
    return a.dv == 128 ? launch<128, float, false>(a, st) : launch<64, float, false>(a, st);
}

cudaError_t launch_gated_norm_backward(const GatedNormArgs& a, cudaStream_t st) {
    if (a.rows == 0) return cudaMemsetAsync(a.dw, 0, sizeof(float) * a.dv, st);
    if (a.dtype == GDN_BF16)
        return a.dv == 128 ? launch<128, __nv_bfloat16, true>(a, st) : launch<64, __nv_bfloat16, true>(a, st);
    return a.dv == 128 ? launch<128, float, true>(a, st) : launch<64, float, true>(a, st);
}

}  // namespace gdn
