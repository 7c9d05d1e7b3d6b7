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
// bound is HBM.  Layout: a row of dv = 128 (64) values is read by 32 (16) lanes, four
// consecutive values each (8-byte loads for bf16, 16-byte for fp32), so a warp instruction
// covers whole 256-byte (bf16) rows.  Each warp takes four rows per step to keep more loads in
// flight; the grid is at most 8 blocks per SM, with grid-stride loops over warp steps.
#include "common.cuh"
#include "internal.h"

namespace gdn {

namespace {

constexpr int kNormThreads = 256;
constexpr int kRowsPerStep = 4;  // rows each lane group loads before computing

// sigmoid(x) = 1 / (1 + e^-x) and 1 / sqrt(x), with the fast exponential, divide and reciprocal
// square root intrinsics (the outputs are rounded to the rows' dtype afterwards)
__device__ __forceinline__ float fast_sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

// sum over the LPR lanes that share a row (LPR a power of two, <= 32)
template <int LPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

template <int DV, typename T>
__global__ void __launch_bounds__(kNormThreads)
gated_norm_kernel(const T* __restrict__ y, const T* __restrict__ z, const float* __restrict__ w,
                  T* __restrict__ o, long long rows, float eps) {
    constexpr int LPR = DV / 4;      // lanes per row
    constexpr int RPW = 32 / LPR;    // rows per warp instruction
    constexpr int RW = RPW * kRowsPerStep;  // rows of one warp step
    const int lane = threadIdx.x & 31;
    const int col = (lane % LPR) * 4;
    // the loop runs per warp (its bound is warp-uniform), so every shuffle sees the whole warp
    const long long gw = ((long long)blockIdx.x * kNormThreads + threadIdx.x) >> 5;
    const long long nw = (long long)gridDim.x * (kNormThreads / 32);
    const float4 wv = *reinterpret_cast<const float4*>(w + col);
    const float4 g = make_float4(1.f + wv.x, 1.f + wv.y, 1.f + wv.z, 1.f + wv.w);
    for (long long wb = gw * RW; wb < rows; wb += nw * RW) {
        float4 yv[kRowsPerStep], zv[kRowsPerStep];
#pragma unroll
        for (int u = 0; u < kRowsPerStep; ++u) {
            const long long row = wb + u * RPW + lane / LPR;
            if (row < rows) {
                yv[u] = load4(y + row * DV + col);
                zv[u] = load4(z + row * DV + col);
            } else {
                yv[u] = zv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < kRowsPerStep; ++u) {
            const long long row = wb + u * RPW + lane / LPR;
            const float r = rsqrtf(row_sum<LPR>(dot4(yv[u], yv[u])) * (1.0f / DV) + eps);
            float4 ov;
            ov.x = g.x * yv[u].x * r * fast_sigmoid(zv[u].x);
            ov.y = g.y * yv[u].y * r * fast_sigmoid(zv[u].y);
            ov.z = g.z * yv[u].z * r * fast_sigmoid(zv[u].z);
            ov.w = g.w * yv[u].w * r * fast_sigmoid(zv[u].w);
            if (row < rows) store4(o + row * DV + col, ov);
        }
    }
}

template <int DV, typename T>
__global__ void __launch_bounds__(kNormThreads)
gated_norm_bwd_kernel(const T* __restrict__ y, const T* __restrict__ z,
                      const float* __restrict__ w, const T* __restrict__ d_o, T* __restrict__ dy,
                      T* __restrict__ dz, float* __restrict__ dw, long long rows, float eps) {
    constexpr int LPR = DV / 4;
    constexpr int RPW = 32 / LPR;
    __shared__ float4 s_dw[kNormThreads / 32][LPR];
    constexpr int RW = RPW * kRowsPerStep;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int col = (lane % LPR) * 4;
    const long long gw = ((long long)blockIdx.x * kNormThreads + threadIdx.x) >> 5;
    const long long nw = (long long)gridDim.x * (kNormThreads / 32);
    const float4 wv = *reinterpret_cast<const float4*>(w + col);
    const float4 g = make_float4(1.f + wv.x, 1.f + wv.y, 1.f + wv.z, 1.f + wv.w);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);  // this lane's columns of dw
    for (long long wb = gw * RW; wb < rows; wb += nw * RW) {
        float4 yv[kRowsPerStep], zv[kRowsPerStep], dv[kRowsPerStep];
#pragma unroll
        for (int u = 0; u < kRowsPerStep; ++u) {
            const long long row = wb + u * RPW + lane / LPR;
            if (row < rows) {
                yv[u] = load4(y + row * DV + col);
                zv[u] = load4(z + row * DV + col);
                dv[u] = load4(d_o + row * DV + col);
            } else {
                yv[u] = zv[u] = dv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < kRowsPerStep; ++u) {
            const long long row = wb + u * RPW + lane / LPR;
            const float r = rsqrtf(row_sum<LPR>(dot4(yv[u], yv[u])) * (1.0f / DV) + eps);
            const float4 n = make_float4(yv[u].x * r, yv[u].y * r, yv[u].z * r, yv[u].w * r);
            const float4 s = make_float4(fast_sigmoid(zv[u].x), fast_sigmoid(zv[u].y),
                                         fast_sigmoid(zv[u].z), fast_sigmoid(zv[u].w));
            const float4 ds = make_float4(dv[u].x * s.x, dv[u].y * s.y, dv[u].z * s.z, dv[u].w * s.w);
            const float4 dn = make_float4(ds.x * g.x, ds.y * g.y, ds.z * g.z, ds.w * g.w);
            const float m = row_sum<LPR>(dot4(dn, n)) * (1.0f / DV);
            float4 gy, gz;
            gy.x = r * (dn.x - n.x * m); gy.y = r * (dn.y - n.y * m);
            gy.z = r * (dn.z - n.z * m); gy.w = r * (dn.w - n.w * m);
            gz.x = dn.x * n.x * (1.f - s.x); gz.y = dn.y * n.y * (1.f - s.y);
            gz.z = dn.z * n.z * (1.f - s.z); gz.w = dn.w * n.w * (1.f - s.w);
            if (row < rows) {  // rows past the end (zeros; r may be inf) add nothing
                acc.x = fmaf(ds.x, n.x, acc.x); acc.y = fmaf(ds.y, n.y, acc.y);
                acc.z = fmaf(ds.z, n.z, acc.z); acc.w = fmaf(ds.w, n.w, acc.w);
                store4(dy + row * DV + col, gy);
                store4(dz + row * DV + col, gz);
            }
        }
    }
    // lanes that share columns (the RPW rows of a warp instruction), then the block's warps
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
    if (lane < LPR) s_dw[warp][lane] = acc;
    __syncthreads();
    if (threadIdx.x < LPR) {
        float4 t = s_dw[0][threadIdx.x];
#pragma unroll
        for (int k = 1; k < kNormThreads / 32; ++k) {
            const float4 x = s_dw[k][threadIdx.x];
            t.x += x.x; t.y += x.y; t.z += x.z; t.w += x.w;
        }
        float* p = dw + threadIdx.x * 4;
        atomicAdd(p + 0, t.x);
        atomicAdd(p + 1, t.y);
        atomicAdd(p + 2, t.z);
        atomicAdd(p + 3, t.w);
    }
}

// Blocks: enough for every row slot, at most 8 resident blocks (2048 threads) per SM.
cudaError_t norm_grid(long long rows, int dv, unsigned* grid) {
    int dev = 0, nsm = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const long long rows_per_block = (long long)(kNormThreads / 32) * (128 / dv) * kRowsPerStep;
    const long long need = (rows + rows_per_block - 1) / rows_per_block;
    const long long cap = 8LL * nsm;
    *grid = (unsigned)(need < cap ? need : cap);
    return cudaSuccess;
}

template <int DV, typename T>
cudaError_t fwd(const GatedNormArgs& a, cudaStream_t st) {
    unsigned grid = 0;
    if (cudaError_t e = norm_grid(a.rows, DV, &grid)) return e;
    gated_norm_kernel<DV, T><<<grid, kNormThreads, 0, st>>>(
        static_cast<const T*>(a.y), static_cast<const T*>(a.z), a.w, static_cast<T*>(a.o), a.rows,
        a.eps);
    return cudaGetLastError();
}

template <int DV, typename T>
cudaError_t bwd(const GatedNormArgs& a, cudaStream_t st) {
    unsigned grid = 0;
    if (cudaError_t e = norm_grid(a.rows, DV, &grid)) return e;
    if (cudaError_t e = cudaMemsetAsync(a.dw, 0, sizeof(float) * DV, st)) return e;
    gated_norm_bwd_kernel<DV, T><<<grid, kNormThreads, 0, st>>>(
        static_cast<const T*>(a.y), static_cast<const T*>(a.z), a.w, static_cast<const T*>(a.d_o),
        static_cast<T*>(a.dy), static_cast<T*>(a.dz), a.dw, a.rows, a.eps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gated_norm(const GatedNormArgs& a, cudaStream_t st) {
    if (a.rows == 0) return cudaSuccess;
    if (a.dtype == GDN_BF16)
        return a.dv == 128 ? fwd<128, __nv_bfloat16>(a, st) : fwd<64, __nv_bfloat16>(a, st);
    return a.dv == 128 ? fwd<128, float>(a, st) : fwd<64, float>(a, st);
}

cudaError_t launch_gated_norm_backward(const GatedNormArgs& a, cudaStream_t st) {
    if (a.rows == 0) return cudaMemsetAsync(a.dw, 0, sizeof(float) * a.dv, st);
    if (a.dtype == GDN_BF16)
        return a.dv == 128 ? bwd<128, __nv_bfloat16>(a, st) : bwd<64, __nv_bfloat16>(a, st);
    return a.dv == 128 ? bwd<128, float>(a, st) : bwd<64, float>(a, st);
}

}  // namespace gdn
