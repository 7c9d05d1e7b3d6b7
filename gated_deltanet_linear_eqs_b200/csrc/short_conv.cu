// short_conv.cu -- the short causal convolution ahead of the GDN recurrence (Qwen3.8-Flash-Next
// summary, picx.dev, "Methodology", "1. GDN Hybrid Token Mixing": "short causal convolutions"),
// in the depthwise reading: per channel c of a [T, C] tensor (q, k or v, C = H * d),
//
//     y[t, c] = act( sum_{i<W} w[c, i] * x[t - (W - 1) + i, c] ),   act = identity or SiLU,
//
// with every document starting from its conv state (its W - 1 inputs before the first token)
// and leaving its last W - 1 inputs as the state after it.
//
// The pass is HBM-bound (one read of x, one write of y, fp32 arithmetic): each thread owns four
// consecutive channels (one 8-byte vector of bf16, 16 bytes of fp32) and a run of 8 tokens.  It
// issues all of the run's loads at once, keeps the last W - 1 inputs in registers and reads the
// W - 1 rows before the run again (from L2, mostly).  A warp covers 128 channels of one token
// row, so every load and store is a coalesced 256-byte (bf16) row segment; few registers per
// thread leave room for four blocks (32 warps) per SM to keep enough loads in flight.
#include "common.cuh"
#include "internal.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;  // threads per block
constexpr int kCh = 4;         // channels per thread: 1024 channels per block
constexpr int kRun = 8;        // tokens per thread

template <typename T>
struct Vec4;
template <>
struct Vec4<__nv_bfloat16> {
    using Raw = uint2;  // four bf16
    static __device__ __forceinline__ Raw load_raw(const __nv_bfloat16* p) {
        return __ldg(reinterpret_cast<const uint2*>(p));
    }
    static __device__ __forceinline__ void unpack(const Raw& r, float* f) {
        f[0] = __uint_as_float(r.x << 16);
        f[1] = __uint_as_float(r.x & 0xffff0000u);
        f[2] = __uint_as_float(r.y << 16);
        f[3] = __uint_as_float(r.y & 0xffff0000u);
    }
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* f) {
        unpack(load_raw(p), f);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* f) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
        const __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
        *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&a),
                                                  *reinterpret_cast<const uint32_t*>(&b));
    }
};
template <>
struct Vec4<float> {
    using Raw = float4;
    static __device__ __forceinline__ Raw load_raw(const float* p) {
        return __ldg(reinterpret_cast<const float4*>(p));
    }
    static __device__ __forceinline__ void unpack(const Raw& r, float* f) {
        f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
    }
    static __device__ __forceinline__ void load(const float* p, float* f) { unpack(load_raw(p), f); }
    static __device__ __forceinline__ void store(float* p, const float* f) {
        *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
    }
};

// SiLU(x) = x sigmoid(x), with the fast exponential and divide intrinsics
__device__ __forceinline__ float conv_act(float x, bool silu) {
    return silu ? __fdividef(x, 1.f + __expf(-x)) : x;
}

// the W - 1 state rows of one document for this thread's channels (zero without a state)
template <typename T, int W>
__device__ __forceinline__ void load_state(const T* st, size_t n, int C, int c0, float (*win)[kCh]) {
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
        if (st) {
            Vec4<T>::load(st + ((size_t)n * (W - 1) + j) * C + c0, win[j]);
        } else {
#pragma unroll
            for (int e = 0; e < kCh; ++e) win[j][e] = 0.f;
        }
    }
}

template <typename T, int W>
__device__ __forceinline__ void store_state(T* st, size_t n, int C, int c0, const float (*win)[kCh]) {
#pragma unroll
    for (int j = 0; j < W - 1; ++j) Vec4<T>::store(st + ((size_t)n * (W - 1) + j) * C + c0, win[j]);
}

// Grid: x = channel blocks of 1024, y = token runs of kRun.  cu has num_seqs + 1 entries.
// four blocks per SM where the run's registers allow it (bf16, W <= 4), else two
template <typename T, int W>
constexpr int conv_min_blocks() { return (sizeof(T) == 2 && W <= 4) ? 4 : 2; }

template <typename T, int W, bool SILU>
__global__ void __launch_bounds__(kThreads, conv_min_blocks<T, W>()) short_conv_varlen_kernel(
    const T* __restrict__ x, const float* __restrict__ w, const int32_t* __restrict__ cu,
    int num_seqs, const T* __restrict__ st_in, T* __restrict__ st_out, T* __restrict__ y, int Ttot,
    int C) {
    const int c0 = (blockIdx.x * kThreads + threadIdx.x) * kCh;
    if (c0 >= C) return;
    // documents of length zero keep their state; block row r handles documents n = r mod rows
    if (st_out) {
        for (int n = blockIdx.y; n < num_seqs; n += gridDim.y) {
            if (__ldg(cu + n) == __ldg(cu + n + 1)) {
                float win[W > 1 ? W - 1 : 1][kCh];
                load_state<T, W>(st_in, n, C, c0, win);
                store_state<T, W>(st_out, n, C, c0, win);
            }
        }
    }
    const int t0 = blockIdx.y * kRun;
    if (t0 >= Ttot) return;
    const int nrun = min(kRun, Ttot - t0);
    // all of the run's inputs first (raw vectors, unpacked when used)
    typename Vec4<T>::Raw xr[kRun];
#pragma unroll
    for (int r = 0; r < kRun; ++r)
        if (r < nrun) xr[r] = Vec4<T>::load_raw(x + (size_t)(t0 + r) * C + c0);
    // this thread's taps: kCh * W contiguous floats starting at a 16-byte boundary (c0 % 4 == 0)
    float wt[W][kCh];
#pragma unroll
    for (int v4 = 0; v4 < W; ++v4) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(w + (size_t)c0 * W) + v4);
        const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) wt[(4 * v4 + u) % W][(4 * v4 + u) / W] = fv[u];
    }
    // the document holding t0: the last n with cu[n] <= t0 (and t0 < cu[n + 1])
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu + mid) <= t0) lo = mid; else hi = mid - 1;
    }
    int n = lo;
    while (n + 1 < num_seqs && __ldg(cu + n + 1) <= t0) ++n;  // skip empty documents
    int start = __ldg(cu + n), end = __ldg(cu + n + 1);
    // window: the inputs at t0 - (W - 1) .. t0 - 1, from x inside the document, else the state
    float win[W > 1 ? W - 1 : 1][kCh];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
        const int pos = t0 - (W - 1) + j;
        if (pos >= start) {
            Vec4<T>::load(x + (size_t)pos * C + c0, win[j]);
        } else if (st_in) {
            Vec4<T>::load(st_in + ((size_t)n * (W - 1) + (pos - start + W - 1)) * C + c0, win[j]);
        } else {
#pragma unroll
            for (int e = 0; e < kCh; ++e) win[j][e] = 0.f;
        }
    }
#pragma unroll
    for (int r = 0; r < kRun; ++r) {
        if (r >= nrun) break;
        const int t = t0 + r;
        if (t >= end) {  // the next non-empty document starts here: its state is the window
            // (n stays below num_seqs whatever cu holds)
            while (n + 1 < num_seqs && __ldg(cu + n + 1) <= t) ++n;
            start = __ldg(cu + n);
            end = __ldg(cu + n + 1);
            load_state<T, W>(st_in, n, C, c0, win);
        }
        float xv[kCh], out[kCh];
        Vec4<T>::unpack(xr[r], xv);
#pragma unroll
        for (int e = 0; e < kCh; ++e) {
            float acc = wt[W - 1][e] * xv[e];
#pragma unroll
            for (int i = 0; i < W - 1; ++i) acc = fmaf(wt[i][e], win[i][e], acc);
            out[e] = conv_act(acc, SILU);
        }
        Vec4<T>::store(y + (size_t)t * C + c0, out);
#pragma unroll
        for (int j = 0; j + 1 < W - 1; ++j)
#pragma unroll
            for (int e = 0; e < kCh; ++e) win[j][e] = win[j + 1][e];
        if (W > 1) {
#pragma unroll
            for (int e = 0; e < kCh; ++e) win[W > 1 ? W - 2 : 0][e] = xv[e];
        }
        if (st_out && t == end - 1) store_state<T, W>(st_out, n, C, c0, win);
    }
}

// One token per sequence, the state updated in place: thread = (sequence, kCh channels).
template <typename T, int W, bool SILU>
__global__ void __launch_bounds__(kThreads) short_conv_step_kernel(
    const T* __restrict__ x, const float* __restrict__ w, T* state, T* __restrict__ y, int N, int C) {
    const long g = (long)blockIdx.x * kThreads + threadIdx.x;
    const int groups = C / kCh;
    if (g >= (long)N * groups) return;
    const int n = (int)(g / groups), c0 = (int)(g % groups) * kCh;
    float xv[kCh], win[W > 1 ? W - 1 : 1][kCh];
    Vec4<T>::load(x + (size_t)n * C + c0, xv);
    load_state<T, W>(state, n, C, c0, win);  // every read before the write below
    float out[kCh];
#pragma unroll
    for (int e = 0; e < kCh; ++e) {
        float acc = __ldg(w + (size_t)(c0 + e) * W + W - 1) * xv[e];
#pragma unroll
        for (int i = 0; i < W - 1; ++i) acc = fmaf(__ldg(w + (size_t)(c0 + e) * W + i), win[i][e], acc);
        out[e] = conv_act(acc, SILU);
    }
    Vec4<T>::store(y + (size_t)n * C + c0, out);
    if (W > 1) {
#pragma unroll
        for (int j = 0; j + 1 < W - 1; ++j)
#pragma unroll
            for (int e = 0; e < kCh; ++e) win[j][e] = win[j + 1][e];
#pragma unroll
        for (int e = 0; e < kCh; ++e) win[W > 1 ? W - 2 : 0][e] = xv[e];
        store_state<T, W>(state, n, C, c0, win);
    }
}

template <typename T, int W, bool SILU>
cudaError_t launch_varlen_t(const ShortConvArgs& a, cudaStream_t st) {
    const unsigned gx = (unsigned)((a.C / kCh + kThreads - 1) / kThreads);
    const unsigned runs = (unsigned)((a.T + kRun - 1) / kRun);
    const unsigned gy = runs > 0 ? runs : 1;  // T = 0: one row of blocks for the empty documents
    short_conv_varlen_kernel<T, W, SILU><<<dim3(gx, gy), kThreads, 0, st>>>(
        static_cast<const T*>(a.x), a.w, a.cu_seqlens, a.num_seqs, static_cast<const T*>(a.state_in),
        static_cast<T*>(a.state_out), static_cast<T*>(a.y), a.T, a.C);
    return cudaGetLastError();
}

template <typename T, int W, bool SILU>
cudaError_t launch_step_t(const ShortConvArgs& a, cudaStream_t st) {
    const long threads = (long)a.num_seqs * (a.C / kCh);
    const unsigned grid = (unsigned)((threads + kThreads - 1) / kThreads);
    short_conv_step_kernel<T, W, SILU><<<grid, kThreads, 0, st>>>(
        static_cast<const T*>(a.x), a.w, static_cast<T*>(a.state_out), static_cast<T*>(a.y),
        a.num_seqs, a.C);
    return cudaGetLastError();
}

template <typename T, bool SILU>
cudaError_t dispatch_w(const ShortConvArgs& a, bool step, cudaStream_t st) {
#define GDN_CONV_CASE(WW) \
    case WW: return step ? launch_step_t<T, WW, SILU>(a, st) : launch_varlen_t<T, WW, SILU>(a, st);
    switch (a.width) {
        GDN_CONV_CASE(1)
        GDN_CONV_CASE(2)
        GDN_CONV_CASE(3)
        GDN_CONV_CASE(4)
        GDN_CONV_CASE(5)
        GDN_CONV_CASE(6)
        GDN_CONV_CASE(7)
        GDN_CONV_CASE(8)
        default: return cudaErrorInvalidValue;
    }
#undef GDN_CONV_CASE
}

template <typename T>
cudaError_t dispatch_act(const ShortConvArgs& a, bool step, cudaStream_t st) {
    return a.silu ? dispatch_w<T, true>(a, step, st) : dispatch_w<T, false>(a, step, st);
}

}  // namespace

cudaError_t launch_short_conv(const ShortConvArgs& a, bool step, cudaStream_t st) {
    if (!step && a.T == 0 && a.state_out == nullptr) return cudaSuccess;
    if (step && a.num_seqs == 0) return cudaSuccess;
    return a.dtype == GDN_BF16 ? dispatch_act<__nv_bfloat16>(a, step, st)
                               : dispatch_act<float>(a, step, st);
}

}  // namespace gdn
