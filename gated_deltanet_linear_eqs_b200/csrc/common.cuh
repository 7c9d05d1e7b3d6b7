// common.cuh -- small helpers shared by the libgdn kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr float kNormEps = 1e-6f;  // x / sqrt(|x|^2 + eps): the library's reading of "L2 norm"
constexpr float kLog2e = 1.4426950408889634f;  // log2(e): ln x * kLog2e = log2 x

// ---- element conversion -----------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load 4 consecutive elements as floats (8-byte load for bf16, 16-byte for fp32).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ---- gates, eqs. (9)-(10) of the Qwen3.8-Flash-Next summary (picx.dev, "Methodology",
// "1. GDN Hybrid Token Mixing") -------------------------------------------------------------
//   beta_t = sigmoid(b_t),  ln alpha_t = -exp(A) softplus(a_t + b_alpha)
// with a_t = W_alpha x_t and b_t = W_beta x_t given per (token, head) and A (as A_log) and
// b_alpha per head.  The decay stays in log space: the chunked kernels consume ln alpha, and
// exp of it would underflow to 0 for strong decays.
// softplus(x) = ln(1 + e^x) = max(x, 0) + ln(1 + e^-|x|): the second term never overflows.
__device__ __forceinline__ float gate_softplus(float x) {
    return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float gate_log_decay(float a, float A_log, float b_alpha) {
    return -expf(A_log) * gate_softplus(a + b_alpha);
}
__device__ __forceinline__ float gate_sigmoid(float x) { return 1.f / (1.f + expf(-x)); }

// Record the first device-side error in the library's status word (never traps).
__device__ __forceinline__ void record_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace gdn

// ---- self checks ---------------------------------------------------------------------------
// Compiled in where GDN_DEBUG is defined: always in prefill.cu, which defines it itself, and in
// every other source only with -DGDN_DEBUG (libgdn_debug.so).  A failed check records
// (code, detail, block) in the device status words and the guarded access is skipped, so a
// bad index is reported instead of faulting.  Where GDN_DEBUG is undefined every guard is `true`.
namespace gdn {
enum DebugCode {
    DBG_GLOBAL_OOB = 100,   // global index out of the tensor's extent
    DBG_SMEM_OOB = 101,     // shared-memory offset outside the kernel's layout
    DBG_TMEM_OOB = 102,     // TMEM column outside the allocation
    DBG_WAIT = 103          // bounded wait gave up (detail = barrier id * 65536 + chunk)
};
#ifdef GDN_DEBUG
__device__ __forceinline__ bool debug_fail(int* status, int code, long long detail) {
    if (status && atomicCAS(status, 0, code) == 0) {
        status[1] = (int)detail;
        status[2] = (int)(detail >> 32);
        status[3] = (int)blockIdx.x;
    }
    return false;
}
#define GDN_GUARD(cond, status, code, detail) \
    ((cond) || ::gdn::debug_fail((status), (code), (long long)(detail)))
#else
#define GDN_GUARD(cond, status, code, detail) true
#endif
}  // namespace gdn
