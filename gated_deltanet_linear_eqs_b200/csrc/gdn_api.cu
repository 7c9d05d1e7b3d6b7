// gdn_api.cu -- the C ABI of libgdn.so: argument validation, device checks, dispatch.
//
// Every entry point validates its arguments on the host first and launches nothing when
// they are rejected; see include/gdn.h for the contract of each call.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

// Device status words: kernels record the first device-side error in word 0 (bounded waits
// that ran out); debug builds add the failing check's detail and block in words 1-3.  One set
// per device; its address is looked up once per device.
__device__ int g_device_status[4];

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    bool sm100 = false;
    int* status = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

int current_device_info(DeviceInfo* out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_CUDA;
        }
        d.sm100 = (major == 10);
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_CUDA;
        }
        d.status = static_cast<int*>(p);
        d.ready = true;
    }
    *out = d;
    return d.sm100 ? GDN_OK : GDN_ERR_UNSUPPORTED_DEVICE;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt_ptr(const void* p) { return p == nullptr || aligned16(p); }

int check_dims(int dk, int dv, int dtype) {
    if (dtype != GDN_BF16 && dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (dk != dv || (dk != 64 && dk != 128)) return GDN_ERR_UNSUPPORTED_SHAPE;
    return GDN_OK;
}

int map_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

}  // namespace

extern "C" {

const char* gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: null/misaligned pointer or bad size";
        case GDN_ERR_UNSUPPORTED_SHAPE: return "GDN_ERR_UNSUPPORTED_SHAPE: need dk == dv in {64, 128}";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing or too small";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA: a CUDA call or kernel launch failed";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: a device-side bounded wait ran out";
        case GDN_ERR_UNSUPPORTED_DEVICE: return "GDN_ERR_UNSUPPORTED_DEVICE: needs an sm_100 GPU";
        default: return "GDN_ERR_UNKNOWN";
    }
}

const char* gdn_version(void) { return "gdn-b200 0.1"; }

int gdn_workspace_bytes(int op, int B, int T, int H, int dk, int dv, int num_seqs,
                        size_t* bytes) {
    if (!bytes) return GDN_ERR_INVALID_ARG;
    *bytes = 0;
    if (T < 1 || H < 1 || dk < 1 || dv < 1) return GDN_ERR_INVALID_ARG;
    switch (op) {
        case GDN_OP_PREFILL:
            if (B < 1) return GDN_ERR_INVALID_ARG;
            *bytes = gdn::prefill_workspace(B, T, H, dk, false).total;
            return GDN_OK;
        case GDN_OP_DECODE:
            if (B < 1) return GDN_ERR_INVALID_ARG;
            return GDN_OK;
        case GDN_OP_PREFILL_VARLEN:
            if (num_seqs < 1) return GDN_ERR_INVALID_ARG;
            *bytes = gdn::prefill_workspace(num_seqs, T, H, dk, true).total;
            return GDN_OK;
        case GDN_OP_BACKWARD:
            if (B < 1) return GDN_ERR_INVALID_ARG;
            *bytes = gdn::backward_chunked_workspace_bytes(B, T, H, dk, dv);
            return GDN_OK;
        case GDN_OP_PREFILL_SEGMENTED: {  // num_seqs carries the number of segments
            if (B < 1 || num_seqs < 1) return GDN_ERR_INVALID_ARG;
            const size_t a = gdn::segmented_layout(B, T, H, dk, num_seqs, GDN_BF16).total;
            const size_t f = gdn::segmented_layout(B, T, H, dk, num_seqs, GDN_FP32).total;
            *bytes = a > f ? a : f;
            return GDN_OK;
        }
        case GDN_OP_QSA_SCORES:
            if (num_seqs < 1) return GDN_ERR_INVALID_ARG;
            *bytes = gdn::qsa_workspace_bytes(num_seqs);
            return GDN_OK;
        default:
            return GDN_ERR_INVALID_ARG;
    }
}

}  // extern "C"

namespace {

// The plain and the gated entry points share these bodies; A_log == nullptr is the plain form.
int prefill_dense(const void* q, const void* k, const void* v, const float* alpha,
                  const float* beta, const float* A_log, const float* b_alpha, const float* s0,
                  void* y, float* s_final, int B, int T, int H, int dk, int dv, int dtype,
                  float scale, int l2norm_qk, void* ws, size_t ws_bytes, void* stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(alpha) || !ok_ptr(beta) ||
        !ok_ptr(y) || !ok_opt_ptr(s0) || !ok_opt_ptr(s_final))
        return GDN_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    if (int rc = check_dims(dk, dv, dtype)) return rc;
    if (dtype == GDN_BF16) {
        const size_t need = gdn::prefill_workspace(B, T, H, dk, false).total;
        if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return GDN_ERR_WORKSPACE;
    }
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::PrefillArgs a{q, k, v, alpha, beta, s0, y, s_final, nullptr, B, T, H, dk, dv,
                       dtype, scale, l2norm_qk ? 1 : 0, dev.status, ws, ws_bytes, A_log, b_alpha};
    return map_cuda(gdn::launch_prefill(a, static_cast<cudaStream_t>(stream)));
}

int prefill_varlen(const void* q, const void* k, const void* v, const float* alpha,
                   const float* beta, const float* A_log, const float* b_alpha,
                   const int32_t* cu_seqlens, int num_seqs, const float* s0, void* y,
                   float* s_final, int T, int H, int dk, int dv, int dtype, float scale,
                   int l2norm_qk, void* ws, size_t ws_bytes, void* stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(alpha) || !ok_ptr(beta) ||
        !ok_ptr(y) || cu_seqlens == nullptr || !ok_opt_ptr(s0) || !ok_opt_ptr(s_final))
        return GDN_ERR_INVALID_ARG;
    if (num_seqs < 1 || T < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    if (int rc = check_dims(dk, dv, dtype)) return rc;
    if (dtype == GDN_BF16) {
        const size_t need = gdn::prefill_workspace(num_seqs, T, H, dk, true).total;
        if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return GDN_ERR_WORKSPACE;
    }
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::PrefillArgs a{q, k, v, alpha, beta, s0, y, s_final, cu_seqlens, num_seqs, T, H, dk, dv,
                       dtype, scale, l2norm_qk ? 1 : 0, dev.status, ws, ws_bytes, A_log, b_alpha};
    return map_cuda(gdn::launch_prefill(a, static_cast<cudaStream_t>(stream)));
}

int decode_step(const void* q, const void* k, const void* v, const float* alpha,
                const float* beta, const float* A_log, const float* b_alpha, float* state,
                void* y, int N, int H, int dk, int dv, int dtype, float scale, int l2norm_qk,
                void* stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(alpha) || !ok_ptr(beta) ||
        !ok_ptr(state) || !ok_ptr(y))
        return GDN_ERR_INVALID_ARG;
    if (N < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    if (int rc = check_dims(dk, dv, dtype)) return rc;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::DecodeArgs a{q, k, v, alpha, beta, state, y, N, H, dk, dv, dtype, scale,
                      l2norm_qk ? 1 : 0, A_log, b_alpha};
    return map_cuda(gdn::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

int backward_chunked(const void* q, const void* k, const void* v, const float* alpha,
                     const float* beta, const float* A_log, const float* b_alpha,
                     const float* s0, const void* dy, const float* ds_final, void* dq,
                     void* dk_out, void* dv_out, float* dalpha, float* dbeta, float* dA_log,
                     float* db_alpha, float* ds0, int B, int T, int H, int dk, int dv, int dtype,
                     float scale, int l2norm_qk, void* ws, size_t ws_bytes, void* stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(alpha) || !ok_ptr(beta) ||
        !ok_ptr(dy) || !ok_ptr(dq) || !ok_ptr(dk_out) || !ok_ptr(dv_out) || !ok_ptr(dalpha) ||
        !ok_ptr(dbeta) || !ok_opt_ptr(s0) || !ok_opt_ptr(ds_final) || !ok_opt_ptr(ds0))
        return GDN_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    if (int rc = check_dims(dk, dv, dtype)) return rc;
    const size_t need = gdn::backward_chunked_workspace_bytes(B, T, H, dk, dv);
    if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return GDN_ERR_WORKSPACE;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::BackwardArgs a{q, k, v, alpha, beta, s0, dy, ds_final, dq, dk_out, dv_out, dalpha,
                        dbeta, ds0, B, T, H, dk, dv, dtype, scale, l2norm_qk ? 1 : 0, ws,
                        ws_bytes, dev.status, A_log, b_alpha, dA_log, db_alpha};
    return map_cuda(gdn::launch_backward_chunked(a, static_cast<cudaStream_t>(stream)));
}

bool ok_gate(const float* A_log, const float* b_alpha) { return ok_ptr(A_log) && ok_ptr(b_alpha); }

}  // namespace

extern "C" {

int gdn_prefill(const void* q, const void* k, const void* v, const float* alpha,
                const float* beta, const float* s0, void* y, float* s_final, int B, int T, int H,
                int dk, int dv, int dtype, float scale, int l2norm_qk, void* ws, size_t ws_bytes,
                void* stream) {
    return prefill_dense(q, k, v, alpha, beta, nullptr, nullptr, s0, y, s_final, B, T, H, dk, dv,
                         dtype, scale, l2norm_qk, ws, ws_bytes, stream);
}

int gdn_prefill_gated(const void* q, const void* k, const void* v, const float* a,
                      const float* b, const float* A_log, const float* b_alpha, const float* s0,
                      void* y, float* s_final, int B, int T, int H, int dk, int dv, int dtype,
                      float scale, int l2norm_qk, void* ws, size_t ws_bytes, void* stream) {
    if (!ok_gate(A_log, b_alpha)) return GDN_ERR_INVALID_ARG;
    return prefill_dense(q, k, v, a, b, A_log, b_alpha, s0, y, s_final, B, T, H, dk, dv, dtype,
                         scale, l2norm_qk, ws, ws_bytes, stream);
}

int gdn_prefill_varlen(const void* q, const void* k, const void* v, const float* alpha,
                       const float* beta, const int32_t* cu_seqlens, int num_seqs,
                       const float* s0, void* y, float* s_final, int T, int H, int dk, int dv,
                       int dtype, float scale, int l2norm_qk, void* ws, size_t ws_bytes,
                       void* stream) {
    return prefill_varlen(q, k, v, alpha, beta, nullptr, nullptr, cu_seqlens, num_seqs, s0, y,
                          s_final, T, H, dk, dv, dtype, scale, l2norm_qk, ws, ws_bytes, stream);
}

int gdn_prefill_varlen_gated(const void* q, const void* k, const void* v, const float* a,
                             const float* b, const float* A_log, const float* b_alpha,
                             const int32_t* cu_seqlens, int num_seqs, const float* s0, void* y,
                             float* s_final, int T, int H, int dk, int dv, int dtype, float scale,
                             int l2norm_qk, void* ws, size_t ws_bytes, void* stream) {
    if (!ok_gate(A_log, b_alpha)) return GDN_ERR_INVALID_ARG;
    return prefill_varlen(q, k, v, a, b, A_log, b_alpha, cu_seqlens, num_seqs, s0, y, s_final, T,
                          H, dk, dv, dtype, scale, l2norm_qk, ws, ws_bytes, stream);
}

int gdn_prefill_varlen_prepare(const void* q, const void* k, const void* v, const float* alpha,
                               const float* beta, const int32_t* cu_seqlens, int num_seqs, int T,
                               int H, int dk, int dv, int dtype, float scale, int l2norm_qk,
                               void* ws, size_t ws_bytes, void* stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(alpha) || !ok_ptr(beta) ||
        cu_seqlens == nullptr)
        return GDN_ERR_INVALID_ARG;
    if (num_seqs < 1 || T < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    if (int rc = check_dims(dk, dv, dtype)) return rc;
    if (dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn::prefill_workspace(num_seqs, T, H, dk, true).total;
    if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return GDN_ERR_WORKSPACE;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::PrefillArgs a{q, k, v, alpha, beta, nullptr, nullptr, nullptr, cu_seqlens, num_seqs,
                       T, H, dk, dv, dtype, scale, l2norm_qk ? 1 : 0, dev.status, ws, ws_bytes};
    return map_cuda(gdn::launch_prefill_phase(a, 0, static_cast<cudaStream_t>(stream)));
}

int gdn_prefill_varlen_finish(const void* q, const void* k, const int32_t* cu_seqlens,
                              int num_seqs, const float* s0, void* y, float* s_final, int T,
                              int H, int dk, int dv, int dtype, void* ws, size_t ws_bytes,
                              void* stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(y) || cu_seqlens == nullptr || !ok_opt_ptr(s0) ||
        !ok_opt_ptr(s_final))
        return GDN_ERR_INVALID_ARG;
    if (num_seqs < 1 || T < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    if (int rc = check_dims(dk, dv, dtype)) return rc;
    if (dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn::prefill_workspace(num_seqs, T, H, dk, true).total;
    if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return GDN_ERR_WORKSPACE;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::PrefillArgs a{q, k, nullptr, nullptr, nullptr, s0, y, s_final, cu_seqlens, num_seqs,
                       T, H, dk, dv, dtype, 1.0f, 1, dev.status, ws, ws_bytes};
    return map_cuda(gdn::launch_prefill_phase(a, 1, static_cast<cudaStream_t>(stream)));
}

int gdn_decode_step(const void* q, const void* k, const void* v, const float* alpha,
                    const float* beta, float* state, void* y, int N, int H, int dk, int dv,
                    int dtype, float scale, int l2norm_qk, void* stream) {
    return decode_step(q, k, v, alpha, beta, nullptr, nullptr, state, y, N, H, dk, dv, dtype,
                       scale, l2norm_qk, stream);
}

int gdn_decode_step_gated(const void* q, const void* k, const void* v, const float* a,
                          const float* b, const float* A_log, const float* b_alpha, float* state,
                          void* y, int N, int H, int dk, int dv, int dtype, float scale,
                          int l2norm_qk, void* stream) {
    if (!ok_gate(A_log, b_alpha)) return GDN_ERR_INVALID_ARG;
    return decode_step(q, k, v, a, b, A_log, b_alpha, state, y, N, H, dk, dv, dtype, scale,
                       l2norm_qk, stream);
}

int gdn_backward(const void* q, const void* k, const void* v, const float* alpha,
                 const float* beta, const float* s0, const void* dy, const float* ds_final,
                 void* dq, void* dk_out, void* dv_out, float* dalpha, float* dbeta, float* ds0,
                 int B, int T, int H, int dk, int dv, int dtype, float scale, int l2norm_qk,
                 void* ws, size_t ws_bytes, void* stream) {
    return backward_chunked(q, k, v, alpha, beta, nullptr, nullptr, s0, dy, ds_final, dq, dk_out,
                            dv_out, dalpha, dbeta, nullptr, nullptr, ds0, B, T, H, dk, dv, dtype,
                            scale, l2norm_qk, ws, ws_bytes, stream);
}

int gdn_backward_gated(const void* q, const void* k, const void* v, const float* a,
                       const float* b, const float* A_log, const float* b_alpha, const float* s0,
                       const void* dy, const float* ds_final, void* dq, void* dk_out,
                       void* dv_out, float* da, float* db, float* dA_log, float* db_alpha,
                       float* ds0, int B, int T, int H, int dk, int dv, int dtype, float scale,
                       int l2norm_qk, void* ws, size_t ws_bytes, void* stream) {
    if (!ok_gate(A_log, b_alpha) || !ok_ptr(dA_log) || !ok_ptr(db_alpha))
        return GDN_ERR_INVALID_ARG;
    return backward_chunked(q, k, v, a, b, A_log, b_alpha, s0, dy, ds_final, dq, dk_out, dv_out,
                            da, db, dA_log, db_alpha, ds0, B, T, H, dk, dv, dtype, scale,
                            l2norm_qk, ws, ws_bytes, stream);
}

int gdn_gated_rmsnorm(const void* y, const void* z, const float* w, void* o, int64_t rows,
                      int dv, int dtype, float eps, void* stream) {
    if (rows < 0 || !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    // no rows: nothing is read or written, and the (empty) tensors may be NULL
    const auto ok = [rows](const void* p) { return rows == 0 ? aligned16(p) : ok_ptr(p); };
    if (!ok(y) || !ok(z) || !ok(w) || !ok(o)) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (dv != 64 && dv != 128) return GDN_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::GatedNormArgs a{y, z, w, nullptr, o, nullptr, nullptr, nullptr, (long long)rows, dv,
                         dtype, eps, dev.status};
    return map_cuda(gdn::launch_gated_norm(a, static_cast<cudaStream_t>(stream)));
}

int gdn_gated_rmsnorm_backward(const void* y, const void* z, const float* w, const void* d_o,
                               void* dy, void* dz, float* dw, int64_t rows, int dv, int dtype,
                               float eps, void* stream) {
    if (rows < 0 || !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    // no rows: only dw is written (zeros); the empty row tensors may be NULL
    const auto ok = [rows](const void* p) { return rows == 0 ? aligned16(p) : ok_ptr(p); };
    if (!ok(y) || !ok(z) || !ok(w) || !ok(d_o) || !ok(dy) || !ok(dz) || !ok_ptr(dw))
        return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (dv != 64 && dv != 128) return GDN_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::GatedNormArgs a{y, z, w, d_o, nullptr, dy, dz, dw, (long long)rows, dv, dtype, eps,
                         dev.status};
    return map_cuda(gdn::launch_gated_norm_backward(a, static_cast<cudaStream_t>(stream)));
}

int gdn_backward_noalloc(const void* q, const void* k, const void* v, const float* alpha,
                         const float* beta, const float* s0, const void* dy,
                         const float* ds_final, void* dq, void* dk_out, void* dv_out,
                         float* dalpha, float* dbeta, float* ds0, int B, int T, int H, int dk,
                         int dv, int dtype, float scale, int l2norm_qk, void* stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(alpha) || !ok_ptr(beta) ||
        !ok_ptr(dy) || !ok_ptr(dq) || !ok_ptr(dk_out) || !ok_ptr(dv_out) || !ok_ptr(dalpha) ||
        !ok_ptr(dbeta) || !ok_opt_ptr(s0) || !ok_opt_ptr(ds_final) || !ok_opt_ptr(ds0))
        return GDN_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    if (int rc = check_dims(dk, dv, dtype)) return rc;
    const size_t need = gdn::backward_workspace_bytes(B, T, H, dk, dv);
    if (need > gdn::kBackwardFixedScratchBytes) return GDN_ERR_WORKSPACE;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    void* scratch = nullptr;
    if (int rc = gdn::backward_fixed_scratch(&scratch)) return rc;
    gdn::BackwardArgs a{q, k, v, alpha, beta, s0, dy, ds_final, dq, dk_out, dv_out, dalpha,
                        dbeta, ds0, B, T, H, dk, dv, dtype, scale, l2norm_qk ? 1 : 0, scratch,
                        gdn::kBackwardFixedScratchBytes, dev.status};
    return map_cuda(gdn::launch_backward_tokenloop(a, static_cast<cudaStream_t>(stream)));
}

size_t gdn_backward_noalloc_max_workspace(void) { return gdn::kBackwardFixedScratchBytes; }

static int check_conv(const float* w, int C, int width, int dtype, int activation) {
    if (!ok_ptr(w) || C < 8 || C % 8 != 0 || width < 1 || width > 8) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_FP32) return GDN_ERR_INVALID_ARG;
    if (activation != 0 && activation != 1) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

int gdn_short_conv_varlen(const void* x, const float* w, const int32_t* cu_seqlens,
                          int num_seqs, const void* conv_state_in, void* conv_state_out, void* y,
                          int T, int C, int width, int dtype, int activation, void* stream) {
    if (int rc = check_conv(w, C, width, dtype, activation)) return rc;
    if (T < 0 || num_seqs < 1 || !ok_ptr(cu_seqlens)) return GDN_ERR_INVALID_ARG;
    const auto ok_tok = [T](const void* p) { return T == 0 ? aligned16(p) : ok_ptr(p); };
    if (!ok_tok(x) || !ok_tok(y) || !ok_opt_ptr(conv_state_in) || !ok_opt_ptr(conv_state_out))
        return GDN_ERR_INVALID_ARG;
    if (conv_state_in != nullptr && conv_state_in == conv_state_out) return GDN_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::ShortConvArgs a{x, w, cu_seqlens, num_seqs, conv_state_in, conv_state_out, y, T, C,
                         width, dtype, activation == 1};
    return map_cuda(gdn::launch_short_conv(a, false, static_cast<cudaStream_t>(stream)));
}

int gdn_short_conv_step(const void* x, const float* w, void* conv_state, void* y, int N, int C,
                        int width, int dtype, int activation, void* stream) {
    if (int rc = check_conv(w, C, width, dtype, activation)) return rc;
    if (N < 1 || !ok_ptr(x) || !ok_ptr(y)) return GDN_ERR_INVALID_ARG;
    if (width > 1 ? !ok_ptr(conv_state) : !ok_opt_ptr(conv_state)) return GDN_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::ShortConvArgs a{x, w, nullptr, N, conv_state, conv_state, y, 1, C, width, dtype,
                         activation == 1};
    return map_cuda(gdn::launch_short_conv(a, true, static_cast<cudaStream_t>(stream)));
}

int gdn_qsa_block_scores(const void* q, const void* k, const float* g, const int32_t* cu_seqlens,
                         int num_seqs, int T, int max_doc_len, void* k_hat, int32_t* block_base,
                         float* scores, int ld, void* ws, size_t ws_bytes, void* stream) {
    if (T < 0 || num_seqs < 1 || max_doc_len < 0 || max_doc_len > T) return GDN_ERR_INVALID_ARG;
    if (ld < max_doc_len / 4 || ld % 4 != 0) return GDN_ERR_INVALID_ARG;
    const auto ok_tok = [T](const void* p) { return T == 0 ? aligned16(p) : ok_ptr(p); };
    if (!ok_tok(q) || !ok_tok(k) || !ok_ptr(g) || !ok_ptr(cu_seqlens) || !ok_ptr(block_base) ||
        !ok_tok(scores))
        return GDN_ERR_INVALID_ARG;
    if (T / 4 > 0 ? !ok_ptr(k_hat) : !aligned16(k_hat)) return GDN_ERR_INVALID_ARG;
    if (ws == nullptr || !aligned16(ws) || ws_bytes < gdn::qsa_workspace_bytes(num_seqs))
        return GDN_ERR_WORKSPACE;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::QsaArgs a{q, k, g, cu_seqlens, num_seqs, T, max_doc_len, k_hat, block_base, scores, ld,
                   0, nullptr, dev.status, ws, ws_bytes};
    return map_cuda(gdn::launch_qsa_scores(a, static_cast<cudaStream_t>(stream)));
}

int gdn_qsa_select_blocks(const float* scores, int ld, const int32_t* cu_seqlens, int num_seqs,
                          int T, int budget, int32_t* sel, void* stream) {
    if (T < 0 || num_seqs < 1 || budget < 1 || ld < 0 || ld % 4 != 0) return GDN_ERR_INVALID_ARG;
    const auto ok_tok = [T](const void* p) { return T == 0 ? aligned16(p) : ok_ptr(p); };
    if (!ok_tok(scores) || !ok_tok(sel) || !ok_ptr(cu_seqlens)) return GDN_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::QsaArgs a{nullptr, nullptr, nullptr, cu_seqlens, num_seqs, T, 0, nullptr, nullptr,
                   const_cast<float*>(scores), ld, budget, sel, dev.status, nullptr, 0};
    return map_cuda(gdn::launch_qsa_select(a, static_cast<cudaStream_t>(stream)));
}

int gdn_qsa_indexer(const void* q, const void* k, const float* g, const int32_t* cu_seqlens,
                    int num_seqs, int T, int max_doc_len, int budget, void* k_hat,
                    int32_t* block_base, float* scores, int ld, int32_t* sel, void* ws,
                    size_t ws_bytes, void* stream) {
    if (budget < 1 || (T > 0 && !ok_ptr(sel))) return GDN_ERR_INVALID_ARG;
    if (int rc = gdn_qsa_block_scores(q, k, g, cu_seqlens, num_seqs, T, max_doc_len, k_hat,
                                      block_base, scores, ld, ws, ws_bytes, stream))
        return rc;
    return gdn_qsa_select_blocks(scores, ld, cu_seqlens, num_seqs, T, budget, sel, stream);
}

int gdn_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000ull) return GDN_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    return map_cuda(gdn::launch_wait_timeout_selftest(dev.status, limit_ns,
                                                      static_cast<cudaStream_t>(stream)));
}

int gdn_prefill_segmented(const void* q, const void* k, const void* v, const float* alpha,
                          const float* beta, const float* s0, void* y, float* s_final, int B,
                          int T, int H, int dk, int dv, int dtype, float scale, int l2norm_qk,
                          int num_segments, void* ws, size_t ws_bytes, void* stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(alpha) || !ok_ptr(beta) ||
        !ok_ptr(y) || !ok_opt_ptr(s0) || !ok_opt_ptr(s_final))
        return GDN_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1 || num_segments < 1) return GDN_ERR_INVALID_ARG;
    if (int rc = check_dims(dk, dv, dtype)) return rc;
    const size_t need = gdn::segmented_layout(B, T, H, dk, num_segments, dtype).total;
    if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return GDN_ERR_WORKSPACE;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    gdn::PrefillArgs a{q, k, v, alpha, beta, s0, y, s_final, nullptr, B, T, H, dk, dv,
                       dtype, scale, l2norm_qk ? 1 : 0, dev.status, ws, ws_bytes};
    return map_cuda(gdn::launch_prefill_segmented(a, num_segments,
                                                  static_cast<cudaStream_t>(stream)));
}

int gdn_read_device_status(int reset, int* device_status) {
    if (!device_status) return GDN_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    int h = 0;
    if (cudaMemcpy(&h, dev.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (reset && h != 0) {
        const int zero[4] = {0, 0, 0, 0};
        if (cudaMemcpy(dev.status, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    *device_status = h;
    return GDN_OK;
}

#ifdef GDN_DEBUG
// Debug builds only: the four status words (code, detail low, detail high, block).
int gdn_debug_words(int* out4) {
    if (!out4) return GDN_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (int rc = current_device_info(&dev)) return rc;
    if (cudaMemcpy(out4, dev.status, 4 * sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GDN_ERR_CUDA;
    return GDN_OK;
}
#endif

}  // extern "C"
