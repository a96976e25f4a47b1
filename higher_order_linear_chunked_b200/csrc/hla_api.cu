// C ABI of the HLA forward library: argument checks, workspace sizing, path choice, launches.
// Declarations and the contract of every entry point: include/hla.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hla.h"
#include "common.cuh"
#include "simt.h"
#include "tc.h"

namespace {

constexpr int kAbiVersion = 2;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Request {
    int op;        // internal op id
    bool norm;     // ratio-normalised
    bool bf16;
    int B, H, T, d, dv;
    int seg;       // tensor-core path: chunks per output segment (0 = automatic), read once per call
};

// Shape / dtype checks shared by the size query and the forward calls.
hla_status_t check_shape(hla_dtype_t dtype, int B, int H, int T, int d, int dv) {
    if (dtype != HLA_F32 && dtype != HLA_BF16) return HLA_ERR_DTYPE;
    if (B < 1 || H < 1 || T < 1 || d < 1 || dv < 1) return HLA_ERR_SHAPE;
    if ((long long)B * H * T >= (1LL << 31)) return HLA_ERR_SHAPE;
    if ((long long)B * H > 65535) return HLA_ERR_SHAPE;        // heads are a grid's y extent
    if (d != dv) return HLA_ERR_UNSUPPORTED;
    if (d != 32 && d != 64) return HLA_ERR_UNSUPPORTED;
    return HLA_OK;
}

Request make_request(hla_op_t op, bool decayed, hla_dtype_t dtype, int B, int H, int T, int d, int dv) {
    Request r{};
    r.norm = (op == HLA_OP_HLA2_NORM || op == HLA_OP_AHLA_NORM || op == HLA_OP_HLA3_NORM);
    r.bf16 = (dtype == HLA_BF16);
    if (op == HLA_OP_HLA2 || op == HLA_OP_HLA2_NORM) r.op = decayed ? hla::OP_HLA2D : hla::OP_HLA2;
    else if (op == HLA_OP_AHLA || op == HLA_OP_AHLA_NORM) r.op = decayed ? hla::OP_AHLAD : hla::OP_AHLA;
    else if (op == HLA_OP_HLA2_UNMASKED) r.op = hla::OP_HLA2U;
    else r.op = decayed ? hla::OP_HLA3D : hla::OP_HLA3;
    r.B = B; r.H = H; r.T = T; r.d = d; r.dv = dv;
    r.seg = hla::tc::segment_chunks();
    return r;
}

bool use_tc(const Request& r) {
    return hla::tc::supported(r.op, r.norm, r.bf16, r.d) && hla::tc::fits(r.op, r.norm, r.B * r.H, r.T, r.seg);
}

// Ops with no decayed form.
bool undecayed_only(hla_op_t op) { return op == HLA_OP_HLA2_UNMASKED; }
bool valid_op(hla_op_t op) { return op >= HLA_OP_HLA2 && op <= HLA_OP_HLA3_NORM; }

size_t workspace_for(const Request& r) {
    const int BH = r.B * r.H;
    if (use_tc(r)) return hla::kStatusBytes + hla::tc::workspace_bytes(r.op, r.norm, BH, r.T, r.seg);
    return hla::kStatusBytes + sizeof(float) * hla::simt::workspace_floats(r.op, r.d, BH, r.T);
}

hla_status_t forward(hla_op_t op, const void* q, const void* k, const void* v, float* o, int B, int H, int T,
                     int d, int dv, hla_dtype_t dtype, const float* gamma, float eps, void* workspace,
                     size_t workspace_bytes, void* stream, void* const* phase_events = nullptr) {
    if (!valid_op(op)) return HLA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !o) return HLA_ERR_NULL;
    hla_status_t s = check_shape(dtype, B, H, T, d, dv);
    if (s != HLA_OK) return s;
    if (gamma && undecayed_only(op)) return HLA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return HLA_ERR_ALIGN;
    if (gamma && (reinterpret_cast<uintptr_t>(gamma) & 3u)) return HLA_ERR_ALIGN;
    const Request r = make_request(op, gamma != nullptr, dtype, B, H, T, d, dv);
    if (!workspace) return HLA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HLA_ERR_ALIGN;
    if (workspace_bytes < workspace_for(r)) return HLA_ERR_WORKSPACE;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* status = static_cast<int*>(workspace);
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return HLA_ERR_CUDA;
    char* body = static_cast<char*>(workspace) + hla::kStatusBytes;
    cudaEvent_t* ev = phase_events ? reinterpret_cast<cudaEvent_t*>(const_cast<void**>(phase_events)) : nullptr;
    cudaError_t e;
    if (use_tc(r)) {
        e = hla::tc::forward(r.op, r.norm, q, k, v, gamma, eps, o, B * H, H, T, body, status, st, ev, r.seg);
    } else {
        e = hla::simt::forward(r.op, r.norm, r.bf16, r.d, q, k, v, gamma, eps, o, B * H, H, T,
                               reinterpret_cast<float*>(body), status, st, ev);
    }
    return e == cudaSuccess ? HLA_OK : HLA_ERR_CUDA;
}

// Streaming-state requests: the undecayed second order with bf16 inputs and d = 64 runs on the
// tensor-core summary walker; everything else on the CUDA-core kernels (fp32 state either way).
bool state_on_tc(const Request& r) { return r.op == hla::OP_HLA2 && use_tc(r); }

size_t state_workspace_for(const Request& r) {
    if (state_on_tc(r)) return hla::kStatusBytes + hla::tc::state_workspace_bytes(r.B * r.H, r.T);
    return hla::kStatusBytes + sizeof(float) * hla::simt::workspace_floats(r.op, r.d, r.B * r.H, r.T);
}

}  // namespace

extern "C" {

int hla_abi_version(void) { return kAbiVersion; }

const char* hla_status_str(hla_status_t s) {
    switch (s) {
    case HLA_OK: return "HLA_OK";
    case HLA_ERR_NULL: return "HLA_ERR_NULL: a required pointer is NULL";
    case HLA_ERR_SHAPE: return "HLA_ERR_SHAPE: B, H, T, d or dv out of range";
    case HLA_ERR_ALIGN: return "HLA_ERR_ALIGN: a base address is not 16-byte aligned";
    case HLA_ERR_DTYPE: return "HLA_ERR_DTYPE: unknown dtype";
    case HLA_ERR_UNSUPPORTED: return "HLA_ERR_UNSUPPORTED: no kernel for this (op, dtype, d, dv, gamma)";
    case HLA_ERR_WORKSPACE: return "HLA_ERR_WORKSPACE: workspace missing or too small";
    case HLA_ERR_CUDA: return "HLA_ERR_CUDA: a CUDA call or launch failed";
    case HLA_ERR_TIMEOUT: return "HLA_ERR_TIMEOUT: a kernel's bounded wait ran out";
    }
    return "unknown hla_status_t";
}

size_t hla_workspace_bytes(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv) {
    if (!valid_op(op)) return 0;
    if (check_shape(dtype, B, H, T, d, dv) != HLA_OK) return 0;
    if (decayed && undecayed_only(op)) return 0;
    return workspace_for(make_request(op, decayed != 0, dtype, B, H, T, d, dv));
}

int hla_kernel_launches(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv) {
    if (hla_workspace_bytes(op, dtype, decayed, B, H, T, d, dv) == 0) return 0;
    const Request r = make_request(op, decayed != 0, dtype, B, H, T, d, dv);
    if (use_tc(r)) return hla::tc::kernel_launches(r.op, r.norm, B * H, T, r.seg);
    return hla::simt::kernel_launches(r.op, r.norm, r.bf16, r.d, T);
}

int hla_uses_tensor_cores(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv) {
    if (hla_workspace_bytes(op, dtype, decayed, B, H, T, d, dv) == 0) return 0;
    const Request r = make_request(op, decayed != 0, dtype, B, H, T, d, dv);
    if (use_tc(r)) return 1;
    if (r.norm || r.bf16 || r.d != 32) return 0;
    if (r.op == hla::OP_HLA3) return 2;                       // tcgen05 summaries and output
    if (r.op == hla::OP_HLA2 && (T + 127) / 128 <= hla::tc::hla2f_max_chunks()) return 2;
    return 0;
}

hla_status_t hla2_forward(const void* q, const void* k, const void* v, float* o, int B, int H, int T, int d,
                          int dv, hla_dtype_t dtype, const float* gamma, void* workspace, size_t workspace_bytes,
                          void* stream) {
    return forward(HLA_OP_HLA2, q, k, v, o, B, H, T, d, dv, dtype, gamma, 0.f, workspace, workspace_bytes, stream);
}

hla_status_t hla2_forward_normalized(const void* q, const void* k, const void* v, float* o, int B, int H, int T,
                                     int d, int dv, hla_dtype_t dtype, const float* gamma, float eps,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    return forward(HLA_OP_HLA2_NORM, q, k, v, o, B, H, T, d, dv, dtype, gamma, eps, workspace, workspace_bytes,
                   stream);
}

hla_status_t ahla_forward(const void* q, const void* k, const void* v, float* o, int B, int H, int T, int d,
                          int dv, hla_dtype_t dtype, const float* gamma, void* workspace, size_t workspace_bytes,
                          void* stream) {
    return forward(HLA_OP_AHLA, q, k, v, o, B, H, T, d, dv, dtype, gamma, 0.f, workspace, workspace_bytes, stream);
}

hla_status_t hla3_forward(const void* q, const void* k, const void* v, float* o, int B, int H, int T, int d,
                          int dv, hla_dtype_t dtype, const float* gamma, void* workspace, size_t workspace_bytes,
                          void* stream) {
    return forward(HLA_OP_HLA3, q, k, v, o, B, H, T, d, dv, dtype, gamma, 0.f, workspace, workspace_bytes, stream);
}

hla_status_t ahla_forward_normalized(const void* q, const void* k, const void* v, float* o, int B, int H, int T,
                                    int d, int dv, hla_dtype_t dtype, const float* gamma, float eps,
                                    void* workspace, size_t workspace_bytes, void* stream) {
    return forward(HLA_OP_AHLA_NORM, q, k, v, o, B, H, T, d, dv, dtype, gamma, eps, workspace, workspace_bytes,
                   stream);
}

hla_status_t hla3_forward_normalized(const void* q, const void* k, const void* v, float* o, int B, int H, int T,
                                    int d, int dv, hla_dtype_t dtype, const float* gamma, float eps,
                                    void* workspace, size_t workspace_bytes, void* stream) {
    return forward(HLA_OP_HLA3_NORM, q, k, v, o, B, H, T, d, dv, dtype, gamma, eps, workspace, workspace_bytes,
                   stream);
}

hla_status_t hla2_forward_unmasked(const void* q, const void* k, const void* v, float* o, int B, int H, int T,
                                   int d, int dv, hla_dtype_t dtype, const float* gamma, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    return forward(HLA_OP_HLA2_UNMASKED, q, k, v, o, B, H, T, d, dv, dtype, gamma, 0.f, workspace,
                   workspace_bytes, stream);
}

hla_status_t hla_forward_profiled(hla_op_t op, const void* q, const void* k, const void* v, float* o, int B,
                                  int H, int T, int d, int dv, hla_dtype_t dtype, const float* gamma, float eps,
                                  void* workspace, size_t workspace_bytes, void* stream,
                                  void* const* phase_events) {
    return forward(op, q, k, v, o, B, H, T, d, dv, dtype, gamma, eps, workspace, workspace_bytes, stream,
                   phase_events);
}

size_t hla_state_floats(hla_op_t op, int decayed, int d, int dv) {
    if (!valid_op(op)) return 0;
    if (d != dv || (d != 32 && d != 64)) return 0;
    if (decayed && undecayed_only(op)) return 0;
    return hla::simt::summary_floats(make_request(op, decayed != 0, HLA_F32, 1, 1, 1, d, dv).op, d);
}

size_t hla_state_workspace_bytes(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv) {
    if (hla_workspace_bytes(op, dtype, decayed, B, H, T, d, dv) == 0) return 0;
    return state_workspace_for(make_request(op, decayed != 0, dtype, B, H, T, d, dv));
}

int hla_state_kernel_launches(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv) {
    if (hla_state_workspace_bytes(op, dtype, decayed, B, H, T, d, dv) == 0) return 0;
    if (state_on_tc(make_request(op, decayed != 0, dtype, B, H, T, d, dv))) return 2;
    return hla::simt::state_launches(T);
}

hla_status_t hla_state(hla_op_t op, const void* q, const void* k, const void* v, float* state, int B, int H, int T,
                       int d, int dv, hla_dtype_t dtype, const float* gamma, void* workspace,
                       size_t workspace_bytes, void* stream) {
    if (!valid_op(op)) return HLA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !state) return HLA_ERR_NULL;
    hla_status_t s = check_shape(dtype, B, H, T, d, dv);
    if (s != HLA_OK) return s;
    if (gamma && undecayed_only(op)) return HLA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state)) return HLA_ERR_ALIGN;
    if (gamma && (reinterpret_cast<uintptr_t>(gamma) & 3u)) return HLA_ERR_ALIGN;
    const Request r = make_request(op, gamma != nullptr, dtype, B, H, T, d, dv);
    if (!workspace) return HLA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HLA_ERR_ALIGN;
    if (workspace_bytes < state_workspace_for(r)) return HLA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess) return HLA_ERR_CUDA;
    float* sums = reinterpret_cast<float*>(static_cast<char*>(workspace) + hla::kStatusBytes);
    const cudaError_t e = state_on_tc(r)
                              ? hla::tc::state(q, k, v, B * H, T, sums, static_cast<int*>(workspace), state, st)
                              : hla::simt::state(r.op, r.bf16, d, q, k, v, gamma, B * H, H, T, sums, state, st);
    return e == cudaSuccess ? HLA_OK : HLA_ERR_CUDA;
}

hla_status_t hla_step(hla_op_t op, float* state, const void* q, const void* k, const void* v, float* o, int B, int H,
                      int d, int dv, hla_dtype_t dtype, const float* gamma, float eps, void* stream) {
    if (!valid_op(op)) return HLA_ERR_UNSUPPORTED;
    if (!state || !q || !k || !v || !o) return HLA_ERR_NULL;
    hla_status_t s = check_shape(dtype, B, H, 1, d, dv);
    if (s != HLA_OK) return s;
    if (gamma && undecayed_only(op)) return HLA_ERR_UNSUPPORTED;
    if (!aligned16(state) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return HLA_ERR_ALIGN;
    if (gamma && (reinterpret_cast<uintptr_t>(gamma) & 3u)) return HLA_ERR_ALIGN;
    const Request r = make_request(op, gamma != nullptr, dtype, B, H, 1, d, dv);
    const cudaError_t e = hla::simt::step(r.op, r.norm, r.bf16, d, state, q, k, v, gamma, eps, B * H, H, o,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HLA_OK : HLA_ERR_CUDA;
}

size_t hla_backward_workspace_bytes(hla_op_t op, hla_dtype_t dtype, int B, int H, int T, int d, int dv) {
    if (op != HLA_OP_HLA2 && op != HLA_OP_HLA2_NORM && op != HLA_OP_AHLA) return 0;
    if (check_shape(dtype, B, H, T, d, dv) != HLA_OK) return 0;
    if (op == HLA_OP_AHLA) return hla::kStatusBytes + sizeof(float) * hla::simt::ahla_backward_workspace_floats(d, B * H, T);
    if (op == HLA_OP_HLA2_NORM)
        return hla::kStatusBytes + sizeof(float) * hla::simt::backward_normalized_workspace_floats(d, B * H, T);
    return hla::kStatusBytes + sizeof(float) * hla::simt::backward_workspace_floats(d, B * H, T);
}

int hla_backward_kernel_launches(hla_op_t op, hla_dtype_t dtype, int B, int H, int T, int d, int dv) {
    if (hla_backward_workspace_bytes(op, dtype, B, H, T, d, dv) == 0) return 0;
    if (op == HLA_OP_AHLA) return hla::simt::ahla_backward_launches(d, T);
    return op == HLA_OP_HLA2_NORM ? hla::simt::backward_normalized_launches(dtype == HLA_BF16, d, T)
                                  : hla::simt::backward_launches(dtype == HLA_BF16, d, T);
}

namespace {
hla_status_t backward_call(hla_op_t op, const void* q, const void* k, const void* v, const float* dout, float* dq,
                           float* dk, float* dv_out, int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                           const float* gamma, float eps, void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv_out) return HLA_ERR_NULL;
    hla_status_t s = check_shape(dtype, B, H, T, d, dv);
    if (s != HLA_OK) return s;
    if (gamma) return HLA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv_out))
        return HLA_ERR_ALIGN;
    if (!workspace) return HLA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HLA_ERR_ALIGN;
    if (workspace_bytes < hla_backward_workspace_bytes(op, dtype, B, H, T, d, dv)) return HLA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess) return HLA_ERR_CUDA;
    float* body = reinterpret_cast<float*>(static_cast<char*>(workspace) + hla::kStatusBytes);
    int* status = static_cast<int*>(workspace);
    cudaError_t e;
    if (op == HLA_OP_AHLA)
        e = hla::simt::ahla_backward(dtype == HLA_BF16, d, q, k, v, dout, dq, dk, dv_out, B * H, T, body, st);
    else if (op == HLA_OP_HLA2_NORM)
        e = hla::simt::backward_normalized(dtype == HLA_BF16, d, q, k, v, dout, eps, dq, dk, dv_out, B * H, T, body,
                                           status, st);
    else
        e = hla::simt::backward(dtype == HLA_BF16, d, q, k, v, dout, dq, dk, dv_out, B * H, T, body, status, st);
    return e == cudaSuccess ? HLA_OK : HLA_ERR_CUDA;
}
}  // namespace

hla_status_t hla2_backward(const void* q, const void* k, const void* v, const float* dout, float* dq, float* dk,
                           float* dv_out, int B, int H, int T, int d, int dv, hla_dtype_t dtype, const float* gamma,
                           void* workspace, size_t workspace_bytes, void* stream) {
    return backward_call(HLA_OP_HLA2, q, k, v, dout, dq, dk, dv_out, B, H, T, d, dv, dtype, gamma, 0.f, workspace,
                         workspace_bytes, stream);
}

hla_status_t ahla_backward(const void* q, const void* k, const void* v, const float* dout, float* dq, float* dk,
                           float* dv_out, int B, int H, int T, int d, int dv, hla_dtype_t dtype, const float* gamma,
                           void* workspace, size_t workspace_bytes, void* stream) {
    return backward_call(HLA_OP_AHLA, q, k, v, dout, dq, dk, dv_out, B, H, T, d, dv, dtype, gamma, 0.f, workspace,
                         workspace_bytes, stream);
}

hla_status_t hla2_backward_normalized(const void* q, const void* k, const void* v, const float* dout, float* dq,
                                      float* dk, float* dv_out, int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                                      const float* gamma, float eps, void* workspace, size_t workspace_bytes,
                                      void* stream) {
    return backward_call(HLA_OP_HLA2_NORM, q, k, v, dout, dq, dk, dv_out, B, H, T, d, dv, dtype, gamma, eps, workspace,
                         workspace_bytes, stream);
}

hla_status_t hla_set_segment_chunks(int chunks) {
    return hla::tc::set_segment_chunks(chunks) ? HLA_OK : HLA_ERR_SHAPE;
}

hla_status_t hla_read_device_status(const void* workspace, void* stream, int* device_status) {
    if (!workspace || !device_status) return HLA_ERR_NULL;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HLA_ERR_CUDA;
    int s = 0;
    if (cudaMemcpy(&s, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return HLA_ERR_CUDA;
    *device_status = s;
    return HLA_OK;
}

hla_status_t hla_selftest_umma(int layout_case, const void* a, const void* b, float* d, int N, int K,
                               void* stream) {
    if (!a || !b || !d) return HLA_ERR_NULL;
    if (layout_case < 0 || layout_case > 31 || (layout_case & 8 && !(layout_case & 4))) return HLA_ERR_UNSUPPORTED;
    if ((layout_case & 16) && (layout_case & 14)) return HLA_ERR_UNSUPPORTED;   // A in TMEM: M = 128, K-major
    if ((N != 64 && N != 128 && N != 192 && N != 256) || (K != 64 && K != 128)) return HLA_ERR_SHAPE;
    if (!aligned16(a) || !aligned16(b) || !aligned16(d)) return HLA_ERR_ALIGN;
    cudaError_t e = hla::tc::selftest(layout_case, a, b, d, N, K, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HLA_OK : HLA_ERR_CUDA;
}

hla_status_t hla_selftest_wait_timeout(void* workspace, size_t workspace_bytes, unsigned timeout_us, void* stream) {
    if (!workspace) return HLA_ERR_NULL;
    if (!aligned16(workspace)) return HLA_ERR_ALIGN;
    if (workspace_bytes < hla::kStatusBytes) return HLA_ERR_WORKSPACE;
    if (timeout_us < 1 || timeout_us > 1000000) return HLA_ERR_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* status = static_cast<int*>(workspace);
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return HLA_ERR_CUDA;
    const cudaError_t e = hla::tc::selftest_wait_timeout(status, timeout_us, st);
    return e == cudaSuccess ? HLA_OK : HLA_ERR_CUDA;
}

}  // extern "C"
