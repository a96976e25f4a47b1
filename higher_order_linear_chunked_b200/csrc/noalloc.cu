// Allocation-free entry point: the ratio-normalised second-order forward with its
// scratch in a fixed device array that ships inside this library.
//
// Some callers cannot hand the library a workspace.  Examples: a plugin that runs
// inside another framework's execution callback, where that framework owns all device
// memory and forbids allocating while it runs; a latency-critical serving loop that
// does all of its allocation at start-up, because cudaMalloc/cudaFree can synchronise
// the device and stall other streams; code that must not face an out-of-memory failure
// half way through a request.  For them this file keeps the scratch the path needs in
// `g_scratch`, a file-scope __device__ array of HLA_NOALLOC_SCRATCH_BYTES.  Every GPU
// that loads the library holds that array until the process exits.
//
// Host code cannot use the name `g_scratch` as a device address (on the host it names
// a stand-in object), so the first call on each device asks the runtime for the
// array's device address with cudaGetSymbolAddress, with that device current, and
// caches it.  All calls on a device share the one array and it keeps whatever the last
// call left there; the only part that must start at zero (the status word) is cleared
// by every call.  Two calls whose work overlaps on the GPU (different streams, or
// host threads) race on the shared array: serialise them.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hla.h"

namespace {

__device__ __align__(256) unsigned char g_scratch[HLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per device).
hla_status_t scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HLA_ERR_CUDA;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return HLA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return HLA_OK;
}

}  // namespace

extern "C" hla_status_t hla2_forward_normalized_noalloc(const void* q, const void* k, const void* v, float* o,
                                                        int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                                                        const float* gamma, float eps, void* stream) {
    const size_t need = hla_workspace_bytes(HLA_OP_HLA2_NORM, dtype, gamma != nullptr, B, H, T, d, dv);
    if (need == 0) {
        // invalid or unsupported request: let the regular entry point name the reason
        return hla2_forward_normalized(q, k, v, o, B, H, T, d, dv, dtype, gamma, eps, nullptr, 0, stream);
    }
    if (need > (size_t)HLA_NOALLOC_SCRATCH_BYTES) return HLA_ERR_WORKSPACE;
    void* scratch = nullptr;
    const hla_status_t s = scratch_address(&scratch);
    if (s != HLA_OK) return s;
    return hla2_forward_normalized(q, k, v, o, B, H, T, d, dv, dtype, gamma, eps, scratch,
                                   (size_t)HLA_NOALLOC_SCRATCH_BYTES, stream);
}

// The status word of the last no-alloc call on this device sits at the start of the scratch
// array (where every forward keeps it in its workspace); the regular hla_read_device_status
// reads it from there.
extern "C" hla_status_t hla_noalloc_read_device_status(void* stream, int* device_status) {
    if (!device_status) return HLA_ERR_NULL;
    void* scratch = nullptr;
    const hla_status_t s = scratch_address(&scratch);
    if (s != HLA_OK) return s;
    return hla_read_device_status(scratch, stream, device_status);
}
