// Shared device/host helpers of the HLA CUDA library (no arithmetic of the method here).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hla {

// Internal operation ids (the C ABI maps its hla_op_t + gamma onto these).
enum Op : int {
    OP_HLA2 = 0,   // second order, undecayed (normalised or not: template flag)
    OP_HLA2D = 1,  // second order with per-head decay
    OP_AHLA = 2,
    OP_HLA3 = 3,
    OP_HLA2U = 4,  // second order without the inner mask (o_t = q_t^T S_t C_t)
    OP_AHLAD = 5,  // AHLA with per-head decay
    OP_HLA3D = 6,  // third order with per-head decay
};

// Device status word values (first int of every workspace).
enum DevStatus : int { DEV_OK = 0, DEV_ALIGN = 3, DEV_TIMEOUT = 8 };

// Bytes reserved at the start of every workspace for the status word.
constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, DEV_OK, code);
}

}  // namespace hla
