// CUDA-core chunk-parallel path (declarations used by the C ABI layer).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

namespace hla {
namespace simt {

// floats in one chunk summary for internal op id `op` at head dim d
size_t summary_floats(int op, int d);
// kernels one forward enqueues (chunk kernel, scan levels, output kernel)
int kernel_launches(int T);
// floats of workspace the path needs after the status block
size_t workspace_floats(int op, int d, int BH, int T);
// enqueue chunk kernel, Blelloch scan levels and output kernel on `st`; `ev` (NULL or
// 4 events) is recorded before the chunk kernel, after it, after the scan, after the output kernel
cudaError_t forward(int op, bool norm, bool bf16, int d, const void* q, const void* k, const void* v,
                    const float* gamma, float eps, float* o, int BH, int H, int T, float* sums,
                    cudaStream_t st, cudaEvent_t* ev);

}  // namespace simt
}  // namespace hla
