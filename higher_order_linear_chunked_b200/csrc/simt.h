// CUDA-core chunk-parallel path (declarations used by the C ABI layer).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

namespace hla {
namespace simt {

// floats in one chunk summary for internal op id `op` at head dim d
size_t summary_floats(int op, int d);
// kernels one forward enqueues (chunk kernel, the scan: one fold launch, or one launch per
// tree level when three summaries do not fit in shared memory, output kernel)
int kernel_launches(int op, bool norm, bool bf16, int d, int T);
// floats of workspace the path needs after the status block
size_t workspace_floats(int op, int d, int BH, int T);
// summary layout helpers for other paths: offsets (in floats) of matrix / vector slots
// (second order: S=0 C=1 R=2 ; m=0 r=1; AHLA: P=0 E=1 Dm=2)
inline size_t mat_offset(int slot, int d) { return (size_t)slot * d * d; }
inline size_t vec_offset(int op, int slot, int d) { return (size_t)(op == 3 ? 6 : op == 1 ? 4 : 3) * d * d + (size_t)slot * d; }
// in-place Blelloch exclusive scan over NCp (power of two) summaries per head
cudaError_t scan(int op, int d, float* sums, int NCp, int BH, cudaStream_t st);
// kernels scan() enqueues
int scan_launches(int NCp);
// enqueue chunk kernel, Blelloch scan levels and output kernel on `st`; `ev` (NULL or
// 4 events) is recorded before the chunk kernel, after it, after the scan, after the output kernel
// allow_tc = false keeps every kernel on the CUDA cores (fp32 FFMA throughout)
cudaError_t forward(int op, bool norm, bool bf16, int d, const void* q, const void* k, const void* v,
                    const float* gamma, float eps, float* o, int BH, int H, int T, float* sums, int* status,
                    cudaStream_t st, cudaEvent_t* ev, bool allow_tc = true);

// Streaming state: one summary (summary_floats(op, d) floats) per head.
// state(): the state of each head after its T tokens (chunk kernel, up-sweep, copy of the
// root) into state_out[BH][summary_floats]; sums is workspace_floats(op, d, BH, T) floats.
cudaError_t state(int op, bool bf16, int d, const void* q, const void* k, const void* v, const float* gamma, int BH,
                  int H, int T, float* sums, float* state_out, cudaStream_t st);
// kernels state() enqueues
int state_launches(int T);
// step(): one token per head ([BH][d] q, k, v): state advanced in place, o [BH][d] written.
cudaError_t step(int op, bool norm, bool bf16, int d, float* state_io, const void* q, const void* k, const void* v,
                 const float* gamma, float eps, int BH, int H, float* o, cudaStream_t st);

// Backward pass of the masked second-order output (no decay, not normalised): dq, dk, dv fp32
// [BH][T][d] for the output gradient dout fp32 [BH][T][d]; ws: backward_workspace_floats floats;
// status: the device status word (a bounded wait that gave up sets it).  bf16 at d = 64 takes
// the tensor-core gradient kernel for its last stage unless fp32_only.
size_t backward_workspace_floats(int d, int BH, int T);
int backward_launches(bool bf16, int d, int T);
cudaError_t backward(bool bf16, int d, const void* q, const void* k, const void* v, const float* dout, float* dq,
                     float* dk, float* dv, int BH, int T, float* ws, int* status, cudaStream_t st,
                     bool fp32_only = false);
// Backward pass of the AHLA output (no decay, not normalised), fp32 on the CUDA cores;
// ws: ahla_backward_workspace_floats floats.
size_t ahla_backward_workspace_floats(int d, int BH, int T);
int ahla_backward_launches(int d, int T);
cudaError_t ahla_backward(bool bf16, int d, const void* q, const void* k, const void* v, const float* dout, float* dq,
                          float* dk, float* dv, int BH, int T, float* ws, cudaStream_t st);
// The same for the ratio-normalised output (two plain forwards, two plain backwards, element-wise
// glue); ws: backward_normalized_workspace_floats floats.
size_t backward_normalized_workspace_floats(int d, int BH, int T);
int backward_normalized_launches(bool bf16, int d, int T);
cudaError_t backward_normalized(bool bf16, int d, const void* q, const void* k, const void* v, const float* dout,
                                float eps, float* dq, float* dk, float* dv, int BH, int T, float* ws, int* status,
                                cudaStream_t st);

}  // namespace simt
}  // namespace hla
