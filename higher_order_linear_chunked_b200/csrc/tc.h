// tcgen05 (5th-generation tensor core) path: declarations used by the C ABI layer.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

namespace hla {
namespace tc {

// true when (internal op, normalised, bf16, d) runs on the tcgen05 kernels
bool supported(int op, bool norm, bool bf16, int d);
// and for this shape: the decayed AHLA walk needs its prefix folded into the output walker
bool fits(int op, bool norm, int BH, int T, int seg_chunks);
// process-wide default segment length (chunks); 0 = automatic; false if invalid
bool set_segment_chunks(int chunks);
// the default, read once by every request (the size query and the forward each take their own
// reading, and each call plans with the value it read)
int segment_chunks();
// kernels one forward enqueues (seg_chunks: the request's segment length)
int kernel_launches(int op, bool norm, int BH, int T, int seg_chunks);
// workspace bytes the path needs after the status block
size_t workspace_bytes(int op, bool norm, int BH, int T, int seg_chunks);
// enqueue the forward (summaries, prefixes, output); gamma: device [H] decay factors or null
cudaError_t forward(int op, bool norm, const void* q, const void* k, const void* v, const float* gamma, float eps,
                    float* o, int BH, int H, int T, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev,
                    int seg_chunks);
// streaming state (second order, bf16, d = 64): the summary walker over every chunk of every
// head, then each head's segments combined into state_out [BH][summary floats]; two launches
size_t state_workspace_bytes(int BH, int T);
cudaError_t state(const void* q, const void* k, const void* v, int BH, int T, void* ws, int* status, float* state_out,
                  cudaStream_t st);
// the carried state at every 128-token chunk (second order, bf16, d = 64): the summary walker
// over one-chunk segments into sums, then the segment-prefix kernels into pre; both
// [BH][next_pow2(chunks)][summary floats] (chunk_prefix_floats each); four launches
size_t chunk_prefix_floats(int BH, int T);
cudaError_t chunk_prefixes(const void* q, const void* k, const void* v, int BH, int T, float* sums, float* pre,
                           int* status, cudaStream_t st);
// backward of the masked second order (bf16, d = 64), 128-token chunks, slots
// [BH][next_pow2(chunks)][3 d d] (fp32):
//   bwd_terms: Y = Q^T dO, U = Q^T (dW Q), C = Q^T V of every chunk into its slot [Y | U | C];
//   bwd_out:   dq, dk, dv of every chunk from the exclusive prefixes of chunk_prefixes (pre) and
//              the slots after the suffix sums (bw: dR', dS')
cudaError_t bwd_terms(const void* q, const void* v, const float* dout, float* terms, int BH, int T, int* status,
                      cudaStream_t st);
cudaError_t bwd_out(const void* q, const void* k, const void* v, const float* dout, const float* pre,
                    const float* bw, float* dq, float* dk, float* dv, int BH, int T, int* status,
                    cudaStream_t st);
// the third order (fp32 q, k, v, d = dv = 32, plain) on tcgen05 from two- and three-term bf16
// splits, 128-token chunks: hla3_summaries writes chunk l's summary of head bh to
// sums + (bh NC + l) slot_floats in the CUDA-core slot layout (the factored prefix then runs in
// place over NC slots per head, NCp = NC); hla3_output reads the exclusive prefix of chunk l at
// sums + (bh NCp + l) slot_floats (S0, P0, F0 at matrices 0, 2, 3) as a programmatic dependent
cudaError_t hla3_summaries(const float* q, const float* k, const float* v, float* sums, int NC, int slot_floats,
                           int BH, int T, int* status, cudaStream_t st);
cudaError_t hla3_output(const float* q, const float* k, const float* v, const float* sums, int NCp, int slot_floats,
                        float* o, int BH, int T, int* status, cudaStream_t st);
// the plain second order (fp32 q, k, v, d = dv = 32) on tcgen05 from two- and three-term bf16
// splits, 128-token chunks, for at most hla2f_max_chunks() chunks per head: the chunk summaries
// into sums ([BH][chunks][slot_floats], the CUDA-core slot layout), then the output with each
// CTA folding the summaries before its chunk; two launches, ev as for forward()
int hla2f_max_chunks();
cudaError_t hla2f_forward(const float* q, const float* k, const float* v, float* sums, int slot_floats, float* o,
                          int BH, int T, int* status, cudaStream_t st, cudaEvent_t* ev);
// one tcgen05 MMA on one CTA (layout self-check; see hla_selftest_umma in include/hla.h)
cudaError_t selftest(int layout_case, const void* a, const void* b, float* d, int N, int K, cudaStream_t st);
// a bounded wait that runs out (see hla_selftest_wait_timeout in include/hla.h)
cudaError_t selftest_wait_timeout(int* status, unsigned timeout_us, cudaStream_t st);

}  // namespace tc
}  // namespace hla
