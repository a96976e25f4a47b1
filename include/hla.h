/*
 * hla.h - C ABI of the B200 (sm_100a) masked Higher-order Linear Attention forward.
 *
 * The operations are those of "Resumen Técnico: Atención Lineal de Orden
 * Superior (HLA)" (gist.science, paper 2510.27258):
 *
 *   hla2_forward            Metodología 1: second-order masked output
 *                           o_t = q_t^T (S^K_t C^QV_t - G_t)
 *                               = sum_{j<=t} sum_{i<=j} (q_t.k_i)(q_j.k_i) v_j.
 *                           With gamma != NULL: the masked operator with
 *                           exponential decay (Contribuciones 2), read as "every
 *                           prefix state is multiplied by gamma_h before each
 *                           token's update".
 *   hla2_forward_normalized Metodología 1, "Normalización": the same numerator
 *                           divided by q_t^T (S^K_t m^Q_t - h_t) + eps.
 *   ahla_forward            Metodología 2: AHLA, Q (K^T Q)(K^T V), masked:
 *                           o_t = sum_{j<=t} (q_t.k_j) sum_{i<=j} (q_j.k_i) v_i.
 *   hla3_forward            Metodología 3: third order A A^T A, masked:
 *                           O = (M A) V, M = L (.) (A A^T), A = L (.) Q K^T.
 *   ahla_forward_normalized Metodología 2 lists the AHLA summaries (P^KV, m^K,
 *   hla3_forward_normalized E, n): the ratio-normalised AHLA divides by the same
 *                           masked operator on a ones value column,
 *                           q_t^T n_t + eps; the third order likewise.
 *   hla2_forward_unmasked   Contribuciones 2, the unmasked configuration: the
 *                           naive product the cross summary G_t corrects,
 *                           o_t = q_t^T S^K_t C^QV_t
 *                               = sum_{j<=t} sum_{i<=t} (q_t.k_i)(q_j.k_i) v_j.
 *
 * The mask L includes the diagonal (j <= t).  Every operator is computed with
 * the chunk-parallel scheme of Metodología 4: per-segment summaries, an
 * exclusive scan with the semidirect-product combine, and a per-chunk output
 * pass that applies each chunk's carried-in prefix.  The scan is a factored
 * segment prefix on the tensor-core path, and a per-head fold or the Blelloch
 * tree (the page's form) on the CUDA-core path; all give the same prefixes.
 *
 * Layout.  q, k: [B][H][T][d]; v: [B][H][T][dv]; o: [B][H][T][dv], contiguous
 * row-major.  q, k, v are fp32 (HLA_F32) or bf16 (HLA_BF16), all three the same
 * type; o is always fp32.  gamma, when given, is fp32 [H], shared across B,
 * each value in (0, 1].  Base addresses must be 16-byte aligned.
 *
 * Supported shapes.  d == dv, d in {32, 64}, HLA_F32 or HLA_BF16, every op.
 * The tcgen05 tensor-core kernels run bf16 d == 64 hla2 (with or without decay),
 * hla2_normalized (without decay) and ahla (plain, normalised, decayed), and
 * fp32 d == 32 hla3 and hla2 (plain; hla2 up to 64 chunks of 128 tokens per
 * head); every other case runs on the CUDA cores (hla_uses_tensor_cores says
 * which).  T >= 1 (any value; the tail chunk is padded), B, H >= 1,
 * B*H <= 65535 (the heads are a grid dimension), B*H*T < 2^31.  Anything else
 * returns HLA_ERR_UNSUPPORTED or HLA_ERR_SHAPE before any launch.
 *
 * Memory ownership.  Every pointer (q, k, v, o, gamma, workspace) is DEVICE
 * memory owned by the caller.  The library never allocates or frees device
 * memory and keeps no pointer after a call returns.  The workspace holds the
 * segment summaries, the scanned prefixes and a device status word; size it
 * with hla_workspace_bytes() for the same (op, dtype, decayed, B, H, T, d, dv).
 *
 * Execution.  Work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 * default stream) and the call returns without synchronising.  Calls that share
 * a workspace must not overlap on the device.
 *
 * Errors.  Status codes only: nothing aborts, throws or traps.  Argument errors
 * are found on the host before anything is enqueued.  A failed launch returns
 * HLA_ERR_CUDA.  Kernels that wait on a barrier give up after a bounded time,
 * set the device status word and return; hla_read_device_status() fetches it.
 */
#ifndef HLA_H_
#define HLA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HLA_OK = 0,
    HLA_ERR_NULL = 1,        /* a required pointer is NULL */
    HLA_ERR_SHAPE = 2,       /* B, H, T, d or dv out of range, or d != dv */
    HLA_ERR_ALIGN = 3,       /* a base address is not 16-byte aligned */
    HLA_ERR_DTYPE = 4,       /* unknown hla_dtype_t */
    HLA_ERR_UNSUPPORTED = 5, /* valid request this build has no kernel for */
    HLA_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than hla_workspace_bytes() */
    HLA_ERR_CUDA = 7,        /* a CUDA runtime call or launch failed */
    HLA_ERR_TIMEOUT = 8      /* device status: a kernel's bounded wait ran out */
} hla_status_t;

typedef enum { HLA_F32 = 0, HLA_BF16 = 1 } hla_dtype_t;

typedef enum {
    HLA_OP_HLA2 = 0,       /* hla2_forward */
    HLA_OP_HLA2_NORM = 1,  /* hla2_forward_normalized */
    HLA_OP_AHLA = 2,       /* ahla_forward */
    HLA_OP_HLA3 = 3,       /* hla3_forward */
    HLA_OP_HLA2_UNMASKED = 4, /* hla2_forward_unmasked */
    HLA_OP_AHLA_NORM = 5,  /* ahla_forward_normalized */
    HLA_OP_HLA3_NORM = 6   /* hla3_forward_normalized */
} hla_op_t;

/* Version of this ABI (bumped on any signature change or addition; 2 added the unmasked and
 * ratio-normalised AHLA / third-order ops and the streaming-state calls). */
int hla_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* hla_status_str(hla_status_t status);

/*
 * Bytes of device workspace one call needs, or 0 when the request is invalid
 * or unsupported.  decayed: nonzero when gamma will be passed (every op but the unmasked one).
 */
size_t hla_workspace_bytes(hla_op_t op, hla_dtype_t dtype, int decayed,
                           int B, int H, int T, int d, int dv);

/* Second-order masked forward (Metodología 1; decay: Contribuciones 2).
 * gamma: device fp32 [H], or NULL for no decay. */
hla_status_t hla2_forward(const void* q, const void* k, const void* v, float* o,
                          int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                          const float* gamma, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Ratio-normalised second-order masked forward (Metodología 1, Normalización):
 * o_t = num_t / (den_t + eps), den_t = q_t^T (S^K_t m^Q_t - h_t). */
hla_status_t hla2_forward_normalized(const void* q, const void* k, const void* v, float* o,
                                     int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                                     const float* gamma, float eps,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* AHLA masked forward (Metodología 2).  gamma: device fp32 [H] or NULL.  With gamma
 * (Contribuciones 2's decayed operators; the page gives no formula, the reading is the second
 * order's: P and E scaled by gamma_h before each token's update), the output is
 * o_t = sum_{j<=t} sum_{i<=j} gamma^(t-i) (q_t.k_j)(q_j.k_i) v_i, on CUDA-core kernels. */
hla_status_t ahla_forward(const void* q, const void* k, const void* v, float* o,
                          int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                          const float* gamma, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Third-order masked forward (Metodología 3).  gamma: device fp32 [H] or NULL.  With gamma
 * (same reading: S, P and F scaled by gamma_h before each token's update) the output is
 * O = (L (.) (At A^T)) (At V) with At_tj = gamma^(t-j) A_tj, on CUDA-core kernels. */
hla_status_t hla3_forward(const void* q, const void* k, const void* v, float* o,
                          int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                          const float* gamma, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Ratio-normalised AHLA and third-order forwards: the output divided by the same masked
 * operator applied to a ones value column, plus eps (for AHLA, q_t^T n_t with the named
 * summaries m^K = sum k and n_t = sum_j k_j (q_j^T m^K_j)).  gamma: NULL, or device fp32 [H] for
 * the decayed operator (divided by the decayed operator on ones).  CUDA-core kernels for every
 * dtype and d. */
hla_status_t ahla_forward_normalized(const void* q, const void* k, const void* v, float* o,
                                     int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                                     const float* gamma, float eps,
                                     void* workspace, size_t workspace_bytes, void* stream);
hla_status_t hla3_forward_normalized(const void* q, const void* k, const void* v, float* o,
                                     int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                                     const float* gamma, float eps,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* Unmasked second-order forward, o_t = q_t^T S^K_t C^QV_t (Contribuciones 2, the unmasked
 * configuration).  gamma must be NULL.  CUDA-core kernels for every dtype and d. */
hla_status_t hla2_forward_unmasked(const void* q, const void* k, const void* v, float* o,
                                   int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                                   const float* gamma, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * Same computation as the four entry points above, selected by `op`, with
 * timing hooks: when `phase_events` is non-NULL it points to four cudaEvent_t
 * handles (created by the caller, timing enabled) that are recorded on
 * `stream` before the segment-summary kernel, after it, after the scan, and
 * after the output kernel.  gamma as for the op's own entry point; eps is used
 * by the ratio-normalised ops only.
 */
hla_status_t hla_forward_profiled(hla_op_t op, const void* q, const void* k, const void* v, float* o,
                                  int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                                  const float* gamma, float eps, void* workspace,
                                  size_t workspace_bytes, void* stream, void* const* phase_events);

/*
 * Number of kernel launches one forward call of this request enqueues
 * (summary kernel + scan levels + output kernel), or 0 when the request is
 * invalid or unsupported.  Same arguments as hla_workspace_bytes().
 */
int hla_kernel_launches(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv);

/*
 * 1 when this request runs on the tcgen05 tensor-core kernels, 2 when it takes
 * the fp32-input tensor-core kernels that get fp32 accuracy from products of
 * two- and three-term bf16 splits (the plain third order at d = 32: summaries
 * and output, with the prefix between them on the CUDA cores; the plain second
 * order at d = 32 with at most 64 chunks of 128 tokens per head: summaries and
 * output, the prefix folded into the output kernel), 0 when
 * it runs on the CUDA-core (fp32 FFMA) kernels or is invalid.  Same arguments
 * as hla_workspace_bytes().
 */
int hla_uses_tensor_cores(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv);

/*
 * Streaming state (decoding one token at a time after a prefill).
 *
 * The pages give every operator both as a masked sum and as a streaming
 * recurrence with an O(1)-per-token state (Metodología 1-3), and build the
 * chunked scan on segment summaries that concatenate (Metodología 4).  A head's
 * state after t tokens is the summary of those t tokens: the recurrence's state
 * reached from zero, plus the maps the combine needs.  Layout, per head, fp32,
 * hla_state_floats() floats: n matrices of d x d (row-major), then vectors of
 * d, then one scalar, padded to a multiple of 32 floats:
 *   second order          S = sum k k^T, C = sum q v^T, R = S C - G;  m = sum q,
 *                         r = S m - h          (o_t = q_t^T R_t, den = q_t^T r_t)
 *   second order, decayed S, C, G, Khat = sum k k^T (undecayed);  m, h;  rho =
 *                         gamma^t              (o_t = q_t^T (S_t C_t - G_t))
 *   AHLA                  P = sum k v^T, E, D = sum k q^T;  m^K = sum k, n
 *                         (o_t = q_t^T E_t, den_t = q_t^T n_t); decayed: P, E, m^K, n
 *                         decay, D does not; then rho = gamma^t
 *   third order           S, Q2 = sum q q^T, P, F, X, Z;  m^K, X1, F1 (X and F with v
 *                         replaced by 1)     (o_t = q_t^T F_t, den_t = q_t^T F1_t);
 *                         decayed: S, P, F, m^K, F1 decay, Q2 weights token s by
 *                         gamma^(s+1), X, Z, X1 do not; then rho = gamma^t
 *   unmasked second order S, C                                 (o_t = q_t^T S_t C_t)
 * A state of zero tokens is all zeros, except rho = 1 for the decayed form.
 * The state of a ratio-normalised op is that of its plain op.
 */

/* Floats of one head's state, or 0 when (op, decayed, d, dv) is invalid or unsupported
 * (the unmasked second order has no decayed form). */
size_t hla_state_floats(hla_op_t op, int decayed, int d, int dv);

/* Workspace bytes hla_state() needs, or 0 when the request is invalid or unsupported.
 * Same arguments as hla_workspace_bytes(). */
size_t hla_state_workspace_bytes(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv);

/* Kernels one hla_state() call enqueues (chunk kernel, up-sweep levels, copy), or 0. */
int hla_state_kernel_launches(hla_op_t op, hla_dtype_t dtype, int decayed, int B, int H, int T, int d, int dv);

/*
 * Prefill: the state of every head after its T tokens, written to state
 * [B*H][hla_state_floats] (device, fp32, 16-byte aligned, caller-owned).
 * q, k, v, gamma, shapes and dtypes as for the forward calls.  The undecayed
 * second order (plain or ratio-normalised) with bf16 inputs and d = dv = 64 runs
 * the tensor-core summary walker over segments of every head, then one CTA per
 * head combines the segment summaries (two launches).  Everything else runs the
 * CUDA-core chunk-summary kernel and the up-sweep half of the Blelloch scan,
 * whose root is the summary of the whole sequence.  Workspace: at least
 * hla_state_workspace_bytes().  Errors as for the forward calls.
 */
hla_status_t hla_state(hla_op_t op, const void* q, const void* k, const void* v, float* state,
                       int B, int H, int T, int d, int dv, hla_dtype_t dtype, const float* gamma,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode: one token per head.  q, k, v: [B][H][d] (device, HLA_F32 or HLA_BF16,
 * 16-byte aligned); o: [B][H][dv] fp32.  Advances state [B*H][hla_state_floats]
 * in place by the recurrence's update and writes each head's o_t (divided by
 * den_t + eps for HLA_OP_HLA2_NORM).  gamma: as for the forward calls; the state
 * must be of the matching (decayed or not) form.  One kernel launch, no
 * workspace.  Argument errors as for the forward calls (T is 1).
 */
hla_status_t hla_step(hla_op_t op, float* state, const void* q, const void* k, const void* v, float* o,
                      int B, int H, int d, int dv, hla_dtype_t dtype, const float* gamma, float eps,
                      void* stream);

/*
 * Backward pass (gradients) of the masked second-order output, plain form
 * ("Higher-order Linear Attention" summary, gist.science 2510.27258: Metodología 4
 * and Contribuciones 2 present the exact chunked scan as the basis of exact
 * parallel training; the page prints no gradient, these are reverse-mode
 * derivatives of O = (L (.) (A A^T)) V, A = L (.) Q K^T).
 *
 * hla_backward_workspace_bytes: device workspace bytes the backward call of op
 * needs for (dtype, B, H, T, d, dv); 0 when the request is invalid or has no
 * backward kernel (HLA_OP_HLA2, HLA_OP_HLA2_NORM and HLA_OP_AHLA, undecayed, d = dv in
 * {32, 64}).
 *
 * hla2_backward: given the output gradient dout [B][H][T][dv] (fp32, device),
 * writes dq, dk [B][H][T][d] and dv_out [B][H][T][dv] (fp32, device, caller-
 * owned, 16-byte aligned) for the forward hla2_forward(q, k, v) of the same
 * inputs (HLA_F32 or HLA_BF16).  The forward's carried chunk states are
 * recomputed from q, k, v (no saved activations).  Kernels: the carried states,
 * per-chunk adjoint terms, two suffix sums and the per-chunk gradients (see
 * hla_backward_kernel_launches).  Arithmetic: fp32 on the CUDA cores, except
 * for HLA_BF16 at d = 64, where the carried states come from the tensor-core
 * summary walker and the per-chunk gradients from a tensor-core kernel with
 * bf16 operands and fp32 accumulation (dout and the intermediate dZ enter as
 * two bf16 terms each); its gradient carries about 2e-3 of the gradient's norm
 * as rounding.  Errors as for the forward calls; a non-NULL gamma is
 * HLA_ERR_UNSUPPORTED.  Enqueued on `stream`, asynchronous.
 */
size_t hla_backward_workspace_bytes(hla_op_t op, hla_dtype_t dtype, int B, int H, int T, int d, int dv);
int hla_backward_kernel_launches(hla_op_t op, hla_dtype_t dtype, int B, int H, int T, int d, int dv);
hla_status_t hla2_backward(const void* q, const void* k, const void* v, const float* dout, float* dq,
                           float* dk, float* dv_out, int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                           const float* gamma, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass of the AHLA output, O = A (A V), A = L (.) Q K^T (Metodología 2; reverse-mode
 * derivatives of the masked form).  Same arguments, layouts, workspace query
 * (hla_backward_workspace_bytes(HLA_OP_AHLA, ...)), errors and stream semantics as
 * hla2_backward.  fp32 on the CUDA cores for every dtype and d: the forward's carried (P0, E0)
 * per 64-token chunk, the adjoint terms Q^T dO, Q^T (A^T dO), Q^T K per chunk, two suffix sums
 * (dE', dP') with their cross term, and the per-chunk gradients.
 */
hla_status_t ahla_backward(const void* q, const void* k, const void* v, const float* dout, float* dq,
                           float* dk, float* dv_out, int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                           const float* gamma, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass of the ratio-normalised second order, o = num / (den + eps) (Metodología 1,
 * Normalización), same arguments as hla2_backward plus eps (as passed to the forward).  The
 * denominator is the same masked operator on a ones value column, so the gradient is the plain
 * backward with dout / (den + eps), plus the plain backward on the ones column with the per-row
 * output gradient -sum_f dout_f num_f / (den + eps)^2 (its dq and dk).  num and den are
 * recomputed by two plain forwards; both backward passes keep the fp32 gradient kernel (their
 * dq and dk terms nearly cancel where o barely depends on q, k).  Workspace: hla_backward_workspace_bytes(
 * HLA_OP_HLA2_NORM, ...), about 8 B*H*T*d floats more than the plain backward's.
 */
hla_status_t hla2_backward_normalized(const void* q, const void* k, const void* v, const float* dout, float* dq,
                                      float* dk, float* dv_out, int B, int H, int T, int d, int dv,
                                      hla_dtype_t dtype, const float* gamma, float eps, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * Tuning knob of the tensor-core path: chunks of 128 tokens per segment (the
 * unit one CTA walks).  0 restores the automatic choice.  Values outside
 * {0, 1, 2, 4, 8, 16} return HLA_ERR_SHAPE.  A process-wide default held in
 * an atomic: every call (the size query and each forward) reads it once and
 * plans with that one value, so a call never mixes two settings.  It changes
 * hla_workspace_bytes(): a forward whose own reading needs more workspace
 * than the caller passed returns HLA_ERR_WORKSPACE before any launch.
 * Results do not depend on it beyond rounding.
 */
hla_status_t hla_set_segment_chunks(int chunks);

/*
 * Synchronises `stream` and copies the device status word of the last call
 * that used `workspace` into *device_status (HLA_OK, or HLA_ERR_TIMEOUT when a
 * bounded wait ran out).  Returns HLA_ERR_CUDA if the copy fails.
 */
hla_status_t hla_read_device_status(const void* workspace, void* stream, int* device_status);

/*
 * Size of the device scratch array built into the library for
 * hla2_forward_normalized_noalloc(): 64 MiB, held on every GPU that loads
 * the library until the process exits.
 */
#define HLA_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * hla2_forward_normalized() for callers that cannot supply a workspace
 * (the paper has no counterpart; this is a deployment convenience).
 *
 * Who needs it: code that may not allocate device memory while it runs, such
 * as a plugin executing inside another framework that owns the device memory,
 * or a serving loop that allocates everything at start-up because cudaMalloc
 * and cudaFree can synchronise the device and stall unrelated streams.
 *
 * Same arguments and result as hla2_forward_normalized() minus the workspace:
 * the scratch lives in a fixed array of HLA_NOALLOC_SCRATCH_BYTES inside the
 * library.  The call allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library routine).  A request whose hla_workspace_bytes() exceeds
 * HLA_NOALLOC_SCRATCH_BYTES returns HLA_ERR_WORKSPACE before anything is
 * enqueued.  The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  All calls on a device share the one array:
 * calls whose work overlaps on the GPU race and must be serialised by the
 * caller.  The array keeps the last call's contents; each call clears what
 * must start at zero.
 */
hla_status_t hla2_forward_normalized_noalloc(const void* q, const void* k, const void* v, float* o,
                                             int B, int H, int T, int d, int dv, hla_dtype_t dtype,
                                             const float* gamma, float eps, void* stream);

/*
 * Device status word of the last hla2_forward_normalized_noalloc() call on the
 * current device (the paper has no counterpart).  That call keeps its status
 * word inside the built-in scratch array, whose address callers never see, so
 * this is how they learn whether one of its kernels gave up a bounded wait.
 * Synchronises `stream`, then copies the word into *device_status: HLA_OK, or
 * HLA_ERR_TIMEOUT when a bounded wait ran out (the output is then undefined).
 * Returns HLA_ERR_NULL for a NULL device_status, HLA_ERR_CUDA if a CUDA call
 * fails; before the first no-alloc call on the device it reports HLA_OK.
 */
hla_status_t hla_noalloc_read_device_status(void* stream, int* device_status);

/*
 * Tensor-core layout self-check (diagnostic; no counterpart on the pages).
 * Runs one tcgen05 bf16 MMA of shape M x N x K on one CTA:
 *   D[M][N] = sum_k A(m,k) B(k,n), fp32 accumulate,
 * with A given row-major as a[M][K] (bit 1 clear: K-major) or as a[K][M]
 * (bit 1 set: MN-major), and B given as b[N][K] (bit 0 clear: K-major) or as
 * b[K][N] (bit 0 set: MN-major).  Bit 2 selects M = 64 (else 128); bit 3 (with
 * bit 2) places the M = 64 accumulator at TMEM lane offset 16.  Bit 4 reads A from
 * tensor memory (M = 128 and a given as a[M][K]; not with bits 1-3).  N is 64, 128,
 * 192 or 256; K is 64 or 128 (else HLA_ERR_SHAPE).
 * a, b: device bf16; d: device fp32 [M][N].  Enqueued on `stream`.
 */
hla_status_t hla_selftest_umma(int layout_case, const void* a, const void* b, float* d,
                               int N, int K, void* stream);

/*
 * Failure-path self-check (diagnostic; no counterpart on the pages).  Launches one small
 * kernel whose bounded mbarrier wait runs out on purpose (nothing ever arrives): after
 * `timeout_us` microseconds of %globaltimer it records HLA_ERR_TIMEOUT in the status word
 * at the start of `workspace`, frees the tensor memory it allocated and returns, as the
 * forward kernels do when one of their waits runs out.  No fault, trap or hang: the context
 * stays usable.  Read the outcome with hla_read_device_status.
 *   workspace: device memory of at least 256 bytes (16-byte aligned); its status word is
 *              cleared by this call.
 *   timeout_us: 1 .. 1000000 (else HLA_ERR_SHAPE).
 * Enqueued on `stream`; returns HLA_OK once launched.
 */
hla_status_t hla_selftest_wait_timeout(void* workspace, size_t workspace_bytes, unsigned timeout_us,
                                       void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HLA_H_ */
