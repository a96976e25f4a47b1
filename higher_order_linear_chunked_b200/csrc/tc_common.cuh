// Pieces shared by the tcgen05 walkers (second order in tc_hla.cu, AHLA in tc_ahla.cu):
// tile geometry, UMMA shared-memory descriptors, epilogue stores into 128B-swizzled
// tiles, the segment-summary slot layout and the host-side set-up (tensor maps, the
// segment plan, the segment-prefix launches).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace hla {
namespace tc {

using bf16 = __nv_bfloat16;

constexpr int C = 128;             // chunk length (tokens) = MMA M
constexpr int D = 64;              // head dim (d = dv)
constexpr int kSMs = 148;          // B200 streaming multiprocessors
constexpr uint32_t TILE = C * D * 2;   // one [128][64] bf16 tile = 16 KB

// Segment summaries use the layout of the shared scan kernel (second order, d = 64):
// S, C, R as 64 x 64 row-major matrices, then m, r, then padding.
struct simt_layout {
    static constexpr int size = (3 * D * D + 2 * D + 4 + 31) / 32 * 32;
    __host__ __device__ static constexpr int mat(int i) { return i * D * D; }
    __host__ __device__ static constexpr int vec(int i) { return 3 * D * D + i * D; }
};

struct Params {
    int T, BH, NCH, NS, NSp;
    int ratio;      // output walk: summary slots per output segment (prefix of segment s at s * ratio)
    int fold;       // output walk: fold the prefix from the summaries (no prefix kernels)
    float eps;
    int norm;       // second order: divide by the denominator
    float* sums;     // [BH][NSp][summary floats]: segment summaries
    float* pre;      // [BH][NSp][summary floats]: carried-in prefixes
    float* o;        // [BH][T][64]
    int* status;
    const float* gamma;  // AHLA with decay: per-head gamma (else nullptr)
    int H;               // heads per batch (gamma index = bh % H)
};

// ---------------------------------------------------------------- descriptors
// K-major tile of `rows` rows, K = 64 per atom; K-step s (16 elements).
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int s) { return ptx::desc_sw128(base + s * 32, 16, 1024); }
// K-major [128][128] tile in two 64-wide atoms.
__device__ __forceinline__ uint64_t kdesc2(uint32_t base, int s) {
    return ptx::desc_sw128(base + (s >> 2) * TILE + (s & 3) * 32, 16, 1024);
}
// MN-major tile: one 128-byte row per token; K-step s covers tokens 16s..16s+15;
// lbo = distance to the next 64-wide M/N block.
__device__ __forceinline__ uint64_t mdesc(uint32_t base, uint32_t lbo, int s) {
    return ptx::desc_sw128(base + s * 2048, lbo, 1024);
}

// ---------------------------------------------------------------- epilogue helpers
// Write 16 consecutive fp32 values (columns c0..c0+15 of row `row`) as bf16 into a
// K-major 128B-swizzled tile whose atoms are `atom_bytes` apart.
__device__ __forceinline__ void st_row16(uint8_t* tile, uint32_t atom_bytes, int row, int c0, const float (&v)[16]) {
    uint8_t* atom = tile + (c0 >> 6) * atom_bytes;
    const int cin = c0 & 63;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint4 u;
        u.x = ptx::pack_bf16(v[8 * h + 0], v[8 * h + 1]);
        u.y = ptx::pack_bf16(v[8 * h + 2], v[8 * h + 3]);
        u.z = ptx::pack_bf16(v[8 * h + 4], v[8 * h + 5]);
        u.w = ptx::pack_bf16(v[8 * h + 6], v[8 * h + 7]);
        const int chunk = (cin >> 3) + h;
        *reinterpret_cast<uint4*>(atom + row * 128 + (((chunk ^ row) & 7) << 4)) = u;
    }
}
// 32 consecutive columns c0..c0+31 (c0 a multiple of 32) of row `row` into a K-major
// [rows][128] tile made of two 64-wide atoms TILE bytes apart (or one atom when c0 < 64).
__device__ __forceinline__ void st_row32(uint8_t* tile, int row, int c0, const float (&v)[32]) {
    uint8_t* atom = tile + (c0 >> 6) * TILE;
    const int cin = c0 & 63;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        uint4 u;
        u.x = ptx::pack_bf16(v[8 * h + 0], v[8 * h + 1]);
        u.y = ptx::pack_bf16(v[8 * h + 2], v[8 * h + 3]);
        u.z = ptx::pack_bf16(v[8 * h + 4], v[8 * h + 5]);
        u.w = ptx::pack_bf16(v[8 * h + 6], v[8 * h + 7]);
        const int chunk = (cin >> 3) + h;
        *reinterpret_cast<uint4*>(atom + row * 128 + (((chunk ^ row) & 7) << 4)) = u;
    }
}
// 32 zero columns c0..c0+31 of row `row` (a block that the causal mask clears).
__device__ __forceinline__ void st_row32_zero(uint8_t* tile, int row, int c0) {
    uint8_t* atom = tile + (c0 >> 6) * TILE;
    const int cin = c0 & 63;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const int chunk = (cin >> 3) + h;
        *reinterpret_cast<uint4*>(atom + row * 128 + (((chunk ^ row) & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
    }
}

// ---------------------------------------------------------------- bf16 splits of fp32 values
// x = x1 + x2 (+ x3): each term the bf16 rounding of what the earlier ones leave (exact in bf16);
// the residual is about 2^-16 |x| after two terms and 2^-24 |x| after three.
__device__ __forceinline__ float bf16_hi(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
__device__ __forceinline__ void bf16_split3(float x, float& a, float& b, float& c) {
    a = bf16_hi(x);
    const float r = x - a;
    b = bf16_hi(r);
    c = bf16_hi(r - b);
}

// ---------------------------------------------------------------- host side
// Dynamic shared memory of a kernel, with the whole unified L1 / shared array preferred as shared
// memory: the default carveout can leave room for only one CTA of ~100 KB on an SM, which would
// halve the walkers that are sized to run two per SM.
template <typename K>
inline cudaError_t set_smem(K* kernel, int bytes) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                static_cast<int>(cudaSharedmemCarveoutMaxShared));
}
// [BH][T][64] bf16 tensor, box = one 128-token chunk, 128-byte swizzle, zero fill past T.
bool make_map(CUtensorMap* map, const void* base, int T, int BH);
// [BH][T][64] fp32 output, box = 32 columns x one chunk, 128-byte swizzle (TMA stores).
bool make_map_out(CUtensorMap* map, float* base, int T, int BH);

struct Plan {
    int NC;    // chunks per head
    int NCH;   // chunks per output segment
    int NS;    // output segments per head
    int NCHs;  // chunks per summary segment (divides NCH)
    int NSf;   // summary segments per head: they cover the chunks before the last output segment
    int NSp;   // NSf + 1 rounded up to a power of two (summary / prefix slots per head)
    int ratio; // NCH / NCHs
};
// Segment lengths for BH heads of T tokens when `slots` walker CTAs can run at once.  The
// last output segment's summary is never needed, so summaries cover (NS - 1) NCH chunks per
// head, in segments short enough to fill the machine.
// seg_chunks: chunks per output segment (0 = automatic).
Plan plan(int BH, int T, int slots, int seg_chunks);

// Up to this many summary slots per head, an output walker folds its prefix itself.
constexpr int PH_MAX = 9;

// Exclusive segment prefixes of the summaries (slot layout simt_layout): `pre` gets, for
// every segment l, (S0(l), m0(l)) and the corrected (R0(l), r0(l)).  Three launches: running
// sums of S and m, the cross term per segment, running sums of the corrected R and r.
// left_vec: the vector of the second slot is a row on the left of the first factor's
// partner (ratio-normalised AHLA: n_AB = n_A + n_B + D_B mK_A, D^T in the C place) instead of
// the second order's r_AB = r_A + r_B + S_A m_B.
cudaError_t launch_prefix(const float* sums, float* pre, int NS, int NSp, int BH, cudaStream_t st,
                          bool left_vec = false);

// The decayed second-order forward as a segment walk (tc_decay.cu): the summary walk, then the
// output walk with the prefix of the summaries folded into each output CTA.
size_t decay_workspace_bytes(int BH, int T, int seg_chunks);
int decay_kernel_launches(int BH, int T, int seg_chunks);
cudaError_t decay_forward(const void* q, const void* k, const void* v, const float* gamma, float* o, int BH,
                          int H, int T, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev, int seg_chunks);

// The AHLA forward on the tcgen05 walkers, plain or ratio-normalised, with per-head decay when
// gamma is given (tc_ahla.cu).  The decayed walk needs the prefix folded into the output walker
// (ahla_folds).
size_t ahla_workspace_bytes(int BH, int T, int seg_chunks, bool norm);
int ahla_ctas_per_sm(bool norm);
bool ahla_folds(int BH, int T, int seg_chunks, bool norm);
cudaError_t ahla_forward(const void* q, const void* k, const void* v, float* o, int BH, int H, int T, bool norm,
                         float eps, const float* gamma, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev,
                         int seg_chunks);

}  // namespace tc
}  // namespace hla
