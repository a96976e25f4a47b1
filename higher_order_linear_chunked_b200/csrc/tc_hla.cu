// tcgen05 tensor-core path for the second-order masked HLA forward (bf16 inputs, d = dv = 64).
//
// "Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 1 and 4.
// The sequence of each head is cut into segments of NCH chunks of c = 128 tokens.
//
//  1. k_walk<SUMMARY>: one CTA per (segment, head) walks its chunks from the zero
//     state and writes the segment summary (S, C, m, R = S C - G, r = S m - h) in fp32.
//  2. the Blelloch exclusive scan with the semidirect-product combine (shared with the
//     CUDA-core path) turns segment summaries into carried-in prefixes.
//  3. k_walk<OUTPUT>: one CTA per (segment, head) starts from its prefix and walks its
//     chunks again, emitting o for every token and carrying (S, R, r) to the next chunk.
//
// Per chunk (Q, K, V: 128 x 64 tiles; S0, R0, r0: state carried into the chunk):
//     A  = L (.) (Q K^T)                         (tcgen05, M=128 N=128 K=64)
//     P  = Q S0                                  (M=128 N=64  K=64)
//     W  = L (.) (P Q^T + A A^T)                 (M=128 N=128 K=64+128)
//     O  = Q [R0 | r0] + W V,  den = q.r0 + W 1  (M=128 N=80 K=64; N=64 K=128)
//     Z  = P + A K        (Z_j = S_j q_j, S_j the key moment up to token j)
//     S0 += K^T K;  [R0 | r0] += Z^T [V | 1]      (stacked M=128 MN-major operands)
// The tensor-core state lives in TMEM (fp32) across the walk; its bf16 copies feed
// the next chunk's MMAs.  TMA stages Q, K, V (128B swizzle, no multicast), double
// buffered; one thread issues TMA and MMA; four warps run the TMEM epilogues.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"
#include "simt.h"
#include "tc.h"

namespace hla {
namespace tc {

using bf16 = __nv_bfloat16;

constexpr int C = 128;             // chunk length (tokens) = MMA M
constexpr int D = 64;              // head dim (d = dv)
constexpr int NT = 128;            // threads: 4 warps <-> 128 TMEM lanes
constexpr int DEFAULT_NCH = 4;     // chunks per segment
constexpr uint32_t TILE = C * D * 2;   // one [128][64] bf16 tile = 16 KB

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t SM_Q0 = 0, SM_Q1 = SM_Q0 + TILE;
constexpr uint32_t SM_K0 = SM_Q1 + TILE, SM_V0 = SM_K0 + TILE;
constexpr uint32_t SM_K1 = SM_V0 + TILE, SM_V1 = SM_K1 + TILE;
constexpr uint32_t SM_Z = SM_V1 + TILE;          // P, then Z  ([tok][feat])
constexpr uint32_t SM_ONES = SM_Z + TILE;        // MN-major [tok][64], column 0 = 1
constexpr uint32_t SM_A = SM_ONES + TILE;        // A, then W: [128][128] K-major (2 atoms)
constexpr uint32_t SM_S0 = SM_A + 2 * TILE;      // S0^T: [64 n][64 k] K-major
constexpr uint32_t SM_R0 = SM_S0 + 64 * 128;     // [R0 | r0]^T: [80 n][64 k] K-major
constexpr uint32_t SM_BAR = SM_R0 + 80 * 128;    // mbarriers
constexpr uint32_t SM_TOTAL = SM_BAR + 64;
constexpr uint32_t SMEM_BYTES = SM_TOTAL + 1024; // + alignment slack

// TMEM columns (fp32 accumulators, 128 lanes).
constexpr uint32_t TM_A = 0;      // A, then W            (128 cols)
constexpr uint32_t TM_P = 128;    // P, then Z            (64)
constexpr uint32_t TM_O = 192;    // O | q.r0             (80)
constexpr uint32_t TM_CR = 272;   // lanes 0-63 [C|m], lanes 64-127 [R|r]  (80)
constexpr uint32_t TM_S = 352;    // lanes 0-63 S         (64)
constexpr uint32_t TM_COLS = 512;

enum Mode { SUMMARY = 0, OUTPUT = 1 };

// Segment summaries use the layout of the shared scan kernel (second order, d = 64):
// S, C, R as 64 x 64 row-major matrices, then m, r, then padding.
struct simt_layout {
    static constexpr int size = (3 * D * D + 2 * D + 4 + 31) / 32 * 32;
    __host__ __device__ static constexpr int mat(int i) { return i * D * D; }
    __host__ __device__ static constexpr int vec(int i) { return 3 * D * D + i * D; }
};

struct Params {
    int T, BH, NCH, NS, NSp;
    float eps;
    int norm;
    float* sums;     // [BH][NSp][summary floats]
    float* o;        // [BH][T][64]
    int* status;
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
// Transposed write: value v[i] is element (n = c0 + i, k = kcol) of a K-major tile.
__device__ __forceinline__ void st_col16(uint8_t* tile, int kcol, int c0, const float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
        *reinterpret_cast<bf16*>(tile + ptx::sw128_offset(c0 + i, kcol)) = __float2bfloat16_rn(v[i]);
}

// ---------------------------------------------------------------- the walker
template <int MODE>
__global__ void __launch_bounds__(NT, 1)
k_walk(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
       const __grid_constant__ CUtensorMap tv, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + SM_BAR);       // [2]
    uint64_t* bar_mma = bar_load + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int seg = blockIdx.x, bh = blockIdx.y;
    using S = simt_layout;
    float* slot = p.sums + ((size_t)bh * p.NSp + seg) * S::size;
    if (seg >= p.NS) {                       // scan padding: identity (zeros)
        if (MODE == SUMMARY)
            for (int e = tid; e < S::size; e += NT) slot[e] = 0.f;
        return;
    }
    const int chunk0 = seg * p.NCH;
    const int nchunks_total = (p.T + C - 1) / C;
    const int nch = min(p.NCH, nchunks_total - chunk0);

    // ---- set-up: barriers, TMEM, constant tiles, carried-in state
    if (tid == 0) {
        ptx::mbar_init(&bar_load[0], 1);
        ptx::mbar_init(&bar_load[1], 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tq);
        ptx::prefetch_tmap(&tk);
        ptx::prefetch_tmap(&tv);
    }
    if (warp == 0) {
        ptx::tmem_alloc(tmem_slot, TM_COLS);
        ptx::tmem_relinquish();
    }
    {   // ones tile: MN-major, element (token kk, column 0) = 1
        uint32_t* w = reinterpret_cast<uint32_t*>(sm + SM_ONES);
        for (int e = tid; e < (int)(TILE / 4); e += NT) w[e] = 0u;
    }
    __syncthreads();
    {
        const bf16 one = __float2bfloat16_rn(1.f);
        *reinterpret_cast<bf16*>(sm + SM_ONES + ptx::sw128_offset(tid, 0)) = one;   // tid = token row 0..127
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

    // Issue the TMA loads of chunk `n` (local index) into buffer n & 1.
    auto issue_load = [&](int n) {
        const int b = n & 1;
        const int t0 = (chunk0 + n) * C;
        ptx::mbar_arrive_expect_tx(&bar_load[b], 3 * TILE);
        ptx::tma_load_3d(sm + (b ? SM_Q1 : SM_Q0), &tq, &bar_load[b], 0, t0, bh);
        ptx::tma_load_3d(sm + (b ? SM_K1 : SM_K0), &tk, &bar_load[b], 0, t0, bh);
        ptx::tma_load_3d(sm + (b ? SM_V1 : SM_V0), &tv, &bar_load[b], 0, t0, bh);
    };
    if (tid == 0) {
        issue_load(0);
        if (nch > 1) issue_load(1);
    }

    // Carried-in state: fp32 into TMEM (S in TM_S lanes 0-63, [R|r] in TM_CR lanes 64-127),
    // bf16 transposed copies into SM_S0 / SM_R0.  The summary walk starts from zero.
    {
        float v[16];
        if (warp < 2) {                      // S row `tid`
            const float* src = slot + S::mat(0) + tid * D;
            for (int c0 = 0; c0 < D; c0 += 16) {
                for (int i = 0; i < 16; ++i) v[i] = (MODE == OUTPUT) ? src[c0 + i] : 0.f;
                if (MODE == OUTPUT) ptx::tmem_st16(tmem + lane_base + TM_S + c0, v);
                st_col16(sm + SM_S0, tid, c0, v);
            }
        } else {                             // [R | r] row tid - 64
            const int r = tid - 64;
            const float* src = slot + S::mat(2) + r * D;
            for (int c0 = 0; c0 < 80; c0 += 16) {
                for (int i = 0; i < 16; ++i) {
                    const int c = c0 + i;
                    float x = 0.f;
                    if (MODE == OUTPUT) x = c < D ? src[c] : (c == D ? slot[S::vec(1) + r] : 0.f);
                    v[i] = x;
                }
                if (MODE == OUTPUT) ptx::tmem_st16(tmem + lane_base + TM_CR + c0, v);
                st_col16(sm + SM_R0, r, c0, v);
            }
        }
        if (MODE == OUTPUT) ptx::tmem_st_wait();
    }
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    const uint32_t sbase = ptx::smem_u32(sm);
    constexpr uint32_t I_QK = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t I_N64_KK = ptx::idesc_bf16(128, 64, false, false);
    constexpr uint32_t I_N64_KM = ptx::idesc_bf16(128, 64, false, true);
    constexpr uint32_t I_N64_MM = ptx::idesc_bf16(128, 64, true, true);
    constexpr uint32_t I_N80_KK = ptx::idesc_bf16(128, 80, false, false);
    constexpr uint32_t I_N80_MM = ptx::idesc_bf16(128, 80, true, true);

    uint32_t mma_phase = 0;
    bool ok = true;
    // Thread 0 waits on the MMA barrier (bounded); the block agrees on the outcome.
    auto wait_mma = [&]() -> bool {
        bool good = true;
        if (tid == 0) {
            ptx::umma_commit(bar_mma);
            good = ptx::mbar_wait(bar_mma, mma_phase);
        }
        mma_phase ^= 1;
        good = __syncthreads_and(good) != 0;
        ptx::tc_fence_after();
        return good;
    };
    auto sync_for_mma = [&]() {
        ptx::fence_proxy_async();
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
    };

    const int row = tid;                      // TMEM lane = row of the 128-row tiles
    const int t_base = chunk0 * C;
    for (int n = 0; n < nch && ok; ++n) {
        const int b = n & 1;
        const uint32_t sQ = sbase + (b ? SM_Q1 : SM_Q0);
        const uint32_t sK = sbase + (b ? SM_K1 : SM_K0);
        const uint32_t sV = sbase + (b ? SM_V1 : SM_V0);
        // ---- phase 1: A = Q K^T, P = Q S0
        if (tid == 0) {
            ok = ptx::mbar_wait(&bar_load[b], (n >> 1) & 1);
            if (ok) {
                ptx::tc_fence_after();
                for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TM_A, kdesc(sQ, s), kdesc(sK, s), I_QK, s > 0);
                for (int s = 0; s < 4; ++s)
                    ptx::umma_bf16(tmem + TM_P, kdesc(sQ, s), kdesc(sbase + SM_S0, s), I_N64_KK, s > 0);
            }
        }
        if (!__syncthreads_and(ok)) { ok = false; break; }
        if (!wait_mma()) { ok = false; break; }
        // ---- epilogue 1: A (masked) and P to bf16 tiles
        {
            float v[16];
            for (int c0 = 0; c0 < C; c0 += 16) {
                ptx::tmem_ld16(tmem + lane_base + TM_A + c0, v);
                for (int i = 0; i < 16; ++i)
                    if (c0 + i > row) v[i] = 0.f;
                st_row16(sm + SM_A, TILE, row, c0, v);
            }
            if (MODE == OUTPUT)
                for (int c0 = 0; c0 < D; c0 += 16) {
                    ptx::tmem_ld16(tmem + lane_base + TM_P + c0, v);
                    st_row16(sm + SM_Z, TILE, row, c0, v);
                }
        }
        sync_for_mma();
        // ---- phase 2: W = P Q^T + A A^T ; Z = P + A K ; S += K^T K ; O = Q [R0|r0]
        if (tid == 0) {
            if (MODE == OUTPUT) {
                for (int s = 0; s < 4; ++s)
                    ptx::umma_bf16(tmem + TM_A, kdesc(sbase + SM_Z, s), kdesc(sQ, s), I_QK, s > 0);
                for (int s = 0; s < 8; ++s)
                    ptx::umma_bf16(tmem + TM_A, kdesc2(sbase + SM_A, s), kdesc2(sbase + SM_A, s), I_QK, 1);
                for (int s = 0; s < 4; ++s)
                    ptx::umma_bf16(tmem + TM_O, kdesc(sQ, s), kdesc(sbase + SM_R0, s), I_N80_KK, s > 0);
            }
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + TM_P, kdesc2(sbase + SM_A, s), mdesc(sK, TILE, s), I_N64_KM, 1);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + TM_S, mdesc(sK, sV - sK, s), mdesc(sK, TILE, s), I_N64_MM,
                               (MODE == OUTPUT || n > 0 || s > 0) ? 1u : 0u);
        }
        if (!wait_mma()) { ok = false; break; }
        // ---- epilogue 2: W (masked) -> bf16 (+ row sums), Z -> bf16, S -> bf16 S0^T
        float rowsum = 0.f;
        {
            float v[16];
            if (MODE == OUTPUT)
                for (int c0 = 0; c0 < C; c0 += 16) {
                    ptx::tmem_ld16(tmem + lane_base + TM_A + c0, v);
                    for (int i = 0; i < 16; ++i) {
                        const float x = (c0 + i > row) ? 0.f : __bfloat162float(__float2bfloat16_rn(v[i]));
                        v[i] = x;
                        rowsum += x;
                    }
                    st_row16(sm + SM_A, TILE, row, c0, v);
                }
            for (int c0 = 0; c0 < D; c0 += 16) {
                ptx::tmem_ld16(tmem + lane_base + TM_P + c0, v);
                st_row16(sm + SM_Z, TILE, row, c0, v);
            }
            if (warp < 2)
                for (int c0 = 0; c0 < D; c0 += 16) {
                    ptx::tmem_ld16(tmem + lane_base + TM_S + c0, v);
                    st_col16(sm + SM_S0, row, c0, v);
                }
        }
        sync_for_mma();
        // ---- phase 3: O += W V ; [C|m ; R|r] += [Q^T ; Z^T] [V | 1]
        if (tid == 0) {
            if (MODE == OUTPUT)
                for (int s = 0; s < 8; ++s)
                    ptx::umma_bf16(tmem + TM_O, kdesc2(sbase + SM_A, s), mdesc(sV, TILE, s), I_N64_KM, 1);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + TM_CR, mdesc(sQ, sbase + SM_Z - sQ, s), mdesc(sV, sbase + SM_ONES - sV, s),
                               I_N80_MM, (MODE == OUTPUT || n > 0 || s > 0) ? 1u : 0u);
        }
        if (!wait_mma()) { ok = false; break; }
        // ---- epilogue 3: output rows; [R|r] -> bf16 transposed copy; next loads
        if (tid == 0 && n + 2 < nch) issue_load(n + 2);
        if (MODE == OUTPUT) {
            float v[16];
            ptx::tmem_ld16(tmem + lane_base + TM_O + 64, v);
            const float den = v[0] + rowsum;
            const float scale = p.norm ? 1.f / (den + p.eps) : 1.f;
            const int t = t_base + n * C + row;
            float* orow = p.o + ((size_t)bh * p.T + t) * D;
            for (int c0 = 0; c0 < D; c0 += 16) {
                ptx::tmem_ld16(tmem + lane_base + TM_O + c0, v);
                if (t < p.T)
                    for (int i = 0; i < 16; i += 4)
                        *reinterpret_cast<float4*>(orow + c0 + i) =
                            make_float4(v[i] * scale, v[i + 1] * scale, v[i + 2] * scale, v[i + 3] * scale);
            }
            if (warp >= 2)
                for (int c0 = 0; c0 < 80; c0 += 16) {
                    ptx::tmem_ld16(tmem + lane_base + TM_CR + c0, v);
                    st_col16(sm + SM_R0, row - 64, c0, v);
                }
        }
        sync_for_mma();
    }

    // ---- summary: write the segment's state (fp32)
    if (MODE == SUMMARY && ok) {
        float v[16];
        if (warp < 2) {
            for (int c0 = 0; c0 < D; c0 += 16) {            // S row
                ptx::tmem_ld16(tmem + lane_base + TM_S + c0, v);
                for (int i = 0; i < 16; ++i) slot[S::mat(0) + row * D + c0 + i] = v[i];
            }
            for (int c0 = 0; c0 < 80; c0 += 16) {           // [C | m] row
                ptx::tmem_ld16(tmem + lane_base + TM_CR + c0, v);
                for (int i = 0; i < 16; ++i) {
                    const int c = c0 + i;
                    if (c < D) slot[S::mat(1) + row * D + c] = v[i];
                    else if (c == D) slot[S::vec(0) + row] = v[i];
                }
            }
        } else {
            const int r = row - 64;
            for (int c0 = 0; c0 < 80; c0 += 16) {           // [R | r] row
                ptx::tmem_ld16(tmem + lane_base + TM_CR + c0, v);
                for (int i = 0; i < 16; ++i) {
                    const int c = c0 + i;
                    if (c < D) slot[S::mat(2) + r * D + c] = v[i];
                    else if (c == D) slot[S::vec(1) + r] = v[i];
                }
            }
        }
    }
    if (!ok) {
        if (tid == 0) {
            set_status(p.status, DEV_TIMEOUT);
            // let copies and MMAs already in flight land before TMEM and smem are released
            ptx::mbar_wait(&bar_load[0], 0, 100000000ull);
            ptx::mbar_wait(&bar_load[1], 0, 100000000ull);
            ptx::umma_commit(bar_mma);
            ptx::mbar_wait(bar_mma, mma_phase, 100000000ull);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) ptx::tmem_dealloc(tmem, TM_COLS);
}

// ---------------------------------------------------------------- host side
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(ptr);
    }
    return fn;
}

// [BH][T][64] bf16 tensor, box = one 128-token chunk, 128-byte swizzle, zero fill past T.
bool make_map(CUtensorMap* map, const void* base, int T, int BH) {
    EncodeTiled fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
    const cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)C, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int next_pow2(int n) {
    int p = 1;
    while (p < n) p *= 2;
    return p;
}

struct Plan {
    int NC, NCH, NS, NSp;
};

int g_segment_chunks = 0;   // 0 = automatic

Plan plan(int BH, int T) {
    Plan pl;
    pl.NC = (T + C - 1) / C;
    if (g_segment_chunks > 0) {
        pl.NCH = g_segment_chunks;
    } else {
        pl.NCH = DEFAULT_NCH;
        // keep at least two waves of CTAs on 148 SMs when the sequence allows it
        while (pl.NCH > 1 && (long long)BH * ((pl.NC + pl.NCH - 1) / pl.NCH) < 2 * 148) pl.NCH /= 2;
    }
    pl.NS = (pl.NC + pl.NCH - 1) / pl.NCH;
    pl.NSp = next_pow2(pl.NS);
    return pl;
}

}  // namespace

bool set_segment_chunks(int chunks) {
    if (chunks != 0 && chunks != 1 && chunks != 2 && chunks != 4 && chunks != 8 && chunks != 16) return false;
    g_segment_chunks = chunks;
    return true;
}

bool supported(int op, bool /*norm*/, bool bf16, int d) { return op == OP_HLA2 && bf16 && d == D; }

size_t workspace_bytes(int /*op*/, bool /*norm*/, int BH, int T) {
    const Plan pl = plan(BH, T);
    return sizeof(float) * (size_t)BH * pl.NSp * simt_layout::size;
}

int kernel_launches(int /*op*/, bool /*norm*/, int BH, int T) { return 2 + simt::scan_launches(plan(BH, T).NSp); }

cudaError_t forward(int op, bool norm, const void* q, const void* k, const void* v, float eps, float* o, int BH,
                    int T, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev) {
    if (op != OP_HLA2) return cudaErrorNotSupported;
    if (simt::summary_floats(OP_HLA2, D) != (size_t)simt_layout::size) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, T, BH) || !make_map(&mk, k, T, BH) || !make_map(&mv, v, T, BH))
        return cudaErrorInvalidValue;
    const Plan pl = plan(BH, T);
    Params prm;
    prm.T = T; prm.BH = BH; prm.NCH = pl.NCH; prm.NS = pl.NS; prm.NSp = pl.NSp;
    prm.eps = eps; prm.norm = norm ? 1 : 0;
    prm.sums = static_cast<float*>(ws);
    prm.o = o;
    prm.status = status;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_walk<SUMMARY>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_walk<OUTPUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
        cudaSuccess)
        return e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    k_walk<SUMMARY><<<dim3(pl.NSp, BH), NT, SMEM_BYTES, st>>>(mq, mk, mv, prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    if ((e = simt::scan(OP_HLA2, D, prm.sums, pl.NSp, BH, st)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[2], st)) != cudaSuccess) return e;
    k_walk<OUTPUT><<<dim3(pl.NS, BH), NT, SMEM_BYTES, st>>>(mq, mk, mv, prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[3], st)) != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace tc
}  // namespace hla
