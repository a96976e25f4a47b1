// tcgen05 gradients of the masked second-order output for bf16 inputs at d = dv = 64: the
// per-chunk stage of the backward pass (dQ, dK, dV of every 128-token chunk).
//
// "Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 1 and 4,
// Contribuciones 2: the page offers the exact chunked scan as the basis of parallel training but
// prints no gradient.  The forward's chunk algebra (second-order walker) in its Z form:
//     A = L (.) Q K^T,   Z = Q S0 + A K          (row j: S_j q_j),
//     W = L (.) Q Z^T,   O = Q R0 + W V,         S0' = S0 + K^T K,   R0' = R0 + Z^T V,
// with (S0, R0) the state carried into the chunk.  Reverse mode, with dO given and (G_S, G_R) the
// adjoints of the state the chunk hands on (dS', dR' of the CUDA-core pipeline):
//     dW = L (.) dO V^T,        dZ = dW^T Q + V G_R^T,       dA = L (.) dZ K^T,
//     dQ = dO R0^T + dZ S0 + dW Z + dA K,
//     dK = K (G_S + G_S^T) + A^T dZ + dA^T Q,
//     dV = W^T dO + Z G_R.
// (L (.) (Q S0 Q^T + A A^T) = L (.) Q Z^T, so this is the derivative of the same output as the
// P form of the CUDA-core kernel; no product here has an inner dimension of c x c x c.)
//
// One CTA per chunk: every chunk's carried state and adjoints come from the earlier stages, so
// the chunks are independent.  Four rounds of MMAs, each followed by an epilogue of the eight
// warps (warp w: TMEM lane quadrant w & 3, column half w >> 2):
//   R1: A* = Q K^T, Z = Q S0, dW* = dO V^T           -> E1: A, dW masked to bf16 tiles
//       (dO: the two-term split below; dZ likewise)
//   R2: Z += A K, dZ = dW^T Q + V G_R^T               -> E2: Z, dZ to bf16 tiles
//   R3: W* = Q Z^T, dA* = dZ K^T,
//       dK = K (G_S^T + G_S) + A^T dZ,                -> E3: W (over A), dA (over dZ, S0, G_S)
//       dQ = dO R0^T + dZ S0   (G_S read K-major and MN-major: no transposed copy)
//   R4: dV = W^T dO + Z G_R, dQ += dW Z + dA K, dK += dA^T Q
//                                                     -> E4: dQ, dK, dV staged, TMA stores
// TMEM (512 columns): A* / W* 0-127, dW* / dA* 128-255, Z / dV 256-319, dZ 320-383, dK 384-447,
// dQ 448-511.  Transposed operands are the same tiles read MN-major.
//
// Precision: every operand is bf16 with fp32 accumulation.  The output gradient dO (fp32 input)
// and dZ (the intermediate every gradient passes through) enter as two bf16 terms, x = hi + lo
// with hi = bf16(x), lo = bf16(x - hi), in each product they take part in: a gradient row can be
// much smaller than its terms, and these two roundings set most of the error left on such rows.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tc.h"
#include "tc_common.cuh"

namespace hla {
namespace tc {
namespace {

constexpr int BNT = 256;                        // 8 warps; thread 0 also issues loads and MMAs
constexpr int BW_SIZE = 3 * D * D;              // adjoint slot per 64-token chunk: dR', dS', C
constexpr uint32_t MAT = D * D * 2;             // one 64 x 64 bf16 tile (8 KB)

// Shared memory (offsets from a 1024-byte aligned base).
constexpr uint32_t SB_Q = 0;                    // Q   [tok][64]
constexpr uint32_t SB_K = SB_Q + TILE;          // K
constexpr uint32_t SB_V = SB_K + TILE;          // V
constexpr uint32_t SB_O = SB_V + TILE;          // dO as bf16 (hi)
constexpr uint32_t SB_OL = SB_O + TILE;         // dO - hi as bf16 (lo)
constexpr uint32_t SB_A = SB_OL + TILE;         // A masked, K-major [t][j] in two atoms; then W
constexpr uint32_t SB_DW = SB_A + 2 * TILE;     // dW masked
constexpr uint32_t SB_Z = SB_DW + 2 * TILE;     // Z   [tok][64]
constexpr uint32_t SB_DZ = SB_Z + TILE;         // dZ  [tok][64]      } after R3: dA (two atoms)
constexpr uint32_t SB_S0 = SB_DZ + TILE;        // S0  [64][64]       }
constexpr uint32_t SB_GS = SB_S0 + MAT;         // G_S                }
constexpr uint32_t SB_DZL = SB_GS + MAT;        // dZ - hi (lo)
constexpr uint32_t SB_R0 = SB_DZL + TILE;       // R0  [64][64]
constexpr uint32_t SB_GR = SB_R0 + MAT;         // G_R [64][64]
constexpr uint32_t SB_DA = SB_DZ;
constexpr uint32_t SB_BAR = SB_GR + MAT;
constexpr uint32_t BSMEM_BYTES = SB_BAR + 64 + 1024;
// staging: dO (fp32, two [128][32] TMA boxes) over A at the start; dQ, dK, dV at the end
constexpr uint32_t SB_OF = SB_A;
constexpr uint32_t SB_ST_Q = SB_Q, SB_ST_K = SB_V, SB_ST_V = SB_A;

constexpr uint32_t TB_A = 0, TB_DW = 128, TB_Z = 256, TB_DZ = 320, TB_DK = 384, TB_DQ = 448, TB_COLS = 512;
constexpr uint32_t TB_W = TB_A, TB_DA = TB_DW, TB_DV = TB_Z;

struct BwdParams {
    int T, NSp;
    const float* pre;    // exclusive prefixes per chunk (NSp slots per head): S0 = mat 0, R0 = mat 2
    const float* bw;     // adjoint slots per chunk (NSp per head): dR' = 0, dS' = 1 (exclusive suffixes)
    float* terms;        // k_bwd_terms: the slots [Y | U | C] it writes
    int* status;
};

// Four 64 x 64 fp32 row-major matrices (global) -> bf16 K-major tiles (128-byte swizzle).  Thread
// t converts row t / 4, columns 16 (t % 4) .. + 15 of each; all sixteen 16-byte loads are issued
// before the first conversion.
__device__ __forceinline__ void mat_tiles4(uint8_t* const (&tiles)[4], const float* const (&m)[4]) {
    const int r = threadIdx.x >> 2, c0 = 16 * (threadIdx.x & 3);
    float4 x[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) x[j][i] = reinterpret_cast<const float4*>(m[j] + r * D + c0)[i];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[4 * i] = x[j][i].x; v[4 * i + 1] = x[j][i].y; v[4 * i + 2] = x[j][i].z; v[4 * i + 3] = x[j][i].w;
        }
        st_row16(tiles[j], TILE, r, c0, v);
    }
}

// 32 fp32 columns c0 .. c0 + 31 of row `row` as two bf16 terms: hi into one [tok][64] tile, the
// remainder x - hi into another
__device__ __forceinline__ void split_row(uint8_t* hi_tile, uint8_t* lo_tile, int row, int c0, float (&x)[32]) {
    st_row32(hi_tile, row, c0, x);
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] -= __bfloat162float(__float2bfloat16_rn(x[i]));
    st_row32(lo_tile, row, c0, x);
}

__global__ void __launch_bounds__(BNT, 1)
k_bwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
         const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
         const __grid_constant__ CUtensorMap tdq, const __grid_constant__ CUtensorMap tdk,
         const __grid_constant__ CUtensorMap tdv, BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + SB_BAR);
    uint64_t* bar_mma = bar_load + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;                       // TMEM lane = token row of the chunk
    const int chunk = blockIdx.x, bh = blockIdx.y;
    const int t0 = chunk * C;

    if (tid == 0) {
        ptx::mbar_init(bar_load, 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        ptx::mbar_arrive_expect_tx(bar_load, 3 * TILE + 2 * TILE);
        ptx::tma_load_3d(sm + SB_Q, &tq, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + SB_K, &tk, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + SB_V, &tv, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + SB_OF, &tdo, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + SB_OF + C * 128, &tdo, bar_load, 32, t0, bh);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, TB_COLS);
        ptx::tmem_relinquish();
    }
    // carried state (the chunk's exclusive prefix) and the adjoints leaving the chunk (the
    // exclusive suffixes) as bf16 tiles, while the loads are in flight
    {
        const float* pre = p.pre + ((size_t)bh * p.NSp + chunk) * simt_layout::size;
        const float* adj = p.bw + ((size_t)bh * p.NSp + chunk) * BW_SIZE;
        uint8_t* const tiles[4] = {sm + SB_S0, sm + SB_R0, sm + SB_GR, sm + SB_GS};
        const float* const mats[4] = {pre + simt_layout::mat(0), pre + simt_layout::mat(2), adj, adj + D * D};
        mat_tiles4(tiles, mats);
    }
    // the loads: every thread waits (bounded), then dO (fp32 boxes) -> bf16 tile
    bool ok = ptx::mbar_wait(bar_load, 0);
    {
        const float4* box = reinterpret_cast<const float4*>(sm + SB_OF + half * (C * 128) + row * 128);
        float x[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 f = box[j ^ (row & 7)];
            x[4 * j] = f.x; x[4 * j + 1] = f.y; x[4 * j + 2] = f.z; x[4 * j + 3] = f.w;
        }
        split_row(sm + SB_O, sm + SB_OL, row, half * 32, x);
    }
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;

    const uint32_t sb = ptx::smem_u32(sm);
    constexpr uint32_t I_128_KK = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t I_64_KK = ptx::idesc_bf16(128, 64, false, false);
    constexpr uint32_t I_64_KM = ptx::idesc_bf16(128, 64, false, true);
    constexpr uint32_t I_64_MM = ptx::idesc_bf16(128, 64, true, true);
    auto k1 = [](uint64_t d0, int s) { return d0 + (uint64_t)(s * 2); };                     // +32 B
    auto k2 = [](uint64_t d0, int s) { return d0 + (uint64_t)(((s >> 2) * TILE + (s & 3) * 32) >> 4); };
    auto mn = [](uint64_t d0, int s) { return d0 + (uint64_t)(s * 128); };                   // +2048 B
    // K-major [tok][64] or [64][64] tiles (K = 64), K-major [t][j] two-atom tiles (K = 128), and
    // MN-major views: [tok][64] tiles as B (N = 64, K = tokens), [t][j] tiles as A (M = j)
    auto kd = [&](uint32_t off) { return kdesc(sb + off, 0); };
    auto kd2 = [&](uint32_t off) { return kdesc2(sb + off, 0); };
    auto md = [&](uint32_t off) { return mdesc(sb + off, TILE, 0); };
    auto mm_kk = [&](uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool acc) {     // K = 64
        const uint64_t da = kd(a), db = kd(b);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + d, k1(da, s), k1(db, s), idesc, (acc || s > 0) ? 1u : 0u);
    };
    auto mm_k2m = [&](uint32_t d, uint32_t a, uint32_t b, bool acc) {   // A K-major [t][j], B MN [tok][64]
        const uint64_t da = kd2(a), db = md(b);
        for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + d, k2(da, s), mn(db, s), I_64_KM, (acc || s > 0) ? 1u : 0u);
    };
    auto mm_mm = [&](uint32_t d, uint32_t a, uint32_t b, bool acc) {    // A MN [t][j] (A^T), B MN [tok][64]
        const uint64_t da = md(a), db = md(b);
        for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + d, mn(da, s), mn(db, s), I_64_MM, (acc || s > 0) ? 1u : 0u);
    };
    auto mm_km = [&](uint32_t d, uint32_t a, uint32_t b, bool acc) {    // A K-major [tok][64], B MN [64][64]
        const uint64_t da = kd(a), db = md(b);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + d, k1(da, s), mn(db, s), I_64_KM, (acc || s > 0) ? 1u : 0u);
    };

    uint32_t mma_phase = 0;
    auto commit_wait = [&]() -> bool {
        bool good = true;
        ptx::tc_fence_before();
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
    // fp32 TMEM [tcol, tcol + 128) of this lane, masked to tokens j <= row, into the K-major
    // [t][j] tile: this warp's blocks 2 half and 2 half + 1 (zeros above the diagonal)
    auto mask_tile = [&](uint32_t tcol, uint32_t off) {
        const int b0 = 2 * half;
        float v0[32], v1[32];
        if (b0 + 1 <= quad) {
            ptx::tmem_ld32x2(tmem + lane_base + tcol + 32 * b0, tmem + lane_base + tcol + 32 * (b0 + 1), v0, v1);
            if (b0 + 1 == quad) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i > lane) v1[i] = 0.f;
            }
            st_row32(sm + off, row, 32 * b0, v0);
            st_row32(sm + off, row, 32 * (b0 + 1), v1);
        } else if (b0 == quad) {
            ptx::tmem_ld32(tmem + lane_base + tcol + 32 * b0, v0);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (i > lane) v0[i] = 0.f;
            st_row32(sm + off, row, 32 * b0, v0);
            st_row32_zero(sm + off, row, 32 * (b0 + 1));
        } else {
            st_row32_zero(sm + off, row, 32 * b0);
            st_row32_zero(sm + off, row, 32 * (b0 + 1));
        }
    };
    // fp32 TMEM [tcol + 32 half, + 32) of this lane -> its half row of a [tok][64] bf16 tile (and
    // the remainder into a second tile when lo_off is not 0)
    auto half_tile = [&](uint32_t tcol, uint32_t off, uint32_t lo_off) {
        float v[32];
        ptx::tmem_ld32(tmem + lane_base + tcol + 32 * half, v);
        if (lo_off) split_row(sm + off, sm + lo_off, row, 32 * half, v);
        else st_row32(sm + off, row, 32 * half, v);
    };
    // fp32 TMEM half row -> a [128][32] fp32 TMA box (128-byte swizzle)
    auto stage = [&](uint32_t tcol, uint32_t off) {
        float v[32];
        ptx::tmem_ld32(tmem + lane_base + tcol + 32 * half, v);
        float4* box = reinterpret_cast<float4*>(sm + off + half * (C * 128) + row * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            box[j ^ (row & 7)] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    };

    int round = 0;
    if (ok) {
        // R1: A* = Q K^T, Z = Q S0, dW* = dO V^T
        if (tid == 0) {
            mm_kk(TB_A, SB_Q, SB_K, I_128_KK, false);
            mm_kk(TB_Z, SB_Q, SB_S0, I_64_KK, false);
            mm_kk(TB_DW, SB_O, SB_V, I_128_KK, false);
            mm_kk(TB_DW, SB_OL, SB_V, I_128_KK, true);
        }
        round = 1;
        ok = commit_wait();
    }
    if (ok) {
        mask_tile(TB_A, SB_A);
        mask_tile(TB_DW, SB_DW);
        sync_for_mma();
        // R2: Z += A K, dZ = dW^T Q + V G_R^T
        if (tid == 0) {
            mm_k2m(TB_Z, SB_A, SB_K, true);
            mm_mm(TB_DZ, SB_DW, SB_Q, false);
            mm_kk(TB_DZ, SB_V, SB_GR, I_64_KK, true);
        }
        round = 2;
        ok = commit_wait();
    }
    if (ok) {
        half_tile(TB_Z, SB_Z, 0);
        half_tile(TB_DZ, SB_DZ, SB_DZL);
        sync_for_mma();
        // R3: W* = Q Z^T, dA* = dZ K^T, dK = K (G_S^T + G_S) + A^T dZ, dQ = dO R0^T + dZ S0
        if (tid == 0) {
            mm_kk(TB_W, SB_Q, SB_Z, I_128_KK, false);
            mm_kk(TB_DA, SB_DZ, SB_K, I_128_KK, false);
            mm_kk(TB_DA, SB_DZL, SB_K, I_128_KK, true);
            mm_kk(TB_DK, SB_K, SB_GS, I_64_KK, false);            // K G_S^T
            mm_km(TB_DK, SB_K, SB_GS, true);                      // K G_S
            mm_mm(TB_DK, SB_A, SB_DZ, true);
            mm_mm(TB_DK, SB_A, SB_DZL, true);
            mm_kk(TB_DQ, SB_O, SB_R0, I_64_KK, false);
            mm_kk(TB_DQ, SB_OL, SB_R0, I_64_KK, true);
            mm_kk(TB_DQ, SB_DZ, SB_S0, I_64_KK, true);
            mm_kk(TB_DQ, SB_DZL, SB_S0, I_64_KK, true);
        }
        round = 3;
        ok = commit_wait();
    }
    if (ok) {
        mask_tile(TB_W, SB_A);               // W over A (A^T dZ is done)
        mask_tile(TB_DA, SB_DA);             // dA over dZ, S0, G_S (their products are done)
        sync_for_mma();
        // R4: dV = W^T dO + Z G_R, dQ += dW Z + dA K, dK += dA^T Q
        if (tid == 0) {
            mm_mm(TB_DV, SB_A, SB_O, false);
            mm_mm(TB_DV, SB_A, SB_OL, true);
            mm_km(TB_DV, SB_Z, SB_GR, true);
            mm_k2m(TB_DQ, SB_DW, SB_Z, true);
            mm_k2m(TB_DQ, SB_DA, SB_K, true);
            mm_mm(TB_DK, SB_DA, SB_Q, true);
        }
        round = 4;
        ok = commit_wait();
    }
    if (ok) {
        // E4: stage dQ, dK, dV (every MMA is done: all tiles are free) and store them
        stage(TB_DQ, SB_ST_Q);
        stage(TB_DK, SB_ST_K);
        stage(TB_DV, SB_ST_V);
        ptx::fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            ptx::tma_store_3d(&tdq, sm + SB_ST_Q, 0, t0, bh);
            ptx::tma_store_3d(&tdq, sm + SB_ST_Q + C * 128, 32, t0, bh);
            ptx::tma_store_3d(&tdk, sm + SB_ST_K, 0, t0, bh);
            ptx::tma_store_3d(&tdk, sm + SB_ST_K + C * 128, 32, t0, bh);
            ptx::tma_store_3d(&tdv, sm + SB_ST_V, 0, t0, bh);
            ptx::tma_store_3d(&tdv, sm + SB_ST_V + C * 128, 32, t0, bh);
            ptx::bulk_commit();
            ptx::bulk_wait_all();
        }
    } else if (tid == 0) {
        set_status(p.status, DEV_TIMEOUT);
        // let the loads and MMAs already in flight land before TMEM and shared memory are released
        ptx::mbar_wait(bar_load, 0, 100000000ull);
        if (round > 0) {
            ptx::umma_commit(bar_mma);
            ptx::mbar_wait(bar_mma, mma_phase, 100000000ull);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, TB_COLS);
}

// ---------------------------------------------------------------- adjoint terms
// Per 128-token chunk, the terms of the adjoint recurrences of the state (exclusive suffix sums
// of them, taken by the CUDA-core kernels, give dR' and dS'):
//     Y = Q^T dO,   C = Q^T V,   U = Q^T (dW Q),   dW = L (.) dO V^T,
// as fp32 64 x 64 matrices into the chunk's slot [Y | U | C].  The Q^T products are one M = 128
// product each over the Q and V tiles stacked ([Q^T ; V^T] X; rows 0-63 kept).  Three rounds:
// dO enters as two bf16 terms (hi + lo), as in the gradient kernel: Y feeds dR' and every dq.
//   R1: dW* = dO V^T, [Y ; .] = [Q^T ; V^T] dO, [C ; .] = [Q^T ; V^T] V  -> E1: dW masked to bf16
//   R2: G = dW Q                                                           -> E2: G to bf16
//   R3: [U ; .] = [Q^T ; V^T] G                                             -> E3: Y, U, C stored
constexpr uint32_t SA_Q = 0, SA_V = TILE, SA_O = 2 * TILE, SA_OL = 3 * TILE, SA_DW = 4 * TILE;
constexpr uint32_t SA_BAR = 6 * TILE;
constexpr uint32_t TSMEM_BYTES = SA_BAR + 64 + 1024;
constexpr uint32_t SA_OF = SA_DW;               // dO (fp32 boxes) before dW is written
constexpr uint32_t SA_G = SA_O;                 // G over dO (read by R1 only)
constexpr uint32_t TT_DW = 0, TT_G = 0, TT_U = 64, TT_Y = 128, TT_C = 192, TT_COLS = 256;

__global__ void __launch_bounds__(BNT, 2)
k_bwd_terms(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tv,
            const __grid_constant__ CUtensorMap tdo, BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + SA_BAR);
    uint64_t* bar_mma = bar_load + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    const int t0 = chunk * C;
    if (tid == 0) {
        ptx::mbar_init(bar_load, 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        ptx::mbar_arrive_expect_tx(bar_load, 4 * TILE);
        ptx::tma_load_3d(sm + SA_Q, &tq, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + SA_V, &tv, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + SA_OF, &tdo, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + SA_OF + C * 128, &tdo, bar_load, 32, t0, bh);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, TT_COLS);
        ptx::tmem_relinquish();
    }
    bool ok = ptx::mbar_wait(bar_load, 0);
    {
        const float4* box = reinterpret_cast<const float4*>(sm + SA_OF + half * (C * 128) + row * 128);
        float x[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 f = box[j ^ (row & 7)];
            x[4 * j] = f.x; x[4 * j + 1] = f.y; x[4 * j + 2] = f.z; x[4 * j + 3] = f.w;
        }
        split_row(sm + SA_O, sm + SA_OL, row, half * 32, x);
    }
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sb = ptx::smem_u32(sm);
    constexpr uint32_t I_128_KK = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t I_64_KM = ptx::idesc_bf16(128, 64, false, true);
    constexpr uint32_t I_64_MM = ptx::idesc_bf16(128, 64, true, true);
    auto k1 = [](uint64_t d0, int s) { return d0 + (uint64_t)(s * 2); };
    auto k2 = [](uint64_t d0, int s) { return d0 + (uint64_t)(((s >> 2) * TILE + (s & 3) * 32) >> 4); };
    auto mn = [](uint64_t d0, int s) { return d0 + (uint64_t)(s * 128); };
    const uint64_t dQV = mdesc(sb + SA_Q, SA_V - SA_Q, 0);      // [Q^T ; V^T], MN-major, M = 128
    auto stacked = [&](uint32_t d, uint32_t b, bool acc) {        // [Q^T ; V^T] X, X a [tok][64] tile
        const uint64_t db = mdesc(sb + b, TILE, 0);
        for (int s = 0; s < 8; ++s)
            ptx::umma_bf16(tmem + d, mn(dQV, s), mn(db, s), I_64_MM, (acc || s > 0) ? 1u : 0u);
    };
    uint32_t mma_phase = 0;
    auto commit_wait = [&]() -> bool {
        bool good = true;
        ptx::tc_fence_before();
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
    int round = 0;
    if (ok) {
        if (tid == 0) {                      // R1
            const uint64_t dO = kdesc(sb + SA_O, 0), dOL = kdesc(sb + SA_OL, 0), dV = kdesc(sb + SA_V, 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TT_DW, k1(dO, s), k1(dV, s), I_128_KK, s > 0 ? 1u : 0u);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TT_DW, k1(dOL, s), k1(dV, s), I_128_KK, 1u);
            stacked(TT_Y, SA_O, false);
            stacked(TT_Y, SA_OL, true);
            stacked(TT_C, SA_V, false);
        }
        round = 1;
        ok = commit_wait();
    }
    if (ok) {
        // E1: dW masked (j <= t) to the K-major [t][j] tile
        const int b0 = 2 * half;
        float v0[32], v1[32];
        if (b0 + 1 <= quad) {
            ptx::tmem_ld32x2(tmem + lane_base + TT_DW + 32 * b0, tmem + lane_base + TT_DW + 32 * (b0 + 1), v0, v1);
            if (b0 + 1 == quad) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i > lane) v1[i] = 0.f;
            }
            st_row32(sm + SA_DW, row, 32 * b0, v0);
            st_row32(sm + SA_DW, row, 32 * (b0 + 1), v1);
        } else if (b0 == quad) {
            ptx::tmem_ld32(tmem + lane_base + TT_DW + 32 * b0, v0);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (i > lane) v0[i] = 0.f;
            st_row32(sm + SA_DW, row, 32 * b0, v0);
            st_row32_zero(sm + SA_DW, row, 32 * (b0 + 1));
        } else {
            st_row32_zero(sm + SA_DW, row, 32 * b0);
            st_row32_zero(sm + SA_DW, row, 32 * (b0 + 1));
        }
        sync_for_mma();
        if (tid == 0) {                      // R2: G = dW Q
            const uint64_t dA = kdesc2(sb + SA_DW, 0), dB = mdesc(sb + SA_Q, TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + TT_G, k2(dA, s), mn(dB, s), I_64_KM, s > 0 ? 1u : 0u);
        }
        round = 2;
        ok = commit_wait();
    }
    if (ok) {
        float v[32];
        ptx::tmem_ld32(tmem + lane_base + TT_G + 32 * half, v);
        st_row32(sm + SA_G, row, 32 * half, v);
        sync_for_mma();
        if (tid == 0) stacked(TT_U, SA_G, false);   // R3
        round = 3;
        ok = commit_wait();
    }
    if (ok && quad < 2) {
        // E3: rows 0-63 (Q features) of Y, U, C into the slot, this thread's half row of each
        float* slot = p.terms + ((size_t)bh * p.NSp + chunk) * BW_SIZE;
        const uint32_t cols[3] = {TT_Y, TT_U, TT_C};
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + cols[m] + 32 * half, v);
            float4* dst = reinterpret_cast<float4*>(slot + m * D * D + row * D + 32 * half);
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
    }
    if (!ok && tid == 0) {
        set_status(p.status, DEV_TIMEOUT);
        ptx::mbar_wait(bar_load, 0, 100000000ull);
        if (round > 0) {
            ptx::umma_commit(bar_mma);
            ptx::mbar_wait(bar_mma, mma_phase, 100000000ull);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, TT_COLS);
}

}  // namespace

static int slots_per_head(int T) {
    int n = 1;
    while (n < (T + C - 1) / C) n *= 2;
    return n;
}

cudaError_t bwd_terms(const void* q, const void* v, const float* dout, float* terms, int BH, int T, int* status,
                      cudaStream_t st) {
    CUtensorMap mq, mv, mdo;
    if (!make_map(&mq, q, T, BH) || !make_map(&mv, v, T, BH) || !make_map_out(&mdo, const_cast<float*>(dout), T, BH))
        return cudaErrorInvalidValue;
    BwdParams prm{};
    prm.T = T;
    prm.NSp = slots_per_head(T);
    prm.terms = terms;
    prm.status = status;
    cudaError_t e = set_smem(k_bwd_terms, (int)TSMEM_BYTES);
    if (e != cudaSuccess) return e;
    k_bwd_terms<<<dim3((T + C - 1) / C, BH), BNT, TSMEM_BYTES, st>>>(mq, mv, mdo, prm);
    return cudaGetLastError();
}

cudaError_t bwd_out(const void* q, const void* k, const void* v, const float* dout, const float* pre,
                    const float* bw, float* dq, float* dk, float* dv, int BH, int T, int* status,
                    cudaStream_t st) {
    CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
    if (!make_map(&mq, q, T, BH) || !make_map(&mk, k, T, BH) || !make_map(&mv, v, T, BH) ||
        !make_map_out(&mdo, const_cast<float*>(dout), T, BH) || !make_map_out(&mdq, dq, T, BH) ||
        !make_map_out(&mdk, dk, T, BH) || !make_map_out(&mdv, dv, T, BH))
        return cudaErrorInvalidValue;
    BwdParams prm{};
    prm.T = T;
    prm.NSp = slots_per_head(T);
    prm.pre = pre;
    prm.bw = bw;
    prm.status = status;
    cudaError_t e = set_smem(k_bwd_tc, (int)BSMEM_BYTES);
    if (e != cudaSuccess) return e;
    k_bwd_tc<<<dim3((T + C - 1) / C, BH), BNT, BSMEM_BYTES, st>>>(mq, mk, mv, mdo, mdq, mdk, mdv, prm);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace hla
