// tcgen05 kernels of the plain second-order forward with fp32 inputs at d = dv = 32, over
// 128-token chunks: the chunk summaries, then the output with the prefix of the summaries
// folded into each output CTA (two launches).
//
// "Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 1 (second
// order) and Metodología 4 (chunked scan).  Summary of a chunk from the zero state (the
// CUDA-core slot layout, S, C, R at matrices 0, 1, 2; the plain op needs no normaliser vectors):
//     S = K^T K,   C = Q^T V,   R = K^T (A^T V),   A = L (.) Q K^T.
// Prefix of chunk n (the factored form of the semidirect combine):
//     S0 = sum_{l<n} S_l,   R0 = sum_{l<n} R_l + sum_{m<n-1} S_m Csuf(m+1),
//     Csuf(m+1) = sum_{m<l<n} C_l.
// Output:  P = Q S0,   W = L (.) (P Q^T + A A^T),   O = Q R0 + W V.
// fp32 accuracy from bf16 tensor-core products of two- and three-term splits, as in the third
// order's kernels (tc_hla3.cu): the output's scores take three terms, everything else two (an
// fp64 emulation gave a 7.6e-6 row error at T = 256 and 1e-5 at T = 4096).
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

constexpr int D2 = 32;
constexpr int NT2 = 256;
constexpr int SLOT_MATS = 3;                 // S, C, R

__device__ __forceinline__ void put16f(uint8_t* tile, uint32_t atom, int row, int c0, const float (&v)[16]) {
    st_row16(tile, atom, row, c0, v);
}

// one 64 x 64 block of hi / lo partial products at TMEM column `col`, lanes lane0 .. lane0+63,
// summed into a 32 x 32 result (staged through `stg`, [64][68] fp32) and written to `dst`
struct BlockSum {
    float* stg;
    __device__ void run(uint32_t tmem, uint32_t lane_base, int row, int half, int tid, uint32_t col, int lane0,
                        float* dst) const {
        constexpr int SLD = 68;
        if (row >= lane0 && row < lane0 + 64) {
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + col + half * 32, v);
            float* p = stg + (row - lane0) * SLD + half * 32;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(p + 4 * j) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
        __syncthreads();
        for (int e = tid; e < D2 * D2; e += NT2) {
            const int a = e / D2, b = e % D2;
            dst[e] = stg[a * SLD + b] + stg[a * SLD + 32 + b] + stg[(32 + a) * SLD + b] + stg[(32 + a) * SLD + 32 + b];
        }
        __syncthreads();
    }
};

struct F2Params {
    int T, NC, slot;   // chunk l's summary of head bh at sums + (bh NC + l) slot
    float* sums;
    float* o;
    int* status;
};

// ---------------------------------------------------------------- summaries
//   R1  A* = Q K^T (concatenated K axis);  D1 = [KK ; QQ] [KK | VV]   -> E1: A hi / lo tiles;
//       S (rows K, columns K) and C (rows Q, columns V) from D1
//   R2  Y = A^T [V_hi | V_lo]                                          -> E2: [Y_hi | Y_lo]
//   R3  D3 = [KK ; QQ] [YY]                                            -> E3: R (rows K) from D3
constexpr uint32_t U_QC = 0;                    // [q_hi | q_lo | q_hi | 0]; [Y_hi | Y_lo] after R1
constexpr uint32_t U_KC = U_QC + 2 * TILE;      // [k_hi | k_hi | k_lo | 0]; fp32 staging after R1
constexpr uint32_t U_KK = U_KC + 2 * TILE;      // [K_hi | K_lo] token rows  } one N = 128 operand
constexpr uint32_t U_VV = U_KK + TILE;          // [V_hi | V_lo]             }
constexpr uint32_t U_QQ = U_VV + TILE;          // [Q_hi | Q_lo]
constexpr uint32_t U_AH = U_QQ + TILE;          // A_hi [128][128], two atoms
constexpr uint32_t U_AL = U_AH + 2 * TILE;
constexpr uint32_t U_BAR = U_AL + 2 * TILE;
constexpr uint32_t U_BYTES = U_BAR + 64 + 1024;

__global__ void __launch_bounds__(NT2, 1)
k_hla2f_sum(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v, F2Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    // the output walk may be scheduled once every summary CTA has started
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int t0 = chunk * C;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + U_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
    float* out = p.sums + ((size_t)bh * p.NC + chunk) * p.slot;
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 256);
        ptx::tmem_relinquish();
    }
    {
        const int r = tid >> 1, h = tid & 1;
        const bool in = t0 + r < p.T;
        const size_t base = ((size_t)bh * p.T + t0 + r) * D2 + 16 * h;
        float xq[16], xk[16], xv[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 a = in ? *reinterpret_cast<const float4*>(q + base + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 b = in ? *reinterpret_cast<const float4*>(k + base + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 c = in ? *reinterpret_cast<const float4*>(v + base + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
            xq[4 * j] = a.x; xq[4 * j + 1] = a.y; xq[4 * j + 2] = a.z; xq[4 * j + 3] = a.w;
            xk[4 * j] = b.x; xk[4 * j + 1] = b.y; xk[4 * j + 2] = b.z; xk[4 * j + 3] = b.w;
            xv[4 * j] = c.x; xv[4 * j + 1] = c.y; xv[4 * j + 2] = c.z; xv[4 * j + 3] = c.w;
        }
        float hi[16], lo[16], z[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            hi[j] = bf16_hi(xq[j]);
            lo[j] = xq[j] - hi[j];
            z[j] = 0.f;
        }
        put16f(sm + U_QC, TILE, r, 16 * h, hi);
        put16f(sm + U_QC, TILE, r, 32 + 16 * h, lo);
        put16f(sm + U_QC, TILE, r, 64 + 16 * h, hi);
        put16f(sm + U_QC, TILE, r, 96 + 16 * h, z);
        put16f(sm + U_QQ, TILE, r, 16 * h, hi);
        put16f(sm + U_QQ, TILE, r, 32 + 16 * h, lo);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            hi[j] = bf16_hi(xk[j]);
            lo[j] = xk[j] - hi[j];
        }
        put16f(sm + U_KC, TILE, r, 16 * h, hi);
        put16f(sm + U_KC, TILE, r, 32 + 16 * h, hi);
        put16f(sm + U_KC, TILE, r, 64 + 16 * h, lo);
        put16f(sm + U_KC, TILE, r, 96 + 16 * h, z);
        put16f(sm + U_KK, TILE, r, 16 * h, hi);
        put16f(sm + U_KK, TILE, r, 32 + 16 * h, lo);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            hi[j] = bf16_hi(xv[j]);
            lo[j] = xv[j] - hi[j];
        }
        put16f(sm + U_VV, TILE, r, 16 * h, hi);
        put16f(sm + U_VV, TILE, r, 32 + 16 * h, lo);
    }
#pragma unroll
    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32)
        if (c0 > quad * 32 + 31) {
            st_row32_zero(sm + U_AH, row, c0);
            st_row32_zero(sm + U_AL, row, c0);
        }
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sb = ptx::smem_u32(sm);
    constexpr uint32_t I_QK = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t I_M128 = ptx::idesc_bf16(128, 128, true, true);
    constexpr uint32_t I_M64 = ptx::idesc_bf16(128, 64, true, true);
    uint32_t phase = 0;
    auto mma_wait = [&]() {
        bool good = true;
        if (tid == 0) {
            ptx::umma_commit(bar);
            good = ptx::mbar_wait(bar, phase);
        }
        phase ^= 1;
        good = __syncthreads_and(good) != 0;
        ptx::tc_fence_after();
        return good;
    };
    auto sync_mma = [&]() {
        ptx::tmem_st_wait();
        ptx::fence_proxy_async();
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
    };
    const BlockSum bs{reinterpret_cast<float*>(sm + U_KC)};
    bool ok = true;
    if (tid == 0) {
        for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + 0, kdesc2(sb + U_QC, s), kdesc2(sb + U_KC, s), I_QK, s > 0);
        const uint64_t dA = mdesc(sb + U_KK, U_QQ - U_KK, 0), dB = mdesc(sb + U_KK, TILE, 0);
        for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + 128, dA + (uint64_t)(s * 128), dB + (uint64_t)(s * 128), I_M128, s > 0);
    }
    ok = mma_wait();                                                  // R1 done
    if (ok) {
        // E1: A = L (.) A* to hi / lo tiles
        float v[32], hi[32], lo[32];
#pragma unroll
        for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
            if (c0 > quad * 32 + 31) continue;
            ptx::tmem_ld32(tmem + lane_base + c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float x = (c0 + i <= row) ? v[i] : 0.f;
                hi[i] = bf16_hi(x);
                lo[i] = x - hi[i];
            }
            st_row32(sm + U_AH, row, c0, hi);
            st_row32(sm + U_AL, row, c0, lo);
        }
        sync_mma();
        if (tid == 0) {
            const uint64_t dV = mdesc(sb + U_VV, TILE, 0);
            const uint64_t dAH = mdesc(sb + U_AH, TILE, 0), dAL = mdesc(sb + U_AL, TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + 0, dAH + (uint64_t)(s * 128), dV + (uint64_t)(s * 128), I_M64, s > 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + 0, dAL + (uint64_t)(s * 128), dV + (uint64_t)(s * 128), I_M64, 1);
        }
        bs.run(tmem, lane_base, row, half, tid, 128, 0, out);            // S = K^T K
        bs.run(tmem, lane_base, row, half, tid, 192, 64, out + D2 * D2); // C = Q^T V
        ok = mma_wait();                                              // R2 done
    }
    if (ok) {
        // E2: Y = A^T V (the sum of its hi and lo halves) to [Y_hi | Y_lo] over the concatenated Q
        float a[16], b[16], hi[16], lo[16];
        ptx::tmem_ld16(tmem + lane_base + 16 * half, a);
        ptx::tmem_ld16(tmem + lane_base + 32 + 16 * half, b);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float y = a[i] + b[i];
            hi[i] = bf16_hi(y);
            lo[i] = y - hi[i];
        }
        put16f(sm + U_QC, TILE, row, 16 * half, hi);
        put16f(sm + U_QC, TILE, row, 32 + 16 * half, lo);
        sync_mma();
        if (tid == 0) {
            const uint64_t dA = mdesc(sb + U_KK, U_QQ - U_KK, 0), dY = mdesc(sb + U_QC, TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + 64, dA + (uint64_t)(s * 128), dY + (uint64_t)(s * 128), I_M64, s > 0);
        }
        ok = mma_wait();                                              // R3 done
    }
    if (ok) {
        bs.run(tmem, lane_base, row, half, tid, 64, 0, out + 2 * D2 * D2);   // R = K^T Y
        for (int e = tid; e < p.slot - SLOT_MATS * D2 * D2; e += NT2) out[SLOT_MATS * D2 * D2 + e] = 0.f;
    } else if (tid == 0) {
        set_status(p.status, DEV_TIMEOUT);
        ptx::umma_commit(bar);
        ptx::mbar_wait(bar, phase, 100000000ull);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- output
//   prologue: fold the slots before this chunk (CUDA cores, fp32)
//   R1  [A* | P | Q R0] = [Q] [K ; S0^T ; R0^T]^T  (N = 192, K = 192 concatenated, three terms)
//       -> E1: A hi / lo pairs and tiles; P to [p1 | p2 | p1] pairs
//   R2  W = P Q^T + A A^T                           -> E2: W = L (.) W to hi / lo pairs
//   R3  D_o = W [V_hi | V_lo]                       -> E3: O = Q R0 + D_o(hi) + D_o(lo)
constexpr uint32_t BROWS2 = C + 2 * D2;           // K rows, S0^T, R0^T
constexpr uint32_t BATOM2 = BROWS2 * 128;         // 24 KB
constexpr uint32_t O_QC = 0;                      // [q1 | q1 | q2 | q1 | q2 | q3], three atoms (48 KB)
constexpr uint32_t O_BC = O_QC + 3 * TILE;        // [y1 | y2 | y1 | y3 | y2 | y1], three atoms of 192 rows
constexpr uint32_t O_AH = O_BC + 3 * BATOM2;      // A_hi [128][128]; the fold's fp32 staging before E1
constexpr uint32_t O_AL = O_AH + 2 * TILE;
constexpr uint32_t O_VV = O_AL + 2 * TILE;        // [V_hi | V_lo]
constexpr uint32_t O_BAR = O_VV + TILE;
constexpr uint32_t O_BYTES = O_BAR + 64 + 1024;
constexpr uint32_t TO_X = 0, TO_P = 128, TO_QR = 160, TO_AH = 192, TO_AL = 256, TO_PC = 320, TO_D = 384;

__global__ void __launch_bounds__(NT2, 1)
k_hla2f_out(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v, F2Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    const int t0 = chunk * C;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + O_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    auto put_b = [&](int r, int h, const float (&y1)[16], const float (&y2)[16], const float (&y3)[16]) {
        put16f(sm + O_BC, BATOM2, r, 16 * h, y1);
        put16f(sm + O_BC, BATOM2, r, 32 + 16 * h, y2);
        put16f(sm + O_BC, BATOM2, r, 64 + 16 * h, y1);
        put16f(sm + O_BC, BATOM2, r, 96 + 16 * h, y3);
        put16f(sm + O_BC, BATOM2, r, 128 + 16 * h, y2);
        put16f(sm + O_BC, BATOM2, r, 160 + 16 * h, y1);
    };
    {
        const int r = tid >> 1, h = tid & 1;
        const bool in = t0 + r < p.T;
        const size_t base = ((size_t)bh * p.T + t0 + r) * D2 + 16 * h;
        float xq[16], xk[16], xv[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 a = in ? *reinterpret_cast<const float4*>(q + base + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 b = in ? *reinterpret_cast<const float4*>(k + base + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 c = in ? *reinterpret_cast<const float4*>(v + base + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
            xq[4 * j] = a.x; xq[4 * j + 1] = a.y; xq[4 * j + 2] = a.z; xq[4 * j + 3] = a.w;
            xk[4 * j] = b.x; xk[4 * j + 1] = b.y; xk[4 * j + 2] = b.z; xk[4 * j + 3] = b.w;
            xv[4 * j] = c.x; xv[4 * j + 1] = c.y; xv[4 * j + 2] = c.z; xv[4 * j + 3] = c.w;
        }
        float x1[16], x2[16], x3[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) bf16_split3(xq[j], x1[j], x2[j], x3[j]);
        put16f(sm + O_QC, TILE, r, 16 * h, x1);
        put16f(sm + O_QC, TILE, r, 32 + 16 * h, x1);
        put16f(sm + O_QC, TILE, r, 64 + 16 * h, x2);
        put16f(sm + O_QC, TILE, r, 96 + 16 * h, x1);
        put16f(sm + O_QC, TILE, r, 128 + 16 * h, x2);
        put16f(sm + O_QC, TILE, r, 160 + 16 * h, x3);
#pragma unroll
        for (int j = 0; j < 16; ++j) bf16_split3(xk[j], x1[j], x2[j], x3[j]);
        put_b(r, h, x1, x2, x3);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            x1[j] = bf16_hi(xv[j]);
            x2[j] = xv[j] - x1[j];
        }
        put16f(sm + O_VV, TILE, r, 16 * h, x1);
        put16f(sm + O_VV, TILE, r, 32 + 16 * h, x2);
    }
    // ---- the carried-in S0 and R0: fold the summaries of chunks 0 .. chunk-1 of this head.
    // Thread (r, c) keeps a 2 x 2 block; S0 = sum S_l, R0 = sum R_l + sum_m S_m Csuf(m+1).
    float* Ssum = reinterpret_cast<float*>(sm + O_AH);           // S0 [32][32] (fp32, over A_hi)
    float* Rsum = Ssum + D2 * D2;                                // R0
    float* Csuf = Rsum + D2 * D2;                                // Csuf(m+1)
    float* Sm = Csuf + D2 * D2;                                  // S_m
    {
        const int r = 2 * (tid >> 4), c = 2 * (tid & 15);
        float s0[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, r0[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, cs[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        const int n = chunk;
        if (n > 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");       // the summaries
            const float* s0p = p.sums + (size_t)bh * p.NC * p.slot;
            for (int m = n - 1; m >= 0; --m) {
                const float* sl = s0p + (size_t)m * p.slot;
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const float x = sl[(r + a) * D2 + c + b];
                        s0[a][b] += x;
                        r0[a][b] += sl[2 * D2 * D2 + (r + a) * D2 + c + b];
                        Sm[(r + a) * D2 + c + b] = x;
                        Csuf[(r + a) * D2 + c + b] = cs[a][b];
                    }
                __syncthreads();
                if (m < n - 1) {                                      // R0 += S_m Csuf(m+1)
#pragma unroll 8
                    for (int kk = 0; kk < D2; ++kk) {
                        const float c0 = Csuf[kk * D2 + c], c1 = Csuf[kk * D2 + c + 1];
#pragma unroll
                        for (int a = 0; a < 2; ++a) {
                            const float sv = Sm[(r + a) * D2 + kk];
                            r0[a][0] = fmaf(sv, c0, r0[a][0]);
                            r0[a][1] = fmaf(sv, c1, r0[a][1]);
                        }
                    }
                }
                __syncthreads();
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int b = 0; b < 2; ++b) cs[a][b] += sl[D2 * D2 + (r + a) * D2 + c + b];
            }
        }
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                Ssum[(r + a) * D2 + c + b] = s0[a][b];
                Rsum[(r + a) * D2 + c + b] = r0[a][b];
            }
    }
    __syncthreads();
    if (tid < 2 * 2 * D2) {
        // B rows 128 + 32 m + g: column g of S0 (m = 0) or R0 (m = 1), split as the key rows
        const int m = tid / (2 * D2), g = (tid >> 1) % D2, h = tid & 1;
        const float* M = m == 0 ? Ssum : Rsum;
        float y1[16], y2[16], y3[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) bf16_split3(M[(16 * h + j) * D2 + g], y1[j], y2[j], y3[j]);
        put_b(C + m * D2 + g, h, y1, y2, y3);
    }
    __syncthreads();                                                  // the fold staging is read
#pragma unroll
    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32)
        if (c0 > quad * 32 + 31) {
            st_row32_zero(sm + O_AH, row, c0);
            st_row32_zero(sm + O_AL, row, c0);
        }
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sb = ptx::smem_u32(sm);
    auto st_pairs = [&](uint32_t tcol, const float* x) {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = ptx::pack_bf16(x[2 * i], x[2 * i + 1]);
        ptx::tmem_st16u(tmem + lane_base + tcol, r);
    };
    {
        uint32_t zr[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) zr[i] = 0u;
#pragma unroll
        for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32)
            if (c0 > quad * 32 + 31) {
                ptx::tmem_st16u(tmem + lane_base + TO_AH + c0 / 2, zr);
                ptx::tmem_st16u(tmem + lane_base + TO_AL + c0 / 2, zr);
            }
    }
    constexpr uint32_t I_R1 = ptx::idesc_bf16(128, 192, false, false);
    constexpr uint32_t I_W = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t I_KM = ptx::idesc_bf16(128, 64, false, true);
    uint32_t phase = 0;
    auto mma_wait = [&]() {
        bool good = true;
        if (tid == 0) {
            ptx::umma_commit(bar);
            good = ptx::mbar_wait(bar, phase);
        }
        phase ^= 1;
        good = __syncthreads_and(good) != 0;
        ptx::tc_fence_after();
        return good;
    };
    auto sync_mma = [&]() {
        ptx::tmem_st_wait();
        ptx::fence_proxy_async();
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
    };
    sync_mma();
    bool ok = true;
    if (tid == 0) {
        for (int s = 0; s < 12; ++s)
            ptx::umma_bf16(tmem + TO_X, kdesc2(sb + O_QC, s),
                           ptx::desc_sw128(sb + O_BC + (s >> 2) * BATOM2 + (s & 3) * 32, 16, 1024), I_R1, s > 0);
    }
    ok = mma_wait();                                                  // R1 done
    if (ok) {
        float v[32], hi[32], lo[32];
#pragma unroll
        for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
            if (c0 > quad * 32 + 31) continue;
            ptx::tmem_ld32(tmem + lane_base + TO_X + c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float x = (c0 + i <= row) ? v[i] : 0.f;
                hi[i] = bf16_hi(x);
                lo[i] = x - hi[i];
            }
            st_pairs(TO_AH + c0 / 2, hi);
            st_pairs(TO_AL + c0 / 2, lo);
            st_row32(sm + O_AH, row, c0, hi);
            st_row32(sm + O_AL, row, c0, lo);
        }
        ptx::tmem_ld32(tmem + lane_base + TO_P, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            hi[i] = bf16_hi(v[i]);
            lo[i] = v[i] - hi[i];
        }
        if (half == 0) {
            st_pairs(TO_PC, hi);
            st_pairs(TO_PC + 32, hi);
        } else {
            st_pairs(TO_PC + 16, lo);
        }
        sync_mma();
        if (tid == 0) {
            for (int s = 0; s < 6; ++s) ptx::umma_bf16_ts(tmem + TO_X, tmem + TO_PC + 8 * s, kdesc2(sb + O_QC, s), I_W, s > 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TO_X, tmem + TO_AH + 8 * s, kdesc2(sb + O_AH, s), I_W, 1);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TO_X, tmem + TO_AH + 8 * s, kdesc2(sb + O_AL, s), I_W, 1);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TO_X, tmem + TO_AL + 8 * s, kdesc2(sb + O_AH, s), I_W, 1);
        }
        ok = mma_wait();                                              // R2 done
    }
    if (ok) {
        float v[32], hi[32], lo[32];
#pragma unroll
        for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
            if (c0 > quad * 32 + 31) continue;
            ptx::tmem_ld32(tmem + lane_base + TO_X + c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float x = (c0 + i <= row) ? v[i] : 0.f;
                hi[i] = bf16_hi(x);
                lo[i] = x - hi[i];
            }
            st_pairs(TO_AH + c0 / 2, hi);
            st_pairs(TO_AL + c0 / 2, lo);
        }
        sync_mma();
        if (tid == 0) {
            const uint64_t dV = mdesc(sb + O_VV, TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TO_D, tmem + TO_AH + 8 * s, dV + (uint64_t)(s * 128), I_KM, s > 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TO_D, tmem + TO_AL + 8 * s, dV + (uint64_t)(s * 128), I_KM, 1);
        }
        ok = mma_wait();                                              // R3 done
    }
    if (ok) {
        float a[16], b[16], c[16];
        ptx::tmem_ld16(tmem + lane_base + TO_QR + 16 * half, a);
        ptx::tmem_ld16(tmem + lane_base + TO_D + 16 * half, b);
        ptx::tmem_ld16(tmem + lane_base + TO_D + 32 + 16 * half, c);
        if (t0 + row < p.T) {
            float4* dst = reinterpret_cast<float4*>(p.o + ((size_t)bh * p.T + t0 + row) * D2 + 16 * half);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                dst[j] = make_float4(a[4 * j] + b[4 * j] + c[4 * j], a[4 * j + 1] + b[4 * j + 1] + c[4 * j + 1],
                                     a[4 * j + 2] + b[4 * j + 2] + c[4 * j + 2], a[4 * j + 3] + b[4 * j + 3] + c[4 * j + 3]);
        }
    } else if (tid == 0) {
        set_status(p.status, DEV_TIMEOUT);
        ptx::umma_commit(bar);
        ptx::mbar_wait(bar, phase, 100000000ull);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace

int hla2f_max_chunks() { return 64; }

cudaError_t hla2f_forward(const float* q, const float* k, const float* v, float* sums, int slot_floats, float* o,
                          int BH, int T, int* status, cudaStream_t st, cudaEvent_t* ev) {
    const int NC = (T + C - 1) / C;
    if (NC > hla2f_max_chunks()) return cudaErrorInvalidValue;
    F2Params prm;
    prm.T = T;
    prm.NC = NC;
    prm.slot = slot_floats;
    prm.sums = sums;
    prm.o = o;
    prm.status = status;
    cudaError_t e;
    if ((e = set_smem(k_hla2f_sum, U_BYTES)) != cudaSuccess) return e;
    if ((e = set_smem(k_hla2f_out, O_BYTES)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    k_hla2f_sum<<<dim3(NC, BH), NT2, U_BYTES, st>>>(q, k, v, prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[2], st)) != cudaSuccess) return e;
    // a programmatic dependent of the summaries: chunk 0 needs none, the others fold them
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(NC, BH);
    cfg.blockDim = dim3(NT2);
    cfg.dynamicSmemBytes = O_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, k_hla2f_out, q, k, v, prm)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[3], st)) != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace tc
}  // namespace hla
