// tcgen05 path for the second-order forward with per-head decay (bf16 inputs, d = dv = 64,
// not ratio-normalised).
//
// "Higher-order Linear Attention" summary (gist.science 2510.27258), Contribuciones 2 (masked
// operators with exponential decay) and Metodología 4 (chunked scan).  Decay reading: before
// each token's update every state is multiplied by gamma_h, then the undecayed updates run:
//     S_t = g S_{t-1} + k k^T,   C_t = g C_{t-1} + q v^T,   G_t = g G_{t-1} + k k^T (g C_{t-1}),
//     o_t = q_t^T (S_t C_t - G_t).
//
// Chunk algebra.  c = 128 tokens, local index tau.  Gam_tau = g^(tau+1), lam_tau = g^(c-1-tau),
// rho = g^c.  A* = Q K^T (no mask), A = L (.) A*, U = strict upper part of A*,
// At[tau][i] = g^(tau-i) A*[tau][i] for i <= tau, H[tau][i] = (g^(tau-i) - 1) A*[tau][i] for
// i < tau (0 elsewhere).
//   summary of a chunk from the zero state:
//     S = K^T Lam K,   C = Q^T Lam V,   Khat = K^T K,   G = K^T (U^T Lam V)
//   state entering chunk l (every earlier chunk is full):
//     S0(l+1) = rho S0(l) + S_l,   C0(l+1) = rho C0(l) + C_l,
//     G0(l+1) = rho G0(l) + G_l + rho Khat_l C0(l)
//   output of a chunk with carried-in (S0, C0, G0), P = Q S0:
//     W = Dg (.) L (.) (Gam P Q^T + At A^T + H U^T),   Dg[tau][j] = g^(tau-j)
//     O = W V + Gam (Gam P + H K) C0 - Gam (Q G0)
// The cross terms are the carried-in S0 times the chunk's C (through P Q^T), the chunk's
// decayed-minus-undecayed key moment times C0 (through H K), and the carried-in
// Gam S0 C0 - G0 (through Gam P C0 and Q G0).
// Inside the chunk, the pair weight g^(tau-i) - [i > j] is split by i <= j (At A^T) and i > j
// (H U^T), so every weight is applied in fp32 before the one rounding of an operand to bf16:
// writing it as a difference of separately rounded products would lose the weight to bf16
// rounding at strong decay (H A*^T + A A^T) or at weak decay (At A*^T - A U^T).
//
// Kernels (every chunk independent):
//   k_dec_summary (tcgen05, two CTAs per SM)   chunk summaries (S, C, Khat, G^T), fp32
//   k_dec_prefix_sc, k_dec_cross, k_dec_prefix_g (CUDA cores)
//                                               in place: S0, C0; Y^T = G^T + rho C0^T Khat;
//                                               G0^T (Khat is symmetric)
//   k_dec_output (tcgen05, persistent: one CTA per SM over the chunks)
//                                               turns (S0, C0, G0^T) into bf16 operand tiles
//                                               and forms O, written by TMA bulk tensor stores
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

constexpr int DNT = 256;                  // 8 warps, two per TMEM lane quadrant
constexpr int DSUM = 4 * D * D;           // chunk state: S, C, Khat, G^T (then Y^T, then G0^T)
constexpr uint32_t QTILE = D * D * 2;     // one 64 x 64 bf16 tile = 8 KB

struct DParams {
    int T, BH, H, NC;
    const float* gamma;
    float* sums;      // per head NC x DSUM fp32, in the blocked layout of dsum()
    int* status;
};

// Chunk states of a head are stored in blocks of 32 consecutive elements of one matrix,
// chunk-major inside a block: element e (0 .. DSUM) of chunk l sits at
//     sums + bh NC DSUM + (e / 32) NC 32 + l 32 + e % 32.
// A warp that follows one block across the chunks reads one contiguous run, and one chunk's
// state is 512 whole 128-byte lines.
__device__ __forceinline__ float* dsum(const DParams& p, int bh, int l, int e) {
    return p.sums + (size_t)bh * p.NC * DSUM + (size_t)(e >> 5) * p.NC * 32 + l * 32 + (e & 31);
}

// g^n for n >= 0 (binary powering).
__device__ __forceinline__ float gpow_n(float g, int n) {
    float r = 1.f, b = g;
    while (n) {
        if (n & 1) r *= b;
        b *= b;
        n >>= 1;
    }
    return r;
}

// Shared bounded commit-and-wait of the issuing thread; the block agrees on the result.
struct MmaSync {
    uint64_t* bar;
    uint32_t phase;
    __device__ bool commit_wait(bool issuer) {
        bool good = true;
        if (issuer) {
            ptx::umma_commit(bar);
            good = ptx::mbar_wait(bar, phase);
        }
        phase ^= 1;
        good = __syncthreads_and(good) != 0;
        ptx::tc_fence_after();
        return good;
    }
};

__device__ __forceinline__ void sync_for_mma() {
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
}

__device__ __forceinline__ auto k1s(uint64_t d0, int s) { return d0 + (uint64_t)(s * 2); }
__device__ __forceinline__ auto k2s(uint64_t d0, int s) {
    return d0 + (uint64_t)(((s >> 2) * TILE + (s & 3) * 32) >> 4);
}
__device__ __forceinline__ auto mns(uint64_t d0, int s) { return d0 + (uint64_t)(s * 128); }

// ---------------------------------------------------------------- chunk summaries
// Shared memory (offsets from the dynamic base, which is 1024-byte aligned):
constexpr uint32_t S1_U = 0;                // U: [128 j][128 i] K-major, two atoms
constexpr uint32_t S1_LK = S1_U + 2 * TILE; // Lam K  [tok][feat]   } equally spaced: the
constexpr uint32_t S1_LV = S1_LK + TILE;    // Lam V  [tok][feat]   } N = 192 MN-major operand
constexpr uint32_t S1_K = S1_LV + TILE;     // K      [tok][feat]   } [Lam K | Lam V | K]
constexpr uint32_t S1_Q = S1_K + TILE;      // Q, then Y = U^T Lam V
constexpr uint32_t S1_V = S1_Q + TILE;      // V
constexpr uint32_t S1_TAB = S1_V + TILE;    // lam[128]
constexpr uint32_t S1_BAR = S1_TAB + C * 4;
constexpr uint32_t S1_BYTES = S1_BAR + 64;  // no slack: checked at run time
// The summary is staged (fp32, rows swizzled by 16-byte chunk) over U, Lam K, Lam V.

// Threads: warp w reads TMEM lane quadrant (w & 3) and half (w >> 2) of the columns.
// Rounds: R1 A* = Q K^T                                -> E1: U to bf16; Lam K, Lam V
//         R2 Y = U^T Lam V; [K^T ; Q^T][Lam K | Lam V | K]  (S, -, Khat ; -, C, -)
//                                                      -> E2: Y to bf16; S, C, Khat staged
//         R3 [Y^T ; V^T] K   (lanes 0-63: G^T)          -> E3: G^T staged; summary stored
__global__ void __launch_bounds__(DNT, 2)
k_dec_summary(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, DParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    if (ptx::smem_u32(sm) & 1023) {            // the swizzled tiles need a 1024-byte base
        if (tid == 0) set_status(p.status, DEV_ALIGN);
        return;
    }
    float* lam = reinterpret_cast<float*>(sm + S1_TAB);
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + S1_BAR);
    MmaSync ms{bar_load + 1, 0};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_load + 2);
    const float g = p.gamma[bh % p.H];
    if (tid == 0) {
        ptx::mbar_init(bar_load, 1);
        ptx::mbar_init(ms.bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        const int t0 = chunk * C;
        ptx::mbar_arrive_expect_tx(bar_load, 3 * TILE);
        ptx::tma_load_3d(sm + S1_Q, &tq, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + S1_K, &tk, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + S1_V, &tv, bar_load, 0, t0, bh);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 256);
        ptx::tmem_relinquish();
    }
    if (tid < C) lam[tid] = gpow_n(g, C - 1 - tid);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sb = ptx::smem_u32(sm);
    bool ok = ptx::mbar_wait(bar_load, 0);     // every thread: the tiles are read below
    if (ok && tid == 0) {
        ptx::tc_fence_after();
        const uint64_t dQ = kdesc(sb + S1_Q, 0), dK = kdesc(sb + S1_K, 0);
        constexpr uint32_t I_QK = ptx::idesc_bf16(128, 128, false, false);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem, k1s(dQ, s), k1s(dK, s), I_QK, s > 0);
    }
    // Lam K and Lam V: scale each token row by lam; the swizzle moves 16-byte chunks within a
    // row, so a chunk keeps its place.
    if (ok) {
        const float l = lam[row];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t off = row * 128 + (half * 4 + c) * 16;
            const uint4 kx = *reinterpret_cast<const uint4*>(sm + S1_K + off);
            const uint4 vx = *reinterpret_cast<const uint4*>(sm + S1_V + off);
            auto scale = [&](uint32_t w) {
                __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w);
                const float2 f = __bfloat1622float2(h);
                return ptx::pack_bf16(f.x * l, f.y * l);
            };
            *reinterpret_cast<uint4*>(sm + S1_LK + off) = make_uint4(scale(kx.x), scale(kx.y), scale(kx.z), scale(kx.w));
            *reinterpret_cast<uint4*>(sm + S1_LV + off) = make_uint4(scale(vx.x), scale(vx.y), scale(vx.z), scale(vx.w));
        }
    }
    ok = __syncthreads_and(ok) != 0;
    if (ok) ok = ms.commit_wait(tid == 0);      // R1 done
    if (ok) {
        // E1: U = strict upper part of A*, row `row` (this thread: columns half*64 .. +63)
        float v[32];
#pragma unroll
        for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
            if (c0 + 31 < quad * 32) {                                 // wholly below the diagonal
                st_row32_zero(sm + S1_U, row, c0);
                continue;
            }
            ptx::tmem_ld32(tmem + lane_base + c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c0 + i <= row) v[i] = 0.f;
            st_row32(sm + S1_U, row, c0, v);
        }
        sync_for_mma();
        if (tid == 0) {
            constexpr uint32_t I_Y = ptx::idesc_bf16(128, 64, true, true);
            constexpr uint32_t I_ST = ptx::idesc_bf16(128, 192, true, true);
            const uint64_t dU = mdesc(sb + S1_U, TILE, 0), dLV = mdesc(sb + S1_LV, TILE, 0);
            const uint64_t dKQ = mdesc(sb + S1_K, S1_Q - S1_K, 0), dB3 = mdesc(sb + S1_LK, TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + 192, mns(dU, s), mns(dLV, s), I_Y, s > 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem, mns(dKQ, s), mns(dB3, s), I_ST, s > 0);
        }
        ok = ms.commit_wait(tid == 0);          // R2 done
    }
    float* stg = reinterpret_cast<float*>(sm + S1_U);   // [4][64][64] fp32, rows chunk-swizzled
    auto put_row = [&](int m, int r, int c0, const float (&x)[32]) {
        float4* dst = reinterpret_cast<float4*>(stg + m * D * D + r * D);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            dst[(c0 / 4 + j) ^ (r & 7)] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
    };
    if (ok) {
        // E2: Y -> bf16 over Q; S (lanes 0-63, cols 0-63), Khat (lanes 0-63, cols 128-191),
        // C (lanes 64-127, cols 64-127) staged
        float v[32];
        ptx::tmem_ld32(tmem + lane_base + 192 + half * 32, v);
        st_row32(sm + S1_Q, row, half * 32, v);
        if (quad < 2) {
            ptx::tmem_ld32(tmem + lane_base + half * 32, v);
            put_row(0, row, half * 32, v);
            ptx::tmem_ld32(tmem + lane_base + 128 + half * 32, v);
            put_row(2, row, half * 32, v);
        } else {
            ptx::tmem_ld32(tmem + lane_base + 64 + half * 32, v);
            put_row(1, row - 64, half * 32, v);
        }
        sync_for_mma();
        if (tid == 0) {
            constexpr uint32_t I_G = ptx::idesc_bf16(128, 64, true, true);
            const uint64_t dYV = mdesc(sb + S1_Q, S1_V - S1_Q, 0), dK = mdesc(sb + S1_K, TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem, mns(dYV, s), mns(dK, s), I_G, s > 0);
        }
        ok = ms.commit_wait(tid == 0);          // R3 done
    }
    if (ok) {
        if (quad < 2) {
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + half * 32, v);
            put_row(3, row, half * 32, v);
        }
        __syncthreads();
        const float4* st4 = reinterpret_cast<const float4*>(stg);
        for (int f = tid; f < DSUM / 4; f += DNT) {
            const int r = (f >> 4) & (D - 1);
            *reinterpret_cast<float4*>(dsum(p, bh, chunk, 4 * f)) = st4[(f & ~15) | ((f & 15) ^ (r & 7))];
        }
    } else if (tid == 0) {
        set_status(p.status, DEV_TIMEOUT);
        ptx::mbar_wait(bar_load, 0, 100000000ull);
        ptx::umma_commit(ms.bar);
        ptx::mbar_wait(ms.bar, ms.phase, 100000000ull);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- prefixes (CUDA cores)
constexpr int PNT = 256;

// Exclusive decayed prefix over chunks of S (slot matrix 0) and C (matrix 1), in place:
// X0(0) = 0, X0(l+1) = rho X0(l) + X_l.  One thread per matrix element.
__global__ void __launch_bounds__(PNT) k_dec_prefix_sc(DParams p) {
    const int e = blockIdx.x * PNT + threadIdx.x, bh = blockIdx.y;
    if (e >= 2 * D * D) return;
    const float rho = gpow_n(p.gamma[bh % p.H], C);
    float* x = dsum(p, bh, 0, e);             // chunk l at x + 32 l
    float run = 0.f;
    for (int l0 = 0; l0 < p.NC; l0 += 16) {
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (l0 + i < p.NC) y[i] = x[(l0 + i) * 32];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (l0 + i < p.NC) {
                x[(l0 + i) * 32] = run;
                run = fmaf(rho, run, y[i]);
            }
    }
}

// Per chunk: Y^T = G^T + rho C0^T Khat, in place of G^T (matrix 3).  (Y = G + rho Khat C0 and
// Khat is symmetric.)
__global__ void __launch_bounds__(PNT) k_dec_cross(DParams p) {
    __shared__ __align__(16) float Kh[D * D];
    __shared__ __align__(16) float C0[D * D];
    const int l = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const float rho = gpow_n(p.gamma[bh % p.H], C);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int f = tid + PNT * i;
        const float4 c = *reinterpret_cast<const float4*>(dsum(p, bh, l, D * D + 4 * f));
        const float4 k = *reinterpret_cast<const float4*>(dsum(p, bh, l, 2 * D * D + 4 * f));
        reinterpret_cast<float4*>(C0)[f] = c;
        reinterpret_cast<float4*>(Kh)[f] = make_float4(rho * k.x, rho * k.y, rho * k.z, rho * k.w);
    }
    __syncthreads();
    const int r = 4 * (tid >> 4), c = 4 * (tid & 15);   // rows r.. of Y^T (columns of C0), columns c..
    float y[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const float4 gx = *reinterpret_cast<const float4*>(dsum(p, bh, l, 3 * D * D + (r + a) * D + c));
        y[a][0] = gx.x; y[a][1] = gx.y; y[a][2] = gx.z; y[a][3] = gx.w;
    }
#pragma unroll 8
    for (int k = 0; k < D; ++k) {
        const float4 cv = *reinterpret_cast<const float4*>(C0 + k * D + r);
        const float4 kv = *reinterpret_cast<const float4*>(Kh + k * D + c);
        const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            y[a][0] = fmaf(cc[a], kv.x, y[a][0]); y[a][1] = fmaf(cc[a], kv.y, y[a][1]);
            y[a][2] = fmaf(cc[a], kv.z, y[a][2]); y[a][3] = fmaf(cc[a], kv.w, y[a][3]);
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4*>(dsum(p, bh, l, 3 * D * D + (r + a) * D + c)) =
            make_float4(y[a][0], y[a][1], y[a][2], y[a][3]);
}

// Exclusive decayed prefix of Y^T (matrix 3) into G0^T, in place.
__global__ void __launch_bounds__(PNT) k_dec_prefix_g(DParams p) {
    const int e = blockIdx.x * PNT + threadIdx.x, bh = blockIdx.y;
    if (e >= D * D) return;
    const float rho = gpow_n(p.gamma[bh % p.H], C);
    float* x = dsum(p, bh, 0, 3 * D * D + e);
    float run = 0.f;
    for (int l0 = 0; l0 < p.NC; l0 += 16) {
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (l0 + i < p.NC) y[i] = x[(l0 + i) * 32];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (l0 + i < p.NC) {
                x[(l0 + i) * 32] = run;
                run = fmaf(rho, run, y[i]);
            }
    }
}

// ---------------------------------------------------------------- output (persistent)
// One CTA per SM takes the (chunk, head) items w = blockIdx.x, blockIdx.x + gridDim.x, ...;
// items are independent.  Q, K, V and the carried-in state tiles are double buffered: the
// next item's TMA loads are issued as an item starts, and the epilogue warps turn the next
// item's fp32 state into bf16 tiles while the current item's second MMA round runs.  At, H,
// W and Gam Z are MMA A operands read from tensor memory.
//
// Shared memory: two stages of [Q | K | S0, G0^T | C0 | V] (72 KB each; K sits directly
// before S0, G0^T so that [K ; S0^T ; G0^T] is one B operand), then A, U (B operands), Gam P,
// the table of gamma powers and the barriers.
constexpr uint32_t SQ_ = 0, SK_ = TILE, SSG_ = 2 * TILE, SC0_ = 2 * TILE + 2 * QTILE;
constexpr uint32_t SV_ = 2 * TILE + 3 * QTILE;
constexpr uint32_t STAGE3 = 3 * TILE + 3 * QTILE;   // 72 KB
constexpr uint32_t S3_A = 2 * STAGE3;               // A, later the O staging boxes
constexpr uint32_t S3_U = S3_A + 2 * TILE;          // U
constexpr uint32_t S3_P = S3_U + 2 * TILE;          // Gam P
constexpr uint32_t S3_TAB = S3_P + TILE;            // g^n, n = 0..256
constexpr uint32_t S3_BAR = S3_TAB + 260 * 4;       // 2 load barriers, the MMA barrier, TMEM slot
constexpr uint32_t S3_BYTES = S3_BAR + 64 + 1024;   // + alignment slack

// TMEM columns
constexpr uint32_t T3_AS = 0;     // A*, then W (fp32)        (128)
constexpr uint32_t T3_P = 128;    // P                        (64)
constexpr uint32_t T3_QG = 192;   // Q G0                     (64)
constexpr uint32_t T3_HK = 256;   // H K                      (64)
constexpr uint32_t T3_O = 320;    // O                        (64)
constexpr uint32_t T3_AT = 384;   // At, then W (bf16 pairs)  (64)
constexpr uint32_t T3_H = 448;    // H, then Gam Z (bf16)     (64)

// Rounds per item: R1 [A* | P | Q G0] = Q [K ; S0^T ; G0^T]^T  -> E1: At, H to TMEM; A, U,
//                                                                  Gam P to shared memory
//                  R2 W = Gam P Q^T + At A^T + H U^T; H K      -> E2: W (masked, Dg) and
//                                                                  Gam Z = Gam (Gam P + H K) to TMEM
//                  R3 O = W V + (Gam Z) C0                     -> E3: O - Gam Q G0, TMA store
__global__ void __launch_bounds__(DNT, 1)
k_dec_output(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
             const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to, DParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int items = p.NC * p.BH;
    const int w0 = blockIdx.x;
    if (w0 >= items) return;
    float* gp = reinterpret_cast<float*>(sm + S3_TAB);
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + S3_BAR);   // [2]
    MmaSync ms{bar_load + 2, 0};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_load + 3);
    if (tid == 0) {
        ptx::mbar_init(&bar_load[0], 1);
        ptx::mbar_init(&bar_load[1], 1);
        ptx::mbar_init(ms.bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    int issued[2] = {0, 0}, waited[2] = {0, 0};       // thread 0's load bookkeeping
    auto issue_loads = [&](int w, int b) {
        uint8_t* st = sm + b * STAGE3;
        const int bh = w / p.NC, t0 = (w % p.NC) * C;
        ptx::mbar_arrive_expect_tx(&bar_load[b], 3 * TILE);
        ptx::tma_load_3d(st + SQ_, &tq, &bar_load[b], 0, t0, bh);
        ptx::tma_load_3d(st + SK_, &tk, &bar_load[b], 0, t0, bh);
        ptx::tma_load_3d(st + SV_, &tv, &bar_load[b], 0, t0, bh);
        ++issued[b];
    };
    // carried-in S0, C0 and G0^T of item w -> bf16 operand tiles of stage b, row for row (row r,
    // 16-byte chunk j at j ^ (r & 7)); S0 is symmetric, so its rows serve as the K-major S0^T
    auto convert_state = [&](int w, int b) {
        uint8_t* st = sm + b * STAGE3;
        const int bh = w / p.NC, l = w % p.NC;
        constexpr int NI = 3 * D * 8 / DNT;
        float4 x[NI][2];
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int f = tid + DNT * i, t = f >> 9, r = (f >> 3) & 63, j = f & 7;
            const float4* src = reinterpret_cast<const float4*>(dsum(p, bh, l, (t == 2 ? 3 : t) * D * D + r * D + 8 * j));
            x[i][0] = src[0];
            x[i][1] = src[1];
        }
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int f = tid + DNT * i, t = f >> 9, r = (f >> 3) & 63, j = f & 7;
            const uint32_t tile = t == 0 ? SSG_ : t == 1 ? SC0_ : SSG_ + QTILE;
            *reinterpret_cast<uint4*>(st + tile + r * 128 + ((j ^ (r & 7)) << 4)) =
                make_uint4(ptx::pack_bf16(x[i][0].x, x[i][0].y), ptx::pack_bf16(x[i][0].z, x[i][0].w),
                           ptx::pack_bf16(x[i][1].x, x[i][1].y), ptx::pack_bf16(x[i][1].z, x[i][1].w));
        }
    };
    if (tid == 0) issue_loads(w0, 0);
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    convert_state(w0, 0);
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sb = ptx::smem_u32(sm);
    constexpr uint32_t I_R1 = ptx::idesc_bf16(128, 256, false, false);
    constexpr uint32_t I_W = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t I_KM = ptx::idesc_bf16(128, 64, false, true);
    // packed bf16 pairs of 32 values (columns c0 .. c0+31) into 16 TMEM columns of this lane
    auto st_pairs = [&](uint32_t tcol, const float (&x)[32]) {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = ptx::pack_bf16(x[2 * i], x[2 * i + 1]);
        ptx::tmem_st16u(tmem + lane_base + tcol, r);
    };
    auto st_pairs_zero = [&](uint32_t tcol) {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = 0u;
        ptx::tmem_st16u(tmem + lane_base + tcol, r);
    };

    bool ok = true;
    int cur_bh = -1;
    int it = 0;
    for (int w = w0; w < items && ok; w += gridDim.x, ++it) {
        const int b = it & 1;
        const uint32_t st = b * STAGE3;
        const int bh = w / p.NC, chunk = w % p.NC;
        const int wn = w + gridDim.x;
        if (bh != cur_bh) {                  // gamma powers of this item's head (block-uniform)
            cur_bh = bh;
            const float g = p.gamma[bh % p.H];
            for (int n = tid; n <= 2 * C; n += DNT) gp[n] = gpow_n(g, n);
        }
        if (tid == 0) {
            if (wn < items) issue_loads(wn, b ^ 1);        // stage b^1 was freed by the last item
            ok = ptx::mbar_wait(&bar_load[b], (it >> 1) & 1);
            if (ok) {
                ++waited[b];
                ptx::tc_fence_after();
                const uint64_t dQ = kdesc(sb + st + SQ_, 0), dKSG = kdesc(sb + st + SK_, 0);
                for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T3_AS, k1s(dQ, s), k1s(dKSG, s), I_R1, s > 0);
            }
            ptx::bulk_wait_read();                          // the last item's O boxes (over A) are read
        }
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;
        if (!ms.commit_wait(tid == 0)) { ok = false; break; }   // R1 done
        {
            // E1: from A* row `row`, columns half*64 .. +63 in two blocks of 32: At, H (TMEM, bf16
            // pairs), A, U (shared memory); Gam P (columns half*32 .. +31).  Blocks wholly above
            // the diagonal are zero in At, H and A, blocks wholly below it zero in U.
            float v[32], w32[32];
#pragma unroll
            for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
                ptx::tmem_ld32(tmem + lane_base + T3_AS + c0, v);
                if (c0 > quad * 32 + 31) {
                    st_pairs_zero(T3_AT + c0 / 2);
                    st_pairs_zero(T3_H + c0 / 2);
                    st_row32_zero(sm + S3_A, row, c0);
                    st_row32(sm + S3_U, row, c0, v);
                    continue;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int d = row - (c0 + i);                      // tau - i
                    w32[i] = d >= 0 ? gp[d] * v[i] : 0.f;              // At
                }
                st_pairs(T3_AT + c0 / 2, w32);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int d = row - (c0 + i);
                    w32[i] = d > 0 ? (gp[d] - 1.f) * v[i] : 0.f;      // H
                }
                st_pairs(T3_H + c0 / 2, w32);
                if (c0 + 31 < quad * 32) {
                    st_row32(sm + S3_A, row, c0, v);
                    st_row32_zero(sm + S3_U, row, c0);
                    continue;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) w32[i] = (c0 + i <= row) ? v[i] : 0.f;   // A
                st_row32(sm + S3_A, row, c0, w32);
#pragma unroll
                for (int i = 0; i < 32; ++i) w32[i] = (c0 + i > row) ? v[i] : 0.f;    // U
                st_row32(sm + S3_U, row, c0, w32);
            }
            ptx::tmem_ld32(tmem + lane_base + T3_P + half * 32, v);
            const float gam = gp[row + 1];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= gam;
            st_row32(sm + S3_P, row, half * 32, v);
            ptx::tmem_st_wait();
        }
        sync_for_mma();
        if (tid == 0) {
            const uint64_t dP = kdesc(sb + S3_P, 0), dQ = kdesc(sb + st + SQ_, 0);
            const uint64_t dA = kdesc2(sb + S3_A, 0), dU = kdesc2(sb + S3_U, 0);
            const uint64_t dKm = mdesc(sb + st + SK_, TILE, 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T3_AS, k1s(dP, s), k1s(dQ, s), I_W, s > 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + T3_AS, tmem + T3_AT + 8 * s, k2s(dA, s), I_W, 1);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + T3_AS, tmem + T3_H + 8 * s, k2s(dU, s), I_W, 1);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + T3_HK, tmem + T3_H + 8 * s, mns(dKm, s), I_KM, s > 0);
        }
        if (wn < items) convert_state(wn, b ^ 1);                  // overlaps R2
        if (!ms.commit_wait(tid == 0)) { ok = false; break; }   // R2 done
        {
            // E2: W[tau][j] = g^(tau-j) x for j <= tau -> TMEM over At; Gam (Gam P + H K) -> over H
            float v[32], w32[32];
#pragma unroll
            for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
                if (c0 > quad * 32 + 31) {
                    st_pairs_zero(T3_AT + c0 / 2);
                    continue;
                }
                ptx::tmem_ld32(tmem + lane_base + T3_AS + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int d = row - (c0 + i);
                    v[i] = d >= 0 ? gp[d] * v[i] : 0.f;
                }
                st_pairs(T3_AT + c0 / 2, v);
            }
            ptx::tmem_ld32x2(tmem + lane_base + T3_P + half * 32, tmem + lane_base + T3_HK + half * 32, v, w32);
            const float gam = gp[row + 1];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = gam * fmaf(gam, v[i], w32[i]);
            st_pairs(T3_H + half * 16, v);
            ptx::tmem_st_wait();
        }
        sync_for_mma();
        if (tid == 0) {
            const uint64_t dVm = mdesc(sb + st + SV_, TILE, 0), dC = mdesc(sb + st + SC0_, TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + T3_O, tmem + T3_AT + 8 * s, mns(dVm, s), I_KM, s > 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16_ts(tmem + T3_O, tmem + T3_H + 8 * s, mns(dC, s), I_KM, 1);
        }
        if (!ms.commit_wait(tid == 0)) { ok = false; break; }   // R3 done
        {
            // E3: O - Gam (Q G0), staged as two [128][32] fp32 boxes over A, then TMA stores
            float o[32], m[32];
            ptx::tmem_ld32x2(tmem + lane_base + T3_O + half * 32, tmem + lane_base + T3_QG + half * 32, o, m);
            const float gam = gp[row + 1];
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = fmaf(-gam, m[i], o[i]);
            float4* box = reinterpret_cast<float4*>(sm + S3_A + half * (C * 128) + row * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j) box[j ^ (row & 7)] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
            ptx::fence_proxy_async();
        }
        __syncthreads();
        if (tid == 0) {
            ptx::tma_store_3d(&to, sm + S3_A, 0, chunk * C, bh);
            ptx::tma_store_3d(&to, sm + S3_A + C * 128, 32, chunk * C, bh);
            ptx::bulk_commit();
        }
    }
    if (tid == 0) {
        ptx::bulk_wait_all();
        if (!ok) {
            set_status(p.status, DEV_TIMEOUT);
            // let loads and MMAs already in flight land before TMEM and shared memory are released
            for (int b = 0; b < 2; ++b)
                if (issued[b] > waited[b]) ptx::mbar_wait(&bar_load[b], (issued[b] - 1) & 1, 100000000ull);
            ptx::umma_commit(ms.bar);
            ptx::mbar_wait(ms.bar, ms.phase, 100000000ull);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace

size_t decay_workspace_bytes(int BH, int T) {
    const size_t NC = (size_t)(T + C - 1) / C;
    return (size_t)BH * NC * DSUM * sizeof(float);
}

int decay_kernel_launches() { return 5; }

cudaError_t decay_forward(const void* q, const void* k, const void* v, const float* gamma, float* o, int BH,
                          int H, int T, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev) {
    if (!gamma || H < 1) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, T, BH) || !make_map(&mk, k, T, BH) || !make_map(&mv, v, T, BH) ||
        !make_map_out(&mo, o, T, BH))
        return cudaErrorInvalidValue;
    DParams prm;
    prm.T = T; prm.BH = BH; prm.H = H; prm.NC = (T + C - 1) / C;
    prm.gamma = gamma;
    prm.sums = static_cast<float*>(ws);
    prm.status = status;
    const int NC = prm.NC;
    cudaError_t e;
    if ((e = set_smem(k_dec_summary, S1_BYTES)) != cudaSuccess)
        return e;
    if ((e = set_smem(k_dec_output, S3_BYTES)) != cudaSuccess)
        return e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    k_dec_summary<<<dim3(NC, BH), DNT, S1_BYTES, st>>>(mq, mk, mv, prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    k_dec_prefix_sc<<<dim3((2 * D * D + PNT - 1) / PNT, BH), PNT, 0, st>>>(prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_dec_cross<<<dim3(NC, BH), PNT, 0, st>>>(prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_dec_prefix_g<<<dim3((D * D + PNT - 1) / PNT, BH), PNT, 0, st>>>(prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[2], st)) != cudaSuccess) return e;
    const int items = NC * BH;
    k_dec_output<<<items < kSMs ? items : kSMs, DNT, S3_BYTES, st>>>(mq, mk, mv, mo, prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[3], st)) != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace tc
}  // namespace hla
