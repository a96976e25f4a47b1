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
// i < tau (0 elsewhere).  With (S0, C0, G0) carried into a chunk (every earlier chunk full):
//     S0' = rho S0 + K^T Lam K,   C0' = rho C0 + Q^T Lam V,   G0' = rho G0 + K^T Y,
//     Y = U^T Lam V + rho K C0        (the chunk's G plus rho Khat C0, Khat = K^T K)
//     O = W V + Gam (Z C0 - Q G0),    Z = Gam P + H K,   P = Q S0,
//     W = Dg (.) L (.) (Gam P Q^T + At A^T + H U^T),   Dg[tau][j] = g^(tau-j).
// The cross terms are the carried-in S0 times the chunk's C (through P Q^T), the chunk's
// decayed-minus-undecayed key moment times C0 (through H K), and the carried-in
// Gam S0 C0 - G0 (through Gam P C0 and Q G0).
// Inside the chunk, the pair weight g^(tau-i) - [i > j] is split by i <= j (At A^T) and i > j
// (H U^T), so every weight is applied in fp32 before the one rounding of an operand to bf16:
// writing it as a difference of separately rounded products would lose the weight to bf16
// rounding at strong decay (H A*^T + A A^T) or at weak decay (At A*^T - A U^T).
//
// Kernels (a segment walk, as for the undecayed second order; only segment summaries reach HBM):
//   k_dsum  (tcgen05, one CTA per summary segment x head)  walks its chunks from the zero state
//                                                         and writes the segment summary
//   k_dwalk (tcgen05, one CTA per output segment x head)   folds the summaries before its
//                                                         segment, then walks its chunks with
//                                                         the state in TMEM, writing O by TMA
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
constexpr uint32_t QTILE = D * D * 2;     // one 64 x 64 bf16 tile = 8 KB

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

// ================================================================ segment walkers
// The decayed second order as a walk (the state carried chunk to chunk inside one CTA, only
// segment summaries in HBM).  Per chunk, with the carried-in (S0, C0, G0):
//     S0' = rho S0 + K^T Lam K,   C0' = rho C0 + Q^T Lam V,   G0' = rho G0 + K^T Y,
//     Y = U^T Lam V + rho K C0                       (G_l + rho Khat_l C0 of the chunk algebra)
//     O = W V + Gam (Z C0 - Q G0),   Z = Gam P + H K,   P = Q S0,
//     W = Dg (.) L (.) (Gam P Q^T + At A^T + H U^T).
// The fp32 state stays in TMEM as MMA accumulators.  The epilogue that turns it into the next
// chunk's bf16 operand tiles writes it back multiplied by rho; the chunk's products then
// accumulate onto it.  S and G occupy TMEM lanes 0-63, C lanes 64-127: their products are
// M = 128 with a stacked MN-major A operand whose other 64-row half is a 2 KB zero block
// ([K^T ; 0], [0 ; Q^T]), so they add nothing to the other half's lanes.  The zero block lies
// after every K tile and before every Q tile, so both stackings have a positive block offset.
//
// Summary slot of a segment of N chunks (fp32): S, C, G, Khat (row-major 64 x 64 each), then
// rho_seg = g^(cN).  Walked from the zero state; S and the G increments enter with the weight
// rho^(N-1-l) of chunk l (on Lam K and on Y), so only C is rescaled chunk by chunk (Y needs
// the running C0); Khat = sum K^T K is unweighted.  An output CTA of segment s folds the slots
// before it (exclusive prefix, m from the last slot back, w the product of the later rho):
//     S0 = sum w_m S_m,   C0 = sum w_m C_m,   G0 = sum w_m (G_m + Ksuf(m+1) C_m),
//     Ksuf(m+1) = sum_{m<l} Khat_l.
constexpr int WSLOT = 4 * D * D + 32;

struct WParams {
    int T, BH, H;
    int NCH, NS;        // output walk: chunks per segment, segments per head
    int NCHs, NSf;      // summary walk: chunks per segment, segments per head
    int ratio;          // summary segments per output segment
    const float* gamma;
    float* sums;        // [BH][NSf][WSLOT]
    int* status;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
// Stacked MN-major A operand of K-step s: the 64-row block at `top` (advancing with s) over
// the zero block `zero` (fixed), or the zero block over the block at `bottom`.
__device__ __forceinline__ uint64_t top_over_zero(uint32_t top, uint32_t zero, int s) {
    const uint32_t a = top + s * 2048;
    return ptx::desc_sw128(a, zero - a, 1024);
}
__device__ __forceinline__ uint64_t zero_over_bottom(uint32_t zero, uint32_t bottom, int s) {
    return ptx::desc_sw128(zero, bottom + s * 2048 - zero, 1024);
}
// Half the 16-byte chunks of row `row` of a [128][64] bf16 tile scaled by x into the same
// place of another tile (the swizzle moves chunks only within a row, so any chunk keeps its
// place).  Half h takes the physical chunks (4h + c) ^ (row mod 8): the lanes of a warp, on
// consecutive rows, then touch eight different chunk columns instead of one.
__device__ __forceinline__ void scale_row_half(const uint8_t* src, uint8_t* dst, int row, int half, float x) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t off = row * 128 + (((half * 4 + c) ^ (row & 7)) << 4);
        const uint4 u = *reinterpret_cast<const uint4*>(src + off);
        auto sc = [&](uint32_t w) {
            __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w);
            const float2 f = __bfloat1622float2(h);
            return ptx::pack_bf16(f.x * x, f.y * x);
        };
        *reinterpret_cast<uint4*>(dst + off) = make_uint4(sc(u.x), sc(u.y), sc(u.z), sc(u.w));
    }
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    float a[16], b[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        a[i] = v[i];
        b[i] = v[16 + i];
    }
    ptx::tmem_st16(taddr, a);
    ptx::tmem_st16(taddr + 16, b);
}

// ---------------------------------------------------------------- summary walk
// Two CTAs per SM (108 KB of shared memory, 256 TMEM columns, at most 128 registers a thread),
// so one CTA's epilogues overlap the other's MMAs.  Shared memory: the zero block Z1, the two
// K tiles, the Q tile, the V tile (V, then Lam V in place), the weighted Lam K tile, the Y tile,
// the rho C0 tile, the zero block Z2 (Z1 lies before every K and Q tile, Z2 after every K tile).
// TMEM columns: X 0-127 (A*^T = K Q^T; then U^T as bf16 pairs in 0-31 and 96-127 and Y in
// 32-95), S | Khat 128-191 (lanes 0-63 | 64-127), G | C 192-255 (lanes 0-63 | 64-127).
constexpr uint32_t W1_Z1 = 0, W1_K0 = 2048, W1_K1 = W1_K0 + TILE, W1_Q = W1_K1 + TILE;
constexpr uint32_t W1_V = W1_Q + TILE;      // V, then Lam V
constexpr uint32_t W1_WK = W1_V + TILE;     // rho^(N-1-l) Lam K
constexpr uint32_t W1_Y = W1_WK + TILE;     // rho^(N-1-l) Y, bf16 [tau][v]
constexpr uint32_t W1_C0 = W1_Y + TILE;     // rho C0, bf16 [f][v]
constexpr uint32_t W1_Z2 = W1_C0 + QTILE;
constexpr uint32_t W1_BAR = W1_Z2 + 2048;
constexpr uint32_t W1_BYTES = W1_BAR + 64;  // the dynamic base must be 1024-aligned (checked)
constexpr uint32_t T1_X = 0, T1_Y = 32, T1_SK = 128, T1_GC = 192;

// Rounds per chunk n: [G += [K^T;0] Y of chunk n-1; A*^T = K Q^T]       -> E1: U^T pairs, Lam V
//                     in place, weighted Lam K
//                     [C += [0;Q^T] Lam V; Y = K (rho C0) + U^T Lam V] (then S += [K^T;0] w Lam K,
//                     Khat += [0;K^T] K in the background)            -> E2: Y tile; rho C0' tile
//                                                                        and back to TMEM
__global__ void __launch_bounds__(DNT, 2)
k_dsum(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
       const __grid_constant__ CUtensorMap tv, WParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int seg = blockIdx.x, bh = blockIdx.y;
    // the output walk may be scheduled once every summary CTA has started
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (ptx::smem_u32(sm) & 1023) {            // the swizzled tiles need a 1024-byte base
        if (tid == 0) set_status(p.status, DEV_ALIGN);
        return;
    }
    const int N = p.NCHs;                     // summary segments are whole chunks
    const int chunk0 = seg * N;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + W1_BAR);
    uint64_t* bar_k = bar;                    // [2] K of a stage
    uint64_t* bar_qv = bar + 2;               // Q and V
    uint64_t* bar_m = bar + 3;                // MMA rounds
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 4);
    const float g = p.gamma[bh % p.H];
    const float rho = gpow_n(g, C);
    const float lam = gpow_n(g, C - 1 - row);
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) ptx::mbar_init(&bar[i], 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    int ik[2] = {0, 0}, wk[2] = {0, 0}, iqv = 0, wqv = 0;
    auto issue_k = [&](int n) {
        const int b = n & 1;
        ptx::mbar_arrive_expect_tx(&bar_k[b], TILE);
        ptx::tma_load_3d(sm + (b ? W1_K1 : W1_K0), &tk, &bar_k[b], 0, (chunk0 + n) * C, bh);
        ++ik[b];
    };
    auto issue_qv = [&](int n) {
        ptx::mbar_arrive_expect_tx(bar_qv, 2 * TILE);
        ptx::tma_load_3d(sm + W1_Q, &tq, bar_qv, 0, (chunk0 + n) * C, bh);
        ptx::tma_load_3d(sm + W1_V, &tv, bar_qv, 0, (chunk0 + n) * C, bh);
        ++iqv;
    };
    if (tid == 0) {
        issue_k(0);
        issue_qv(0);
        if (N > 1) issue_k(1);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 256);
        ptx::tmem_relinquish();
    }
    // the zero blocks and rho C0 = 0
    for (int i = tid; i < 2048 / 16; i += DNT) {
        reinterpret_cast<uint4*>(sm + W1_Z1)[i] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4*>(sm + W1_Z2)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = tid; i < QTILE / 16; i += DNT) reinterpret_cast<uint4*>(sm + W1_C0)[i] = make_uint4(0u, 0u, 0u, 0u);
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sb = ptx::smem_u32(sm);
    {
        // S | Khat and G | C start at zero.  Their products always accumulate: one that cleared
        // its accumulator would clear the lanes that the other half holds.
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
        tmem_st32(tmem + lane_base + T1_SK + half * 32, z);
        tmem_st32(tmem + lane_base + T1_GC + half * 32, z);
        ptx::tmem_st_wait();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    constexpr uint32_t I_QK = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t I_KM = ptx::idesc_bf16(128, 64, false, true);
    constexpr uint32_t I_MN = ptx::idesc_bf16(128, 64, true, true);
    uint32_t phase = 0;
    auto mma_wait = [&]() {                   // thread 0 has committed; the block agrees
        bool good = true;
        if (tid == 0) good = ptx::mbar_wait(bar_m, phase);
        phase ^= 1;
        good = __syncthreads_and(good) != 0;
        ptx::tc_fence_after();
        return good;
    };
    bool ok = true;
    for (int n = 0; n < N; ++n) {
        const int b = n & 1;
        const uint32_t Kb = b ? W1_K1 : W1_K0;
        // every thread: this chunk's K, Q, V (K and V are read below)
        ok = ptx::mbar_wait(&bar_k[b], (n >> 1) & 1) && ptx::mbar_wait(bar_qv, n & 1);
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;
        ++wk[b];
        ++wqv;
        if (tid == 0) {
            ptx::tc_fence_after();
            if (n > 0) {                                        // G of chunk n-1
                const uint32_t Kp = b ? W1_K0 : W1_K1;
                const uint64_t dY = mdesc(sb + W1_Y, TILE, 0);
                for (int s = 0; s < 8; ++s)
                    ptx::umma_bf16(tmem + T1_GC, top_over_zero(sb + Kp, sb + W1_Z2, s), mns(dY, s), I_MN, 1);
            }
            const uint64_t dK = kdesc(sb + Kb, 0), dQ = kdesc(sb + W1_Q, 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T1_X, k1s(dK, s), k1s(dQ, s), I_QK, s > 0);
            ptx::umma_commit(bar_m);
        }
        if (!mma_wait()) { ok = false; break; }
        if (tid == 0 && n + 1 < N && n >= 1) issue_k(n + 1);   // stage b^1: chunk n-1's G is done
        {
            // E1: row `row` = key token i of A*^T; U^T keeps the query columns tau < i.  Each half
            // packs its 64 columns into the 32 columns it read first (0-31, 96-127), leaving
            // 32-95 for Y.
            float v0[32], v1[32];
            ptx::tmem_ld32x2(tmem + lane_base + T1_X + half * 64, tmem + lane_base + T1_X + half * 64 + 32, v0, v1);
            uint32_t pr[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t0 = half * 64 + 2 * i;
                pr[i] = ptx::pack_bf16(t0 < row ? v0[2 * i] : 0.f, t0 + 1 < row ? v0[2 * i + 1] : 0.f);
            }
            const uint32_t pcol = T1_X + half * 96;
            ptx::tmem_st16u(tmem + lane_base + pcol, pr);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t0 = half * 64 + 32 + 2 * i;
                pr[i] = ptx::pack_bf16(t0 < row ? v1[2 * i] : 0.f, t0 + 1 < row ? v1[2 * i + 1] : 0.f);
            }
            ptx::tmem_st16u(tmem + lane_base + pcol + 16, pr);
            scale_row_half(sm + Kb, sm + W1_WK, row, half, lam * gpow_n(rho, N - 1 - n));
            scale_row_half(sm + W1_V, sm + W1_V, row, half, lam);
            ptx::tmem_st_wait();
        }
        sync_for_mma();
        if (tid == 0) {
            const uint64_t dLV = mdesc(sb + W1_V, TILE, 0), dC0 = mdesc(sb + W1_C0, TILE, 0);
            const uint64_t dK = kdesc(sb + Kb, 0);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + T1_GC, zero_over_bottom(sb + W1_Z1, sb + W1_Q, s), mns(dLV, s), I_MN, 1);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T1_Y, k1s(dK, s), mns(dC0, s), I_KM, s > 0);
            for (int s = 0; s < 8; ++s)         // U^T pairs: K-steps 0-3 in columns 0-31, 4-7 in 96-127
                ptx::umma_bf16_ts(tmem + T1_Y, tmem + T1_X + (s < 4 ? 8 * s : 96 + 8 * (s - 4)), mns(dLV, s), I_KM, 1);
            ptx::umma_commit(bar_m);
            const uint64_t dWK = mdesc(sb + W1_WK, TILE, 0), dKm = mdesc(sb + Kb, TILE, 0);
            for (int s = 0; s < 8; ++s)         // S (lanes 0-63) and Khat (lanes 64-127) in the background
                ptx::umma_bf16(tmem + T1_SK, top_over_zero(sb + Kb, sb + W1_Z2, s), mns(dWK, s), I_MN, 1);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + T1_SK, zero_over_bottom(sb + W1_Z1, sb + Kb, s), mns(dKm, s), I_MN, 1);
        }
        if (!mma_wait()) { ok = false; break; }
        if (tid == 0 && n + 1 < N) issue_qv(n + 1);             // Q and Lam V are read
        {
            // E2: the weighted Y to bf16; rho C0' (lanes 64-127) to its tile and back to TMEM
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + T1_Y + half * 32, v);
            const float wy = gpow_n(rho, N - 1 - n);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= wy;
            st_row32(sm + W1_Y, row, half * 32, v);
            if (quad >= 2 && n + 1 < N) {
                ptx::tmem_ld32(tmem + lane_base + T1_GC + half * 32, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= rho;
                st_row32(sm + W1_C0, row - 64, half * 32, v);
                tmem_st32(tmem + lane_base + T1_GC + half * 32, v);
                ptx::tmem_st_wait();
            }
        }
        sync_for_mma();
    }
    if (ok) {
        if (tid == 0) {
            const uint32_t Kp = ((N - 1) & 1) ? W1_K1 : W1_K0;
            const uint64_t dY = mdesc(sb + W1_Y, TILE, 0);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + T1_GC, top_over_zero(sb + Kp, sb + W1_Z2, s), mns(dY, s), I_MN, 1);
            ptx::umma_commit(bar_m);
        }
        ok = mma_wait();
    }
    if (ok) {
        // the slot: lanes 0-63 hold rows of S and G, lanes 64-127 rows of Khat and C
        float* slot = p.sums + ((size_t)bh * p.NSf + seg) * WSLOT;
        const int r = row & 63;
        float v[32];
        auto put = [&](int m) {
            float4* dst = reinterpret_cast<float4*>(slot + m * D * D + r * D + half * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        };
        ptx::tmem_ld32(tmem + lane_base + T1_SK + half * 32, v);
        put(quad < 2 ? 0 : 3);
        ptx::tmem_ld32(tmem + lane_base + T1_GC + half * 32, v);
        put(quad < 2 ? 2 : 1);
        if (tid == 0) slot[4 * D * D] = gpow_n(g, C * N);
    } else if (tid == 0) {
        set_status(p.status, DEV_TIMEOUT);
        for (int b = 0; b < 2; ++b)
            if (ik[b] > wk[b]) ptx::mbar_wait(&bar_k[b], (ik[b] - 1) & 1, 100000000ull);
        if (iqv > wqv) ptx::mbar_wait(bar_qv, (iqv - 1) & 1, 100000000ull);
        ptx::umma_commit(bar_m);
        ptx::mbar_wait(bar_m, phase, 100000000ull);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- output walk
// Shared memory: stage b holds K_b directly followed by S0_b (one K-major B operand [K ; S0]
// of N = 192) and Q_b.  The A tile's second atom begins with 64 rows that the causal mask
// keeps zero; its first 2 KB are the zero block of the stacked operands (after both K tiles,
// before both Q tiles).  V(n) sits in V slot n&1 and Lam V(n) in the other; V(n+1) is loaded
// over Lam V(n) once R2(n) has read it.
constexpr uint32_t W3_K0 = 0, W3_S00 = TILE, W3_K1 = TILE + QTILE, W3_S01 = 2 * TILE + QTILE;
constexpr uint32_t W3_A = 2 * TILE + 2 * QTILE;   // A [128 tau][128 j] K-major, two atoms
constexpr uint32_t W3_Z = W3_A + TILE;
constexpr uint32_t W3_Q0 = W3_A + 2 * TILE, W3_Q1 = W3_Q0 + TILE;
constexpr uint32_t W3_V0 = W3_Q1 + TILE, W3_V1 = W3_V0 + TILE;
constexpr uint32_t W3_LK = W3_V1 + TILE;          // Lam K
constexpr uint32_t W3_M1 = W3_LK + TILE;          // Gam P (E1 -> R2), then Y (E2 -> R3)
constexpr uint32_t W3_C0 = W3_M1 + TILE;          // C0, bf16 [f][v]
constexpr uint32_t W3_G0 = W3_C0 + QTILE;         // -G0, bf16 [f][v]
constexpr uint32_t W3_U = W3_G0 + QTILE;          // U [128][128] K-major, two atoms
constexpr uint32_t W3_TAB = W3_U + 2 * TILE;      // g^n, n = 0 .. 256
constexpr uint32_t W3_BAR = W3_TAB + 260 * 4;
constexpr uint32_t W3_BYTES = W3_BAR + 128 + 1024;
// TMEM columns
constexpr uint32_t T3W_X = 0;     // A*, then W; O2 = Z C0 - Q G0 (columns 0-63) in R3
constexpr uint32_t T3W_P = 128;   // P, Gam P, then Z; O1 = W V in R3
constexpr uint32_t T3W_Y = 192;   // K C0, rho K C0, then Y
constexpr uint32_t T3W_AT = 256;  // At, then W (bf16 pairs)
constexpr uint32_t T3W_H = 320;   // H (bf16 pairs), then Z (pairs, 320-351)
constexpr uint32_t T3W_S = 384;   // S (lanes 0-63)
constexpr uint32_t T3W_GC = 448;  // G (lanes 0-63) | C (lanes 64-127)

// Rounds per chunk: R1 [A* | P] = Q [K ; S0]^T (issued during the last chunk's E3), K C0;
//                     then S += [K^T;0] Lam K, C += [0;Q^T] Lam V
//                     -> E1: At, H pairs; A, U tiles; Gam P (tile and TMEM); rho K C0
//                   R2 W = Gam P Q^T + At A^T + H U^T; Z = Gam P + H K; Y = rho K C0 + U^T Lam V
//                     -> E2: W pairs (Dg, mask); Z pairs; Y tile; S0' tile, rho S0'
//                   R3 O1 = W V; O2 = Z C0 - Q G0; G += [K^T;0] Y
//                     -> E3: O = O1 + Gam O2 (TMA store from the chunk's Q, K tiles); C0', -G0'
//                        tiles, rho C0', rho G0';
//                        Lam K, Lam V of the next chunk
__global__ void __launch_bounds__(DNT, 1)
k_dwalk(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to, WParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int seg = blockIdx.x, bh = blockIdx.y;
    const int NC = (p.T + C - 1) / C;
    const int chunk0 = seg * p.NCH;
    const int nch = min(p.NCH, NC - chunk0);
    float* gp = reinterpret_cast<float*>(sm + W3_TAB);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + W3_BAR);
    uint64_t* bar_qk = bar;          // [2] Q, K of a stage
    uint64_t* bar_v = bar + 2;       // [2] V of a slot
    uint64_t* bar_m1 = bar + 4;      // MMA rounds (first commit)
    uint64_t* bar_m2 = bar + 5;      // MMA rounds (second commit: products an epilogue reads last)
    uint64_t* bar_f = bar + 6;       // [2] prologue fold, one per operand buffer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 8);
    const float g = p.gamma[bh % p.H];
    if (tid == 0) {
        for (int i = 0; i < 8; ++i) ptx::mbar_init(&bar[i], 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    int iq[2] = {0, 0}, wq[2] = {0, 0}, iv[2] = {0, 0}, wv[2] = {0, 0};   // loads issued / waited
    auto issue_qk = [&](int n) {
        const int b = n & 1, t0 = (chunk0 + n) * C;
        ptx::mbar_arrive_expect_tx(&bar_qk[b], 2 * TILE);
        ptx::tma_load_3d(sm + (b ? W3_Q1 : W3_Q0), &tq, &bar_qk[b], 0, t0, bh);
        ptx::tma_load_3d(sm + (b ? W3_K1 : W3_K0), &tk, &bar_qk[b], 0, t0, bh);
        ++iq[b];
    };
    auto issue_v = [&](int n) {
        const int b = n & 1, t0 = (chunk0 + n) * C;
        ptx::mbar_arrive_expect_tx(&bar_v[b], TILE);
        ptx::tma_load_3d(sm + (b ? W3_V1 : W3_V0), &tv, &bar_v[b], 0, t0, bh);
        ++iv[b];
    };
    if (tid == 0) {
        issue_qk(0);
        issue_v(0);
        if (nch > 1) issue_qk(1);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    for (int n = tid; n <= 2 * C; n += DNT) gp[n] = gpow_n(g, n);
    const float rho = gpow_n(g, C), lam = gpow_n(g, C - 1 - row), gam = gpow_n(g, row + 1);
    // A's blocks above the diagonal are zero in every chunk (the zero block among them)
#pragma unroll
    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32)
        if (c0 > quad * 32 + 31) st_row32_zero(sm + W3_A, row, c0);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sb = ptx::smem_u32(sm);
    constexpr uint32_t I_R1 = ptx::idesc_bf16(128, 192, false, false);
    constexpr uint32_t I_W = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t I_KM = ptx::idesc_bf16(128, 64, false, true);
    constexpr uint32_t I_MN = ptx::idesc_bf16(128, 64, true, true);
    uint32_t ph1 = 0, ph2 = 0, phf[2] = {0, 0};
    int fold_pending[2] = {0, 0};
    auto mwait = [&](uint64_t* b, uint32_t& ph) {   // thread 0 has committed to b; the block agrees
        bool good = true;
        if (tid == 0) good = ptx::mbar_wait(b, ph);
        ph ^= 1;
        good = __syncthreads_and(good) != 0;
        ptx::tc_fence_after();
        return good;
    };

    // ---- carried-in state: fold the slots m < ns of this head (the exclusive prefix of segment
    // seg), from the last slot back with w = the product of the later rho and Ksuf = the sum of
    // the later Khat: S0 = sum w S_m, C0 = sum w C_m, G0 = sum w G_m + X, X = sum Ksuf (w C_m).
    // Each thread keeps a 4 x 4 block of S0, C0, sum w G and Ksuf in fp32.  X runs on the tensor
    // core from two-term bf16 splits: A = [Ksuf_hi ; Ksuf_lo] (M = 128) times B = (w C_m)_hi and
    // (w C_m)_lo, so X = D(lanes 0-63) + D(lanes 64-127) carries about 16 bits of each factor
    // (TMEM columns T3W_Y; operand buffers over U and over Lam K + M1, alternately).
    float* FS = reinterpret_cast<float*>(sm + W3_LK);    // fp32 staging (rows swizzled by
    float* FC = reinterpret_cast<float*>(sm + W3_M1);    // 16-byte chunk), free until E0(0)
    float* FG = reinterpret_cast<float*>(sm + W3_V1);
    float* FX = reinterpret_cast<float*>(sm + W3_U);     // the lanes 64-127 half of X
    auto sw = [](int i, int j) { return i * D + ((((j >> 2) ^ (i & 7)) << 2) | (j & 3)); };
    const int ns = seg * p.ratio;
    bool ok = true;
    {
        const int r = 4 * (tid >> 4), c = 4 * (tid & 15);   // this thread's 4 x 4 block
        float aS[4][4], aC[4][4], aG[4][4], ks[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int e = 0; e < 4; ++e) aS[a][e] = aC[a][e] = aG[a][e] = ks[a][e] = 0.f;
        if (ns > 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");       // the summary walk's slots
            const float* s0 = p.sums + (size_t)bh * p.NSf * WSLOT;
            const uint32_t buf[2] = {W3_U, W3_LK};                    // A2 16 KB, B hi 8 KB, B lo 8 KB
            auto put4 = [&](uint32_t tile, int rr, int cc, float x0, float x1, float x2, float x3) {
                *reinterpret_cast<uint2*>(sm + tile + ptx::sw128_offset(rr, cc)) =
                    make_uint2(ptx::pack_bf16(x0, x1), ptx::pack_bf16(x2, x3));
            };
            auto lo_of = [](float x) { return x - __bfloat162float(__float2bfloat16_rn(x)); };
            float4 xs[4], xc[4], xg[4], xk[4];
            float rho_m = 1.f;
            auto load = [&](int m) {
                const float* sl = s0 + (size_t)m * WSLOT;
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    xs[a] = *reinterpret_cast<const float4*>(sl + (r + a) * D + c);
                    xc[a] = *reinterpret_cast<const float4*>(sl + D * D + (r + a) * D + c);
                    xg[a] = *reinterpret_cast<const float4*>(sl + 2 * D * D + (r + a) * D + c);
                    xk[a] = *reinterpret_cast<const float4*>(sl + 3 * D * D + (r + a) * D + c);
                }
                rho_m = sl[4 * D * D];
            };
            load(ns - 1);
            float w = 1.f;
            for (int m = ns - 1; m >= 0 && ok; --m) {
                float wc[4][4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    wc[a][0] = w * xc[a].x; wc[a][1] = w * xc[a].y; wc[a][2] = w * xc[a].z; wc[a][3] = w * xc[a].w;
                }
                if (m < ns - 1) {                                     // X += Ksuf (w C_m)
                    const int j = m & 1;
                    if (fold_pending[j]) {                            // the MMAs that read buffer j
                        bool good = true;
                        if (tid == 0) good = ptx::mbar_wait(&bar_f[j], phf[j]);
                        phf[j] ^= 1;
                        fold_pending[j] = 0;
                        if (!__syncthreads_and(good)) { ok = false; break; }
                    }
                    const uint32_t A2 = buf[j], Bh = buf[j] + TILE, Bl = Bh + QTILE;
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        put4(A2, r + a, c, ks[a][0], ks[a][1], ks[a][2], ks[a][3]);
                        put4(A2, 64 + r + a, c, lo_of(ks[a][0]), lo_of(ks[a][1]), lo_of(ks[a][2]), lo_of(ks[a][3]));
                        put4(Bh, r + a, c, wc[a][0], wc[a][1], wc[a][2], wc[a][3]);
                        put4(Bl, r + a, c, lo_of(wc[a][0]), lo_of(wc[a][1]), lo_of(wc[a][2]), lo_of(wc[a][3]));
                    }
                    ptx::fence_proxy_async();
                    __syncthreads();
                    if (tid == 0) {
                        ptx::tc_fence_after();
                        const uint64_t dA = kdesc(sb + A2, 0), dBh = mdesc(sb + Bh, TILE, 0), dBl = mdesc(sb + Bl, TILE, 0);
                        for (int s = 0; s < 4; ++s)
                            ptx::umma_bf16(tmem + T3W_Y, k1s(dA, s), mns(dBh, s), I_KM, m < ns - 2 || s > 0);
                        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T3W_Y, k1s(dA, s), mns(dBl, s), I_KM, 1);
                        ptx::umma_commit(&bar_f[j]);
                    }
                    fold_pending[j] = 1;
                }
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float sx[4] = {xs[a].x, xs[a].y, xs[a].z, xs[a].w};
                    const float gx[4] = {xg[a].x, xg[a].y, xg[a].z, xg[a].w};
                    const float kx[4] = {xk[a].x, xk[a].y, xk[a].z, xk[a].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        aS[a][e] = fmaf(w, sx[e], aS[a][e]);
                        aC[a][e] += wc[a][e];
                        aG[a][e] = fmaf(w, gx[e], aG[a][e]);
                        ks[a][e] += kx[e];
                    }
                }
                w *= rho_m;
                if (m > 0) load(m - 1);
            }
            for (int j = 0; j < 2; ++j)
                if (fold_pending[j]) {
                    bool good = true;
                    if (tid == 0) good = ptx::mbar_wait(&bar_f[j], phf[j], ok ? 1000000000ull : 100000000ull);
                    phf[j] ^= 1;
                    fold_pending[j] = 0;
                    if (!__syncthreads_and(good)) ok = false;
                }
            ptx::tc_fence_after();
        }
        if (ns > 1 && ok && quad >= 2) {                              // X, lanes 64-127 half
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + T3W_Y + half * 32, v);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(FX + sw(row - 64, half * 32 + 4 * j)) =
                    make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            *reinterpret_cast<float4*>(FS + sw(r + a, c)) = make_float4(aS[a][0], aS[a][1], aS[a][2], aS[a][3]);
            *reinterpret_cast<float4*>(FC + sw(r + a, c)) = make_float4(aC[a][0], aC[a][1], aC[a][2], aC[a][3]);
            *reinterpret_cast<float4*>(FG + sw(r + a, c)) = make_float4(aG[a][0], aG[a][1], aG[a][2], aG[a][3]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
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
    auto frow = [&](const float* F, int i, float (&v)[32]) {     // row i, columns half*32 .. +31
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 x = *reinterpret_cast<const float4*>(F + sw(i, half * 32 + 4 * j));
            v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
        }
    };
    if (ok) {
        // the state to its operand tiles (S0 by rows: S is symmetric) and, times rho, to TMEM;
        // the At / W and H pairs above the diagonal (those that nothing overwrites) to zero
        float v[32];
        if (quad < 2) {
            frow(FS, row, v);
            st_row32(sm + W3_S00, row, half * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= rho;
            tmem_st32(tmem + lane_base + T3W_S + half * 32, v);
            frow(FG, row, v);
            if (ns > 1) {
                float x[32], y[32];
                ptx::tmem_ld32(tmem + lane_base + T3W_Y + half * 32, x);
                frow(FX, row, y);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] += x[i] + y[i];
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = -v[i];
            st_row32(sm + W3_G0, row, half * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= -rho;
            tmem_st32(tmem + lane_base + T3W_GC + half * 32, v);
        } else {
            frow(FC, row - 64, v);
            st_row32(sm + W3_C0, row - 64, half * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= rho;
            tmem_st32(tmem + lane_base + T3W_GC + half * 32, v);
        }
#pragma unroll
        for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32)
            if (c0 > quad * 32 + 31) {
                st_pairs_zero(T3W_AT + c0 / 2);
                st_pairs_zero(T3W_H + c0 / 2);
            }
        ptx::tmem_st_wait();
    }
    __syncthreads();                                                  // FS, FC, FG, FX read
    if (ok) {
        ok = ptx::mbar_wait(&bar_qk[0], 0) && ptx::mbar_wait(&bar_v[0], 0);
        if (ok) {                                                     // E0 of chunk 0
            ++wq[0];
            ++wv[0];
            scale_row_half(sm + W3_K0, sm + W3_LK, row, half, lam);
            scale_row_half(sm + W3_V0, sm + W3_V1, row, half, lam);
        }
    }
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    ptx::tc_fence_after();
    // [A* | P] = Q [K ; S0]^T of a chunk is issued as soon as its tiles are in place: for chunk 0
    // here, for chunk n+1 while E3 of chunk n runs
    auto issue_qks = [&](int n) {
        const uint32_t Qb = (n & 1) ? W3_Q1 : W3_Q0, Kb = (n & 1) ? W3_K1 : W3_K0;
        const uint64_t dQ = kdesc(sb + Qb, 0), dKS = kdesc(sb + Kb, 0);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T3W_X, k1s(dQ, s), k1s(dKS, s), I_R1, s > 0);
    };
    if (ok && tid == 0) issue_qks(0);

    for (int n = 0; n < nch && ok; ++n) {
        const int b = n & 1;
        const bool more = n + 1 < nch;
        const uint32_t Qb = b ? W3_Q1 : W3_Q0, Kb = b ? W3_K1 : W3_K0;
        const uint32_t Vn = b ? W3_V1 : W3_V0, LVn = b ? W3_V0 : W3_V1;
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint64_t dKS = kdesc(sb + Kb, 0), dC = mdesc(sb + W3_C0, TILE, 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T3W_Y, k1s(dKS, s), mns(dC, s), I_KM, s > 0);
            ptx::umma_commit(bar_m1);
            // the state products run during E1
            const uint64_t dLK = mdesc(sb + W3_LK, TILE, 0), dLV = mdesc(sb + LVn, TILE, 0);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + T3W_S, top_over_zero(sb + Kb, sb + W3_Z, s), mns(dLK, s), I_MN, 1);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + T3W_GC, zero_over_bottom(sb + W3_Z, sb + Qb, s), mns(dLV, s), I_MN, 1);
        }
        if (!mwait(bar_m1, ph1)) { ok = false; break; }              // R1 done
        if (tid == 0 && n >= 1 && more) {
            // stage b^1: chunk n-1 is consumed and its O boxes (over its Q, K tiles) are read
            ptx::bulk_wait_read();
            issue_qk(n + 1);
        }
        {
            // E1: row `row` of A*, columns half*64 .. +63 in two blocks of 32.  With the weight
            // g^d, d = row - column: At = g^d x (d >= 0), H = At - x (d > 0), A = x (d >= 0),
            // U = x (d < 0).
            float vb[2][32], w32[32];
            ptx::tmem_ld32x2(tmem + lane_base + T3W_X + half * 64, tmem + lane_base + T3W_X + half * 64 + 32,
                             vb[0], vb[1]);
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                const int c0 = half * 64 + 32 * blk;
                float (&v)[32] = vb[blk];
                if (c0 > quad * 32 + 31) {                              // above the diagonal
                    st_row32(sm + W3_U, row, c0, v);
                    if (c0 < 64) st_pairs_zero(T3W_H + c0 / 2);        // Z pairs were here
                    continue;
                }
                if (c0 + 31 < quad * 32) {                              // below the diagonal
#pragma unroll
                    for (int i = 0; i < 32; ++i) w32[i] = gp[row - c0 - i] * v[i];
                    st_pairs(T3W_AT + c0 / 2, w32);
#pragma unroll
                    for (int i = 0; i < 32; ++i) w32[i] -= v[i];
                    st_pairs(T3W_H + c0 / 2, w32);
                    st_row32(sm + W3_A, row, c0, v);
                    st_row32_zero(sm + W3_U, row, c0);
                    continue;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int d = row - (c0 + i);
                    w32[i] = d >= 0 ? gp[d] * v[i] : 0.f;
                }
                st_pairs(T3W_AT + c0 / 2, w32);
#pragma unroll
                for (int i = 0; i < 32; ++i) w32[i] = (c0 + i < row) ? w32[i] - v[i] : 0.f;
                st_pairs(T3W_H + c0 / 2, w32);
#pragma unroll
                for (int i = 0; i < 32; ++i) w32[i] = (c0 + i <= row) ? v[i] : 0.f;
                st_row32(sm + W3_A, row, c0, w32);
#pragma unroll
                for (int i = 0; i < 32; ++i) w32[i] = (c0 + i > row) ? v[i] : 0.f;
                st_row32(sm + W3_U, row, c0, w32);
            }
            ptx::tmem_ld32x2(tmem + lane_base + T3W_P + half * 32, tmem + lane_base + T3W_Y + half * 32, vb[0], w32);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                vb[0][i] *= gam;
                w32[i] *= rho;
            }
            st_row32(sm + W3_M1, row, half * 32, vb[0]);
            tmem_st32(tmem + lane_base + T3W_P + half * 32, vb[0]);
            tmem_st32(tmem + lane_base + T3W_Y + half * 32, w32);
            ptx::tmem_st_wait();
        }
        sync_for_mma();
        if (tid == 0) {
            const uint64_t dGP = kdesc(sb + W3_M1, 0), dQ = kdesc(sb + Qb, 0);
            const uint64_t dA = kdesc2(sb + W3_A, 0), dU = kdesc2(sb + W3_U, 0);
            const uint64_t dKm = mdesc(sb + Kb, TILE, 0), dUm = mdesc(sb + W3_U, TILE, 0);
            const uint64_t dLV = mdesc(sb + LVn, TILE, 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T3W_X, k1s(dGP, s), k1s(dQ, s), I_W, s > 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + T3W_X, tmem + T3W_AT + 8 * s, k2s(dA, s), I_W, 1);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + T3W_X, tmem + T3W_H + 8 * s, k2s(dU, s), I_W, 1);
            ptx::umma_commit(bar_m1);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + T3W_P, tmem + T3W_H + 8 * s, mns(dKm, s), I_KM, 1);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + T3W_Y, mns(dUm, s), mns(dLV, s), I_MN, 1);
            ptx::umma_commit(bar_m2);
        }
        if (!mwait(bar_m1, ph1)) { ok = false; break; }              // W done
        {
            // E2a: W = Dg (.) L (.) x to pairs
            float v[32];
#pragma unroll
            for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
                if (c0 > quad * 32 + 31) continue;                      // zero since set-up
                ptx::tmem_ld32(tmem + lane_base + T3W_X + c0, v);
                if (c0 + 31 < quad * 32) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= gp[row - c0 - i];
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int d = row - (c0 + i);
                        v[i] = d >= 0 ? gp[d] * v[i] : 0.f;
                    }
                }
                st_pairs(T3W_AT + c0 / 2, v);
            }
        }
        if (!mwait(bar_m2, ph2)) { ok = false; break; }              // Z, Y and the state products done
        if (tid == 0 && more) issue_v(n + 1);                         // over Lam V(n)
        {
            // E2b: Z to pairs; Y to its tile; S0' to the next stage's tile, rho S0' back
            float v[32], y[32];
            ptx::tmem_ld32x2(tmem + lane_base + T3W_P + half * 32, tmem + lane_base + T3W_Y + half * 32, v, y);
            st_pairs(T3W_H + half * 16, v);
            st_row32(sm + W3_M1, row, half * 32, y);
            if (quad < 2 && more) {
                ptx::tmem_ld32(tmem + lane_base + T3W_S + half * 32, v);
                st_row32(sm + (b ? W3_S00 : W3_S01), row, half * 32, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= rho;
                tmem_st32(tmem + lane_base + T3W_S + half * 32, v);
            }
            ptx::tmem_st_wait();
        }
        sync_for_mma();
        if (tid == 0) {
            const uint64_t dV = mdesc(sb + Vn, TILE, 0), dC = mdesc(sb + W3_C0, TILE, 0);
            const uint64_t dG = mdesc(sb + W3_G0, TILE, 0), dQ = kdesc(sb + Qb, 0);
            const uint64_t dY = mdesc(sb + W3_M1, TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + T3W_P, tmem + T3W_AT + 8 * s, mns(dV, s), I_KM, s > 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16_ts(tmem + T3W_X, tmem + T3W_H + 8 * s, mns(dC, s), I_KM, s > 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + T3W_X, k1s(dQ, s), mns(dG, s), I_KM, 1);
            ptx::umma_commit(bar_m1);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + T3W_GC, top_over_zero(sb + Kb, sb + W3_Z, s), mns(dY, s), I_MN, 1);
            ptx::umma_commit(bar_m2);
        }
        if (!mwait(bar_m1, ph1)) { ok = false; break; }              // O1, O2 done
        // E3: O = O1 + Gam O2, staged as two [128][32] fp32 boxes over this chunk's Q and K
        // tiles: Q is read for the last time by R3's first products, K by the G product, so the
        // second box waits for it.  Then the next chunk's C0, -G0 tiles and rho C0, rho G0 back;
        // Lam K, Lam V of the next chunk.
        float o[32];
        {
            float m[32];
            ptx::tmem_ld32x2(tmem + lane_base + T3W_P + half * 32, tmem + lane_base + T3W_X + half * 32, o, m);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = fmaf(gam, m[i], o[i]);
        }
        auto put_box = [&]() {
            float4* box = reinterpret_cast<float4*>(sm + (half ? Kb : Qb) + row * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j) box[j ^ (row & 7)] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        };
        if (half == 0) put_box();
        ptx::tc_fence_before();
        if (!mwait(bar_m2, ph2)) { ok = false; break; }              // G done; O1, O2 read
        if (tid == 0 && more && ptx::mbar_wait(&bar_qk[b ^ 1], ((n + 1) >> 1) & 1))
            issue_qks(n + 1);                                         // over O2, O1: runs during E3b
        if (half == 1) put_box();
        bool good = true;
        if (more) {
            float m[32];
            ptx::tmem_ld32(tmem + lane_base + T3W_GC + half * 32, m);
            if (quad < 2) {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = -m[i];
                st_row32(sm + W3_G0, row, half * 32, o);
            } else {
                st_row32(sm + W3_C0, row - 64, half * 32, m);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) m[i] *= rho;
            tmem_st32(tmem + lane_base + T3W_GC + half * 32, m);
            ptx::tmem_st_wait();
            const int nb = b ^ 1, par = ((n + 1) >> 1) & 1;
            good = ptx::mbar_wait(&bar_qk[nb], par) && ptx::mbar_wait(&bar_v[nb], par);
            if (good) {
                ++wq[nb];
                ++wv[nb];
                scale_row_half(sm + (nb ? W3_K1 : W3_K0), sm + W3_LK, row, half, lam);
                scale_row_half(sm + LVn, sm + Vn, row, half, lam);   // V(n+1) -> Lam V(n+1)
            }
        }
        ptx::fence_proxy_async();
        ptx::tc_fence_before();
        ok = __syncthreads_and(good) != 0;
        ptx::tc_fence_after();
        if (tid == 0) {
            const int t0 = (chunk0 + n) * C;
            ptx::tma_store_3d(&to, sm + Qb, 0, t0, bh);
            ptx::tma_store_3d(&to, sm + Kb, 32, t0, bh);
            ptx::bulk_commit();
        }
    }
    if (tid == 0) {
        ptx::bulk_wait_all();
        if (!ok) {
            set_status(p.status, DEV_TIMEOUT);
            // let loads and MMAs already in flight land before TMEM and shared memory are released
            for (int b = 0; b < 2; ++b) {
                if (iq[b] > wq[b]) ptx::mbar_wait(&bar_qk[b], (iq[b] - 1) & 1, 100000000ull);
                if (iv[b] > wv[b]) ptx::mbar_wait(&bar_v[b], (iv[b] - 1) & 1, 100000000ull);
            }
            ptx::umma_commit(bar_m1);
            ptx::mbar_wait(bar_m1, ph1, 100000000ull);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace

namespace {
// Segment plan of the decayed walk, from a makespan model in microseconds per CTA wave:
// an output chunk ~7 (one CTA per SM), a summary chunk ~4 (two CTAs per SM), set-up ~3 per
// walk, ~0.6 per folded slot.
// Summaries cover the chunks before the last output segment.
struct DPlan {
    int NC, NCH, NS, NCHs, NSf, ratio;
};
DPlan dwalk_plan(int BH, int T, int seg_chunks) {
    DPlan pl;
    pl.NC = (T + C - 1) / C;
    auto waves = [](long long ctas) { return (double)((ctas + kSMs - 1) / kSMs); };
    auto waves2 = [](long long ctas) { return (double)((ctas + 2 * kSMs - 1) / (2 * kSMs)); };   // two per SM
    double best = -1.0;
    pl.NCH = 1;
    pl.NCHs = 1;
    for (int nch = 1; nch <= 128; nch *= 2) {
        if (seg_chunks > 0 && nch != seg_chunks) continue;
        const int NS = (pl.NC + nch - 1) / nch;
        const int ncsum = (NS - 1) * nch;
        for (int len = nch; len >= 1; len /= 2) {
            const double out = waves((long long)BH * NS) * (nch * 7.0 + 3.0 + 0.6 * (NS - 1) * (nch / len));
            const double sum = ncsum ? waves2((long long)BH * (ncsum / len)) * (len * 4.0 + 3.0) : 0.0;
            if (best < 0.0 || out + sum < best) {
                best = out + sum;
                pl.NCH = nch;
                pl.NCHs = len;
            }
            if (ncsum == 0) break;
        }
        if (seg_chunks <= 0 && nch >= pl.NC) break;
    }
    pl.NS = (pl.NC + pl.NCH - 1) / pl.NCH;
    pl.ratio = pl.NCH / pl.NCHs;
    pl.NSf = (pl.NS - 1) * pl.ratio;
    return pl;
}
}  // namespace

size_t decay_workspace_bytes(int BH, int T, int seg_chunks) {
    const DPlan pl = dwalk_plan(BH, T, seg_chunks);
    return (size_t)BH * (pl.NSf > 0 ? pl.NSf : 1) * WSLOT * sizeof(float);
}

int decay_kernel_launches(int BH, int T, int seg_chunks) {
    return dwalk_plan(BH, T, seg_chunks).NSf > 0 ? 2 : 1;
}

cudaError_t decay_forward(const void* q, const void* k, const void* v, const float* gamma, float* o, int BH,
                               int H, int T, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev,
                               int seg_chunks) {
    if (!gamma || H < 1) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, T, BH) || !make_map(&mk, k, T, BH) || !make_map(&mv, v, T, BH) ||
        !make_map_out(&mo, o, T, BH))
        return cudaErrorInvalidValue;
    const DPlan pl = dwalk_plan(BH, T, seg_chunks);
    WParams prm;
    prm.T = T; prm.BH = BH; prm.H = H;
    prm.NCH = pl.NCH; prm.NS = pl.NS; prm.NCHs = pl.NCHs; prm.NSf = pl.NSf; prm.ratio = pl.ratio;
    prm.gamma = gamma;
    prm.sums = static_cast<float*>(ws);
    prm.status = status;
    cudaError_t e;
    if ((e = set_smem(k_dsum, W1_BYTES)) != cudaSuccess) return e;
    if ((e = set_smem(k_dwalk, W3_BYTES)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    if (pl.NSf > 0) {
        k_dsum<<<dim3(pl.NSf, BH), DNT, W1_BYTES, st>>>(mq, mk, mv, prm);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[2], st)) != cudaSuccess) return e;
    // the output walk is a programmatic dependent of the summary walk: CTAs of segment 0 (and
    // every CTA's set-up and first loads) overlap the summary walk; the folding CTAs wait for it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.NS, BH);
    cfg.blockDim = dim3(DNT);
    cfg.dynamicSmemBytes = W3_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pl.NSf > 0 ? 1 : 0;
    if ((e = cudaLaunchKernelEx(&cfg, k_dwalk, mq, mk, mv, mo, prm)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[3], st)) != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace tc
}  // namespace hla
