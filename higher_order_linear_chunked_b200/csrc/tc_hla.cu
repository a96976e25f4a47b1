// tcgen05 tensor-core path for the second-order masked HLA forward (bf16 inputs, d = dv = 64).
//
// "Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 1 and 4.
// The sequence of each head is cut into output segments of NCH chunks of c = 128 tokens;
// the chunks before the last output segment are also cut into summary segments of NCHs
// chunks (see plan()).
//
//  1. k_walk<SUMMARY>: one CTA per (summary segment, head) walks its chunks from the zero
//     state and writes the segment summary (S, C, m, R = S C - G, r = S m - h) in fp32.
//  2. The exclusive prefix of the summaries under the semidirect-product combine, in its
//     factored form (see "segment prefixes"): folded by each output CTA in its prologue when
//     a head has few summary slots, else k_prefix_cross + k_prefix_sum.
//  3. k_walk<OUTPUT>: one CTA per (output segment, head) starts from its prefix and walks
//     its chunks again, emitting o for every token and carrying (S, R, r) to the next chunk.
//
// Per chunk (Q, K, V: 128 x 64 tiles; S0, R0, r0: state carried into the chunk):
//     A  = L (.) (Q K^T)                         (tcgen05, M=128 N=128 K=64)
//     P  = Q S0                                  (M=128 N=64  K=64)
//     W  = L (.) (P Q^T + A A^T)                 (M=128 N=128 K=64+128)
//     O  = Q [R0 | r0] + W [V | 1]               (M=128 N=80 K=64; N=80 K=128; column 64: den)
//     Z  = P + A K        (Z_j = S_j q_j, S_j the key moment up to token j)
//     S0 += K^T K;  [R0 | r0] += Z^T [V | 1]      (stacked M=128 MN-major operands)
// W_tj = q_t^T S_j q_j (j <= t) is the pair weight of the masked definition.  It equals
// q_t . Z_j too, but that dot product of the rounded Z can cancel far below its terms
// when q and k have mixed signs, while P Q^T + A A^T sums it key by key from the rounded
// scores, so its rounding error stays relative to the terms of the sum itself.
// The tensor-core state lives in TMEM (fp32) across the walk; its bf16 copies feed
// the next chunk's MMAs.  TMA stages Q, K, V (128B swizzle, no multicast), double
// buffered; one warp issues TMA and MMA; eight warps run the TMEM epilogues; O leaves
// through shared memory by TMA bulk tensor stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "common.cuh"
#include "ptx.cuh"
#include "simt.h"
#include "tc.h"
#include "tc_common.cuh"

namespace hla {
namespace tc {

constexpr int NT = 256;            // epilogue threads: 8 warps, two per TMEM lane quadrant
constexpr int NTH = NT + 32;       // + one warp that issues the TMA loads and the MMAs
constexpr int ISSUER = NT;         // the issuing thread (lane 0 of warp 8)

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t SM_Q0 = 0, SM_Q1 = SM_Q0 + TILE;
constexpr uint32_t SM_K0 = SM_Q1 + TILE, SM_V0 = SM_K0 + TILE;
constexpr uint32_t SM_K1 = SM_V0 + TILE, SM_V1 = SM_K1 + TILE;
constexpr uint32_t SM_Z = SM_V1 + TILE;          // Z  ([tok][feat])
constexpr uint32_t SM_ONES = SM_Z + TILE;        // MN-major [tok][64], column 0 = 1
constexpr uint32_t SM_A = SM_ONES + TILE;        // output: masked A [128][128] K-major (2 atoms);
                                                 // set-up: the carried-in state, fp32 S | R
constexpr uint32_t SM_S0 = SM_A + 2 * TILE;      // S0^T: [64 n][64 k] K-major
constexpr uint32_t SM_R0 = SM_S0 + 64 * 128;     // [R0 | r0]^T: [80 n][64 k] K-major
constexpr uint32_t SM_OST = SM_R0 + 80 * 128;    // O staging: two [128][32] fp32 TMA boxes
constexpr uint32_t SM_BAR = SM_OST + 2 * C * 128; // mbarriers
constexpr uint32_t SM_TOTAL = SM_BAR + 64;
constexpr uint32_t SMEM_BYTES = SM_TOTAL + 1024; // + alignment slack

// TMEM columns (fp32 accumulators, 128 lanes).
constexpr uint32_t TM_A = 0;      // A; output walk: then W (128 cols)
constexpr uint32_t TM_P = 128;    // P, then Z            (64)
constexpr uint32_t TM_O = 192;    // output: [O | den]    (80)
constexpr uint32_t TM_CR = 272;   // summary: lanes 0-63 [C|m], lanes 64-127 [R|r]  (80)
                                  // output: lanes 0-63 R^T, lane 64 r^T, rest 0   (64)
constexpr uint32_t TM_S = 352;    // lanes 0-63 S         (64)
constexpr uint32_t TM_W = 416;    // summary: masked A; output: masked W; as bf16 pairs, the A
                                  // operand of K-step s (16 tokens) at TM_W + 8 s  (64)
constexpr uint32_t TM_PP = 480;   // output: P as bf16 pairs  (32)
constexpr uint32_t TM_COLS = 512;

enum Mode { SUMMARY = 0, OUTPUT = 1 };

// ---------------------------------------------------------------- the walker
// Threads: 8 epilogue warps and one issuing warp.  Epilogue warp w reads TMEM lane
// quadrant (w & 3), i.e. tile rows 32 (w & 3) .. + 31 (the hardware ties a warp to the
// quadrant w mod 4, and so to one SM sub-partition), and handles half (w >> 2) of each
// tile's columns.  Lane 0 of warp 8 issues the TMA loads and the MMAs, so the epilogue
// warps never wait for an issue in progress.
//
// Summary walk, rounds of MMAs per chunk n, each followed by an epilogue:
//   R1(n): A = Q K^T, P = Q S0                      -> E1(n): A to a bf16 tile
//   R2(n): Z = P + A K, S += K^T K                  -> E2(n): Z, S0 to bf16 tiles
//   R3(n): [C|m ; R|r] += [Q^T;Z^T][V|1]
// R3(n) and R1(n+1) are issued together and their epilogues run together.
//
// Output walk, per chunk n (products marked * run while an epilogue converts something else):
//   R1(n): A = Q K^T, P = Q S0              -> E1: A (masked) to a bf16 tile, P to bf16 pairs
//                                                   in TMEM; [R0|r0]^T tile of chunk n
//          * S += K^T K
//   R2(n): W = P Q^T + A A^T, Z = P + A K   -> E2: W (masked) to bf16 pairs in TMEM; Z, S0 to
//          (P read from TMEM)                      bf16 tiles
//          * O = Q [R0|r0]^T
//   R3(n): [O|den] += W [V|1] (W read from TMEM), [R^T ; r^T] += [V^T ; 1^T] Z
// with R3(n) and R1(n+1) issued together.  Blocks above the diagonal of the masked A tile
// and of the masked pairs in TMEM are zeroed once.  The 32 x 32 blocks that the mask keeps
// and the other conversions are spread so that no warp does more than three 32-column
// pieces in one epilogue: a warp pair on one quadrant shares that sub-partition's issue
// slots, and quadrant 3 holds the longest rows.  O(n-1) leaves TMEM while R2(n) runs, and
// HBM by TMA stores.
template <int MODE>
__global__ void __launch_bounds__(NTH, 1)
k_walk(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + SM_BAR);       // [2]
    uint64_t* bar_mma = bar_load + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = (warp >> 2) & 1;
    const int row = quad * 32 + lane;                                     // TMEM lane = tile row
    const bool epi = warp < NT / 32;                                      // an epilogue warp
    const int seg = blockIdx.x, bh = blockIdx.y;
    using S = simt_layout;
    float* slot = MODE == OUTPUT ? p.pre + ((size_t)bh * p.NSp + seg * p.ratio) * S::size
                                 : p.sums + ((size_t)bh * p.NSp + seg) * S::size;
    // Programmatic dependent launch: the output walk may be scheduled once every summary CTA
    // has started; its CTAs that fold summaries wait for this grid's completion first.
    if (MODE == SUMMARY && tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (seg >= p.NS) {                       // padding slots: identity (zeros)
        if (MODE == SUMMARY) {
            float4* s4 = reinterpret_cast<float4*>(slot);
            for (int e = tid; e < S::size / 4; e += NTH) s4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        return;
    }
    const int chunk0 = seg * p.NCH;
    const int nchunks_total = (p.T + C - 1) / C;
    const int nch = min(p.NCH, nchunks_total - chunk0);

    // ---- set-up: barriers, first loads, TMEM, the ones tile
    if (tid == ISSUER) {
        ptx::mbar_init(&bar_load[0], 1);
        ptx::mbar_init(&bar_load[1], 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    auto issue_load = [&](int n) {
        const int b = n & 1;
        const int t0 = (chunk0 + n) * C;
        ptx::mbar_arrive_expect_tx(&bar_load[b], 3 * TILE);
        ptx::tma_load_3d(sm + (b ? SM_Q1 : SM_Q0), &tq, &bar_load[b], 0, t0, bh);
        ptx::tma_load_3d(sm + (b ? SM_K1 : SM_K0), &tk, &bar_load[b], 0, t0, bh);
        ptx::tma_load_3d(sm + (b ? SM_V1 : SM_V0), &tv, &bar_load[b], 0, t0, bh);
    };
    if (tid == ISSUER) {
        issue_load(0);
        if (nch > 1) issue_load(1);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, TM_COLS);
        ptx::tmem_relinquish();
    }
    if (tid < C) {
        // ones tile, [token][64]: column 0 = 1, the rest 0.  As the second N block of an
        // MN-major B operand it appends a ones column ([V | 1]); as the second M block of a
        // stacked MN-major A operand it appends a row of column sums ([V^T ; 1^T]).
        uint8_t* r = sm + SM_ONES + tid * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(r + (((j ^ tid) & 7) << 4)) = make_uint4(j == 0 ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    // Carried-in state (OUTPUT): the prefix (S, R, r) is staged in shared memory (rows swizzled
    // by 16-byte chunk: element (i, j) at i*64 + ((j/4 ^ (i & 7)) * 4) + j % 4), then every
    // thread takes its row.  With p.fold the CTA folds the summaries of slots 0 .. seg*ratio - 1
    // itself (R0 += R_l + S0 C_l, r0 += r_l + S0 m_l, then S0 += S_l), while its first loads
    // are in flight; otherwise it reads the prefix the prefix kernels wrote.
    float* stage = reinterpret_cast<float*>(sm + SM_A);                   // S [64][64] | R [64][64]
    float* stage_r = reinterpret_cast<float*>(sm + SM_Z);                 // r [64]
    auto sw = [](int i, int j) { return i * D + ((((j >> 2) ^ (i & 7)) << 2) | (j & 3)); };
    // The summaries are read below: wait for the summary walk (a no-op without a programmatic
    // dependency).  Segment 0 reads none and does not wait.
    if (MODE == OUTPUT && p.fold && seg > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (MODE == OUTPUT && epi && p.fold) {
        // n = seg * ratio slots: S0 = sum_l S_l, R0 = sum_l R_l + sum_{m < n-1} S_m Csuf(m+1),
        // r0 = sum_l r_l + sum_{m < n-1} S_m msuf(m+1), with Csuf(m) = sum_{m <= l < n} C_l (the
        // factored prefix, cross terms grouped by their S factor).  The plain sums are one batch
        // of loads; each cross term is one 64 x 64 x 64 product.
        const int n = seg * p.ratio;
        const float* sb = p.sums + (size_t)bh * p.NSp * S::size;
        float* Cs = reinterpret_cast<float*>(sm + SM_OST);                // Csuf [64][64]
        float* msuf = Cs + D * D;                                         // msuf [64]
        float* Sm = stage + D * D;                                        // S_m [64][64] (R part, for now)
        const int r = 4 * (tid >> 4), c = 4 * (tid & 15);                 // this thread's 4 x 4 of R0
        constexpr int NF = D * D / 4 / NT;                                // float4 per thread
        float racc[4][4];
        float4 sacc[NF];
        float r0 = 0.f;
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) racc[a][b] = 0.f;
#pragma unroll
        for (int i = 0; i < NF; ++i) sacc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int l = 0; l < n; ++l) {
            const float* sl = sb + (size_t)l * S::size;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float4 x = *reinterpret_cast<const float4*>(sl + S::mat(2) + (r + a) * D + c);
                racc[a][0] += x.x; racc[a][1] += x.y; racc[a][2] += x.z; racc[a][3] += x.w;
            }
#pragma unroll
            for (int i = 0; i < NF; ++i) {
                const float4 x = reinterpret_cast<const float4*>(sl + S::mat(0))[tid + NT * i];
                sacc[i] = make_float4(sacc[i].x + x.x, sacc[i].y + x.y, sacc[i].z + x.z, sacc[i].w + x.w);
            }
            if (tid < D) r0 += sl[S::vec(1) + tid];
        }
        for (int m = n - 2; m >= 0; --m) {
            const float* cl = sb + (size_t)(m + 1) * S::size;
            const float* smp = sb + (size_t)m * S::size;
            for (int f = tid; f < D * D / 4; f += NT) {
                const float4 x = reinterpret_cast<const float4*>(cl + S::mat(1))[f];
                const float4 o = m == n - 2 ? make_float4(0.f, 0.f, 0.f, 0.f) : reinterpret_cast<float4*>(Cs)[f];
                reinterpret_cast<float4*>(Cs)[f] = make_float4(o.x + x.x, o.y + x.y, o.z + x.z, o.w + x.w);
                reinterpret_cast<float4*>(Sm)[f] = reinterpret_cast<const float4*>(smp + S::mat(0))[f];
            }
            if (tid < D) msuf[tid] = (m == n - 2 ? 0.f : msuf[tid]) + cl[S::vec(0) + tid];
            ptx::named_sync(1, NT);          // the epilogue warps only
#pragma unroll 8
            for (int k = 0; k < D; ++k) {
                const float4 cv = *reinterpret_cast<const float4*>(Cs + k * D + c);
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float sv = Sm[(r + a) * D + k];
                    racc[a][0] = fmaf(sv, cv.x, racc[a][0]);
                    racc[a][1] = fmaf(sv, cv.y, racc[a][1]);
                    racc[a][2] = fmaf(sv, cv.z, racc[a][2]);
                    racc[a][3] = fmaf(sv, cv.w, racc[a][3]);
                }
            }
            if (tid < D) {                   // (S_m msuf)[tid] = sum_k S_m[k][tid] msuf[k] (S_m is symmetric)
                float y = 0.f;
                for (int k = 0; k < D; ++k) y = fmaf(Sm[k * D + tid], msuf[k], y);
                r0 += y;
            }
            ptx::named_sync(1, NT);
        }
#pragma unroll
        for (int i = 0; i < NF; ++i) {
            const int f = tid + NT * i, rr = f >> 4, ch = (f & 15) ^ (rr & 7);
            reinterpret_cast<float4*>(stage)[rr * 16 + ch] = sacc[i];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) stage[D * D + sw(r + a, c + b)] = racc[a][b];
        if (tid < D) stage_r[tid] = r0;
    } else if (MODE == OUTPUT && epi) {
        const float4* s4 = reinterpret_cast<const float4*>(slot + S::mat(0));
        const float4* r4 = reinterpret_cast<const float4*>(slot + S::mat(2));
        float4 xs[4], xr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            xs[i] = s4[tid + NT * i];
            xr[i] = r4[tid + NT * i];
        }
        const float rv = tid < D ? slot[S::vec(1) + tid] : 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int f = tid + NT * i, rr = f >> 4, ch = (f & 15) ^ (rr & 7);
            reinterpret_cast<float4*>(stage)[rr * 16 + ch] = xs[i];
            reinterpret_cast<float4*>(stage + D * D)[rr * 16 + ch] = xr[i];
        }
        if (tid < D) stage_r[tid] = rv;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    if (epi) {
        // state -> TMEM (fp32) and bf16 copies (S0 rows: S is symmetric; [R0|r0]^T); zeros
        // for the summary walk
        float v[16];
        if (quad < 2) {                      // S row `row`, columns half*32 .. +31
            for (int c0 = half * 32; c0 < half * 32 + 32; c0 += 16) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int ch = (c0 / 4 + j) ^ (row & 7);
                    const float4 x = MODE == OUTPUT ? reinterpret_cast<const float4*>(stage)[row * 16 + ch]
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                if (MODE == OUTPUT) ptx::tmem_st16(tmem + lane_base + TM_S + c0, v);
                st_row16(sm + SM_S0, TILE, row, c0, v);
            }
        } else if (MODE == SUMMARY) {        // [R0|r0]^T starts at zero: rows n = row - 64 < 80
            const int n = row - 64;
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = 0.f;
            for (int c0 = half * 32; c0 < half * 32 + 32; c0 += 16) {
                st_row16(sm + SM_R0, TILE, n, c0, v);
                if (n < 16) st_row16(sm + SM_R0, TILE, 64 + n, c0, v);
            }
        }
        if (MODE == OUTPUT && quad < 3) {
            // [R^T ; r^T] rows: row n < 64 is column n of R; row 64 is r; rows 65.. are 0.
            // TMEM lanes 0..95 of TM_CR and tile rows 0..79 (rows n < 64 by quads 0-1,
            // rows 64..79 by lanes 0..15 of quad 2).
            for (int c0 = half * 32; c0 < half * 32 + 32; c0 += 16) {
                if (quad < 2) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int k = c0 + i;                                 // R[k][row]
                        v[i] = stage[D * D + k * D + ((((row >> 2) ^ (k & 7)) << 2) | (row & 3))];
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = (lane == 0) ? stage_r[c0 + i] : 0.f;
                }
                ptx::tmem_st16(tmem + lane_base + TM_CR + c0, v);
                if (quad < 2 || lane < 16) st_row16(sm + SM_R0, TILE, quad < 2 ? row : 64 + lane, c0, v);
            }
        }
        {
            // The 32 x 32 blocks of the masked A (and W) above the diagonal (token block b of a
            // row in quadrant q < b) are zero in every chunk: written once, here.
            uint32_t z[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
            for (int j = 0; j < 2; ++j)
                if (2 * half + j > quad) ptx::tmem_st16u(tmem + lane_base + TM_W + 16 * (2 * half + j), z);
            ptx::tmem_st_wait();
        }
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
    constexpr uint32_t I_N80_KM = ptx::idesc_bf16(128, 80, false, true);
    constexpr uint32_t I_N80_MM = ptx::idesc_bf16(128, 80, true, true);
    // Descriptor of K-step s from the step-0 descriptor: only the 14-bit start address moves.
    auto k1 = [](uint64_t d0, int s) { return d0 + (uint64_t)(s * 2); };                         // +32 B
    auto k2 = [](uint64_t d0, int s) { return d0 + (uint64_t)(((s >> 2) * TILE + (s & 3) * 32) >> 4); };
    auto mn = [](uint64_t d0, int s) { return d0 + (uint64_t)(s * 128); };                       // +2048 B
    auto bufQ = [&](int n) { return sbase + ((n & 1) ? SM_Q1 : SM_Q0); };
    auto bufK = [&](int n) { return sbase + ((n & 1) ? SM_K1 : SM_K0); };
    auto bufV = [&](int n) { return sbase + ((n & 1) ? SM_V1 : SM_V0); };
    const uint64_t dS0 = kdesc(sbase + SM_S0, 0), dR0 = kdesc(sbase + SM_R0, 0);
    const uint64_t dA2 = kdesc2(sbase + SM_A, 0);
    const uint64_t dZm = mdesc(sbase + SM_Z, TILE, 0);

    auto issue_r1 = [&](int n) {             // A = Q K^T, P = Q S0
        const uint64_t dQ = kdesc(bufQ(n), 0), dK = kdesc(bufK(n), 0);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TM_A, k1(dQ, s), k1(dK, s), I_QK, s > 0);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TM_P, k1(dQ, s), k1(dS0, s), I_N64_KK, s > 0);
    };
    auto issue_s = [&](int n) {              // S += K^T K (rows 0-63 of [K^T ; V^T] K)
        const uint32_t sK = bufK(n), sV = bufV(n);
        const uint64_t dKm = mdesc(sK, TILE, 0), dKV = mdesc(sK, sV - sK, 0);
        for (int s = 0; s < 8; ++s)
            ptx::umma_bf16(tmem + TM_S, mn(dKV, s), mn(dKm, s), I_N64_MM, (MODE == OUTPUT || n > 0 || s > 0) ? 1u : 0u);
    };
    auto issue_z = [&](int n) {              // summary: Z = P + A K, masked A read from TMEM as bf16 pairs
        const uint64_t dKm = mdesc(bufK(n), TILE, 0);
        for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TM_P, tmem + TM_W + 8 * s, mn(dKm, s), I_N64_KM, 1);
    };
    auto issue_wz = [&](int n) {             // output: W = P Q^T + A A^T, Z = P + A K (A from the bf16 tile)
        const uint64_t dQ = kdesc(bufQ(n), 0), dKm = mdesc(bufK(n), TILE, 0);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16_ts(tmem + TM_A, tmem + TM_PP + 8 * s, k1(dQ, s), I_QK, s > 0);
        for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + TM_A, k2(dA2, s), k2(dA2, s), I_QK, 1);
        for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + TM_P, k2(dA2, s), mn(dKm, s), I_N64_KM, 1);
    };
    auto issue_qr0 = [&](int n) {            // [O | q.r0] = Q [R0|r0]^T
        const uint64_t dQ = kdesc(bufQ(n), 0);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TM_O, k1(dQ, s), k1(dR0, s), I_N80_KK, s > 0);
    };
    auto issue_r3 = [&](int n) {             // [O | den] += W [V | 1] ; [C|m ; R|r] += [Q^T ; Z^T] [V | 1]
        const uint32_t sQ = bufQ(n), sV = bufV(n);
        const uint64_t dQZ = mdesc(sQ, sbase + SM_Z - sQ, 0);
        const uint64_t dV1 = mdesc(sV, sbase + SM_ONES - sV, 0);
        if (MODE == OUTPUT) {
            const uint64_t dV1t = mdesc(sV, sbase + SM_ONES - sV, 0);     // stacked [V^T ; 1^T]
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TM_O, tmem + TM_W + 8 * s, mn(dV1, s), I_N80_KM, 1);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + TM_CR, mn(dV1t, s), mn(dZm, s), I_N64_MM, 1);
        } else {
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + TM_CR, mn(dQZ, s), mn(dV1, s), I_N80_MM, (n > 0 || s > 0) ? 1u : 0u);
        }
    };

    uint32_t mma_phase = 0;
    bool ok = true;
    // Thread 0 commits the MMAs issued so far and waits for them (bounded); the block agrees.
    auto commit_wait = [&]() -> bool {
        bool good = true;
        ptx::tc_fence_before();              // this thread's TMEM reads before MMAs issued after
        if (tid == ISSUER) {
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

    // 32 fp32 columns of this lane -> 16 bf16 pairs in TMEM (column 2i in the low half).  On
    // the diagonal block (diag), the columns past this lane's token are cleared first.
    auto st_pairs = [&](uint32_t tcol, const float (&x)[32], bool diag) {
        uint32_t r[16];
        if (diag) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                r[i] = ptx::pack_bf16(2 * i > lane ? 0.f : x[2 * i], 2 * i + 1 > lane ? 0.f : x[2 * i + 1]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = ptx::pack_bf16(x[2 * i], x[2 * i + 1]);
        }
        ptx::tmem_st16u(tmem + lane_base + tcol, r);
    };
    // Masked A (summary E1) or masked W (output E2): TM_A (fp32) -> bf16 pairs at TM_W.  Warp
    // (quad, half) converts its rows' token blocks 2 half and 2 half + 1 where the mask keeps
    // them (block b <= quad); the blocks above stay the zeros written at set-up.
    auto epi_mask = [&]() {
        const int b0 = 2 * half;
        if (b0 > quad) return;
        float v0[32], v1[32];
        if (b0 + 1 <= quad) {
            ptx::tmem_ld32x2(tmem + lane_base + TM_A + 32 * b0, tmem + lane_base + TM_A + 32 * (b0 + 1), v0, v1);
            st_pairs(TM_W + 16 * b0, v0, false);
            st_pairs(TM_W + 16 * (b0 + 1), v1, b0 + 1 == quad);
        } else {                             // b0 == quad
            ptx::tmem_ld32(tmem + lane_base + TM_A + 32 * b0, v0);
            st_pairs(TM_W + 16 * b0, v0, true);
        }
    };
    // Output E1: masked A -> SM_A (the K-major tile that is both operands of
    // A A^T); blocks above the diagonal stay the zeros of set-up
    auto epi_a_tile = [&]() {
        const int b0 = 2 * half;
        if (b0 > quad) return;
        float v0[32], v1[32];
        if (b0 + 1 <= quad) {
            ptx::tmem_ld32x2(tmem + lane_base + TM_A + 32 * b0, tmem + lane_base + TM_A + 32 * (b0 + 1), v0, v1);
            if (b0 + 1 == quad) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i > lane) v1[i] = 0.f;
            }
            st_row32(sm + SM_A, row, 32 * b0, v0);
            st_row32(sm + SM_A, row, 32 * (b0 + 1), v1);
        } else {
            ptx::tmem_ld32(tmem + lane_base + TM_A + 32 * b0, v0);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (i > lane) v0[i] = 0.f;
            st_row32(sm + SM_A, row, 32 * b0, v0);
        }
    };
    // Output E1: P -> bf16 pairs at TM_PP (this warp: columns half*32 .. +31)
    auto epi_p_pairs = [&]() {
        float v[32];
        ptx::tmem_ld32(tmem + lane_base + TM_P + half * 32, v);
        st_pairs(TM_PP + 16 * half, v, false);
    };
    // Summary E2: Z -> SM_Z; S -> SM_S0 (by rows: S is symmetric)
    auto epi2_sum = [&]() {
        float v0[32], v1[32];
        if (quad < 2) {
            ptx::tmem_ld32x2(tmem + lane_base + TM_P + half * 32, tmem + lane_base + TM_S + half * 32, v0, v1);
            st_row32(sm + SM_Z, row, half * 32, v0);
            st_row32(sm + SM_S0, row, half * 32, v1);
        } else {
            ptx::tmem_ld32(tmem + lane_base + TM_P + half * 32, v0);
            st_row32(sm + SM_Z, row, half * 32, v0);
        }
    };
    // Output E2, beside epi_mask: Z -> SM_Z
    auto epi2_out = [&]() {
        float v[32];
        ptx::tmem_ld32(tmem + lane_base + TM_P + half * 32, v);
        st_row32(sm + SM_Z, row, half * 32, v);
    };
    // Output E2, beside epi_mask: S -> SM_S0 rows, by the two warps that convert no mask block
    auto epi_s0 = [&]() {
        if (half != 1 || quad >= 2) return;
        float v0[32], v1[32];
        ptx::tmem_ld32x2(tmem + lane_base + TM_S, tmem + lane_base + TM_S + 32, v0, v1);
        st_row32(sm + SM_S0, row, 0, v0);
        st_row32(sm + SM_S0, row, 32, v1);
    };
    // Output E1, beside epi_mask: [R^T ; r^T] rows 0..64 of TM_CR -> [R0|r0]^T tile rows
    // (rows 65..79 stay the zeros of set-up), by the half-1 warps of quadrants 0-2, which
    // convert at most one mask block.
    auto epi3_state = [&]() {
        if (half != 1 || quad == 3) return;
        float v0[32], v1[32];
        ptx::tmem_ld32x2(tmem + lane_base + TM_CR, tmem + lane_base + TM_CR + 32, v0, v1);   // warp-collective
        if (quad < 2 || lane == 0) {
            const int r = quad < 2 ? row : 64;
            st_row32(sm + SM_R0, r, 0, v0);
            st_row32(sm + SM_R0, r, 32, v1);
        }
    };
    // Output: O rows of the last finished chunk (normalised by column 64, q.r0 + rowsum W)
    // staged as two [128 rows][32 cols] fp32 boxes in the 128B-swizzled TMA layout
    auto epi3_out = [&]() {
        float v[32];
        float d[16];
        const uint32_t tmo = tmem + TM_O + lane_base;
        ptx::tmem_ld16(tmo + 64, d);
        const float scale = p.norm ? 1.f / (d[0] + p.eps) : 1.f;
        ptx::tmem_ld32(tmo + half * 32, v);
        float4* box = reinterpret_cast<float4*>(sm + SM_OST + half * (C * 128) + row * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            box[j ^ (row & 7)] = make_float4(v[4 * j] * scale, v[4 * j + 1] * scale, v[4 * j + 2] * scale,
                                             v[4 * j + 3] * scale);
        ptx::fence_proxy_async();
    };
    // Issuing thread: store the staged O of chunk n (rows past T are clipped by the map).
    auto store_o = [&](int n) {
        const int t0 = (chunk0 + n) * C;
        ptx::tma_store_3d(&to, sm + SM_OST, 0, t0, bh);
        ptx::tma_store_3d(&to, sm + SM_OST + C * 128, 32, t0, bh);
        ptx::bulk_commit();
    };
    // Issuing thread: wait for the loads of chunk n + 1, then issue R3(n) and R1(n + 1).
    auto issue_r3_r1 = [&](int n) -> bool {
        issue_r3(n);
        if (n + 1 < nch) {
            if (!ptx::mbar_wait(&bar_load[(n + 1) & 1], ((n + 1) >> 1) & 1)) return false;
            ptx::tc_fence_after();
            issue_r1(n + 1);
        }
        return true;
    };

    // ---- the walk
    if (MODE == OUTPUT && epi) {
        // masked-A tile blocks above the diagonal: zero in every chunk (the set-up staging that
        // shared this space has been read); the first E1's proxy fence publishes them
#pragma unroll
        for (int j = 0; j < 2; ++j)
            if (2 * half + j > quad) st_row32_zero(sm + SM_A, row, 32 * (2 * half + j));
    }
    if (tid == ISSUER) {
        ok = ptx::mbar_wait(&bar_load[0], 0);
        if (ok) {
            ptx::tc_fence_after();
            issue_r1(0);
        }
    }
    ok = __syncthreads_and(ok) != 0;
    for (int n = 0; n < nch && ok; ++n) {
        if (!commit_wait()) { ok = false; break; }          // R1(n) [+ R3(n-1)] done
        if (tid == ISSUER) {
            issue_s(n);                                     // runs during E1
            if (n >= 1 && n + 1 < nch) issue_load(n + 1);   // buffer freed by R3(n-1)
            if (MODE == OUTPUT) ptx::bulk_wait_read();     // the O staging is free again
        }
        if (epi) {
            if (MODE == OUTPUT) {
                epi_a_tile();
                epi_p_pairs();
                if (n > 0) epi3_state();
            } else {
                epi_mask();
            }
            ptx::tmem_st_wait();
        }
        sync_for_mma();
        if (tid == ISSUER) {
            if (MODE == OUTPUT) issue_wz(n);
            else issue_z(n);
        }
        if (MODE == OUTPUT) {
            if (n > 0 && epi) epi3_out();                   // O(n-1), while W(n), Z(n) run
            if (!commit_wait()) { ok = false; break; }      // W(n), Z(n) and S done
            if (tid == ISSUER) {
                if (n > 0) store_o(n - 1);
                issue_qr0(n);                               // runs during E2
            }
            if (epi) {
                epi_mask();
                epi2_out();
                epi_s0();
                ptx::tmem_st_wait();
            }
        } else {
            if (!commit_wait()) { ok = false; break; }      // Z(n) and S done
            if (epi) epi2_sum();
        }
        sync_for_mma();
        if (tid == ISSUER) ok = issue_r3_r1(n);
        ok = __syncthreads_and(ok) != 0;
    }
    if (ok) {
        if (MODE == OUTPUT && tid == ISSUER) ptx::bulk_wait_read();
        ok = commit_wait();                                  // R3(last) done
        if (ok && MODE == OUTPUT) {
            if (epi) epi3_out();
            __syncthreads();
            if (tid == ISSUER) store_o(nch - 1);
        }
    }
    if (MODE == OUTPUT && tid == ISSUER) ptx::bulk_wait_all();   // O stores done before the CTA exits

    // ---- summary: stage the segment's state (fp32) in shared memory, then coalesced stores
    if (MODE == SUMMARY && ok) {
        float* st = reinterpret_cast<float*>(sm + SM_Q0);   // the slot layout, rows chunk-swizzled
        float v[32];
        float d[16];
        auto put_row = [&](int m, int rr, int c0, const float (&x)[32]) {
            float4* dst = reinterpret_cast<float4*>(st + S::mat(m) + rr * D);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                dst[(c0 / 4 + j) ^ (rr & 7)] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
        };
        if (!epi) {
        } else if (quad < 2) {
            ptx::tmem_ld32(tmem + lane_base + TM_S + half * 32, v);
            put_row(0, row, half * 32, v);
            ptx::tmem_ld32(tmem + lane_base + TM_CR + half * 32, v);
            put_row(1, row, half * 32, v);
            if (half == 0) {
                ptx::tmem_ld16(tmem + lane_base + TM_CR + 64, d);
                st[S::vec(0) + row] = d[0];
            }
        } else {
            const int r = row - 64;
            ptx::tmem_ld32(tmem + lane_base + TM_CR + half * 32, v);
            put_row(2, r, half * 32, v);
            if (half == 0) {
                ptx::tmem_ld16(tmem + lane_base + TM_CR + 64, d);
                st[S::vec(1) + r] = d[0];
            }
        }
        __syncthreads();
        float4* out4 = reinterpret_cast<float4*>(slot);
        const float4* st4 = reinterpret_cast<const float4*>(st);
        for (int f = tid; f < 3 * D * D / 4; f += NTH) {
            const int rr = (f >> 4) & (D - 1);
            out4[f] = st4[(f & ~15) | ((f & 15) ^ (rr & 7))];
        }
        for (int f = 3 * D * D / 4 + tid; f < S::size / 4; f += NTH) out4[f] = st4[f];
    }
    if (!ok) {
        if (tid == ISSUER) {
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
    if (warp == 1) ptx::tmem_dealloc(tmem, TM_COLS);
}

// ---------------------------------------------------------------- segment prefixes
// Exclusive prefix of the segment summaries under the semidirect-product combine
//     (S, C, m, R, r)_A o (S, C, m, R, r)_B
//       = (S_A + S_B, C_A + C_B, m_A + m_B, R_A + R_B + S_A C_B, r_A + r_B + S_A m_B).
// Unrolled, the prefix of segments 0..n-1 is
//     S0(n) = sum_{l<n} S_l,   R0(n) = sum_{l<n} (R_l + S0(l) C_l),
//     r0(n) = sum_{l<n} (r_l + S0(l) m_l):
// the cross term of the combine depends on the earlier part only through its S, so
// the scan splits into a prefix of S, one independent product per segment and a
// prefix of the corrected R.  Both prefixes are plain sums, so every segment and every
// matrix element runs in parallel; the result equals the Blelloch tree's (up to the
// order of fp32 additions).
//   k_prefix_run (one thread per element of S and m): S0(l), m0(l) as running sums into the
//       prefix slots;
//   k_prefix_cross (one CTA per segment x head): Y_l = R_l + S0(l) C_l and
//       y_l = r_l + S0(l) m_l, written to the prefix slot l;
//   k_prefix_sum (one thread per matrix element): R0(n) = sum_{l<n} Y_l in place.
constexpr int PX_NT = 256;

// S0(l) = sum_{m<l} S_m and m0(l) likewise, element-wise running sums (32 loads in flight).
__global__ void __launch_bounds__(PX_NT) k_prefix_run(const float* __restrict__ sums, float* __restrict__ pre, int NS,
                                                      int NSp) {
    using S = simt_layout;
    const int e = blockIdx.x * PX_NT + threadIdx.x;     // element of the S | m region
    if (e >= D * D + D) return;
    const int off = e < D * D ? S::mat(0) + e : S::vec(0) + (e - D * D);
    const size_t base = (size_t)blockIdx.y * NSp * S::size + off;
    float run = 0.f;
    for (int l0 = 0; l0 < NS; l0 += 32) {
        float y[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (l0 + i < NS) y[i] = sums[base + (size_t)(l0 + i) * S::size];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (l0 + i < NS) {
                pre[base + (size_t)(l0 + i) * S::size] = run;
                run += y[i];
            }
    }
}

__global__ void __launch_bounds__(PX_NT) k_prefix_cross(const float* __restrict__ sums, float* __restrict__ pre,
                                                        int NSp, int left_vec) {
    using S = simt_layout;
    __shared__ __align__(16) float S0s[D * (D + 4)];   // padded rows: conflict-free column walks
    __shared__ __align__(16) float Cs[D * D];
    __shared__ float ms[D], m0s[D];
    const int l = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const float* sb = sums + (size_t)bh * NSp * S::size;
    float* out = pre + ((size_t)bh * NSp + l) * S::size;
    // S0(l), m0(l): from k_prefix_run, this thread's float4 items tid + 256 i (i < 4)
    float4 acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = reinterpret_cast<const float4*>(out + S::mat(0))[tid + PX_NT * i];
    const float m0 = tid < D ? out[S::vec(0) + tid] : 0.f;
    {
        const float* cl = sb + (size_t)l * S::size;
        float4 c[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) c[i] = reinterpret_cast<const float4*>(cl + S::mat(1))[tid + PX_NT * i];
        const float mv = tid < D ? cl[S::vec(0) + tid] : 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int f = tid + PX_NT * i, r = f >> 4, c4 = f & 15;
            *reinterpret_cast<float4*>(S0s + r * (D + 4) + 4 * c4) = acc[i];
            reinterpret_cast<float4*>(Cs)[f] = c[i];
        }
        if (tid < D) {
            ms[tid] = mv;
            m0s[tid] = m0;
        }
    }
    __syncthreads();
    // Y_l = R_l + S0 C_l: thread owns rows 4 (tid / 16) .. +3, columns 4 (tid % 16) .. +3
    {
        const int r = 4 * (tid >> 4), c = 4 * (tid & 15);
        float y[4][4];
        const float* Rl = sb + (size_t)l * S::size + S::mat(2);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const float4 x = *reinterpret_cast<const float4*>(Rl + (r + a) * D + c);
            y[a][0] = x.x; y[a][1] = x.y; y[a][2] = x.z; y[a][3] = x.w;
        }
#pragma unroll 8
        for (int k = 0; k < D; ++k) {
            const float4 cv = *reinterpret_cast<const float4*>(Cs + k * D + c);
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float sv = S0s[(r + a) * (D + 4) + k];
                y[a][0] = fmaf(sv, cv.x, y[a][0]);
                y[a][1] = fmaf(sv, cv.y, y[a][1]);
                y[a][2] = fmaf(sv, cv.z, y[a][2]);
                y[a][3] = fmaf(sv, cv.w, y[a][3]);
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
            *reinterpret_cast<float4*>(out + S::mat(2) + (r + a) * D + c) = make_float4(y[a][0], y[a][1], y[a][2], y[a][3]);
        if (tid < D) {
            float yv = sb[(size_t)l * S::size + S::vec(1) + tid];
            if (left_vec)                                                    // y_l = n_l + m0(l)^T C_l
                for (int k = 0; k < D; ++k) yv = fmaf(m0s[k], Cs[k * D + tid], yv);
            else                                                             // y_l = r_l + S0(l) m_l
                for (int k = 0; k < D; ++k) yv = fmaf(S0s[tid * (D + 4) + k], ms[k], yv);
            out[S::vec(1) + tid] = yv;
        }
    }
}

// R0(n) = sum_{l<n} Y_l and r0(n) = sum_{l<n} y_l, elementwise and in place.
__global__ void __launch_bounds__(PX_NT) k_prefix_sum(float* __restrict__ pre, int NS, int NSp) {
    using S = simt_layout;
    const int e = blockIdx.x * PX_NT + threadIdx.x;     // element of the R | r region
    if (e >= D * D + D) return;
    const int off = e < D * D ? S::mat(2) + e : S::vec(1) + (e - D * D);
    float* p = pre + (size_t)blockIdx.y * NSp * S::size + off;
    float run = 0.f;
    for (int l0 = 0; l0 < NS; l0 += 32) {    // 32 loads in flight, then the dependent adds
        float y[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (l0 + i < NS) y[i] = p[(size_t)(l0 + i) * S::size];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (l0 + i < NS) {
                p[(size_t)(l0 + i) * S::size] = run;
                run += y[i];
            }
    }
}

// ---------------------------------------------------------------- streaming state
// The state after a head's T tokens is the combine of its segment summaries in order:
//   S = sum_l S_l,  C = sum_l C_l,  m = sum_l m_l,
//   R = sum_l R_l + sum_{j < NS-1} S_j Csuf(j+1),  r = sum_l r_l + sum_{j < NS-1} S_j msuf(j+1),
// with Csuf(j) = sum_{l >= j} C_l (the combine's cross terms grouped by their S factor).  One
// CTA per head; the result is written in the slot layout, which is also the state layout.
__global__ void __launch_bounds__(PX_NT) k_state_total(const float* __restrict__ sums, int NS, int NSp,
                                                       float* __restrict__ state) {
    using S = simt_layout;
    __shared__ __align__(16) float Sj[D * (D + 4)];
    __shared__ __align__(16) float Cs[D * D];
    __shared__ float ms[D];
    const int bh = blockIdx.x, tid = threadIdx.x;
    const float* sb = sums + (size_t)bh * NSp * S::size;
    float* out = state + (size_t)bh * S::size;
    const int r = 4 * (tid >> 4), c = 4 * (tid & 15);      // this thread's 4 x 4 of R
    float racc[4][4];
    for (int a = 0; a < 4; ++a)
        for (int b = 0; b < 4; ++b) racc[a][b] = 0.f;
    float rv = 0.f;
    // plain sums of S, C, m, R, r
    for (int f = tid; f < 2 * D * D / 4; f += PX_NT) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int l = 0; l < NS; ++l) {
            const float4 x = reinterpret_cast<const float4*>(sb + (size_t)l * S::size)[f];
            acc = make_float4(acc.x + x.x, acc.y + x.y, acc.z + x.z, acc.w + x.w);
        }
        reinterpret_cast<float4*>(out)[f] = acc;               // S, then C
    }
    if (tid < D) {
        float mv = 0.f;
        for (int l = 0; l < NS; ++l) {
            mv += sb[(size_t)l * S::size + S::vec(0) + tid];
            rv += sb[(size_t)l * S::size + S::vec(1) + tid];
        }
        out[S::vec(0) + tid] = mv;
    }
    for (int l = 0; l < NS; ++l)
        for (int a = 0; a < 4; ++a) {
            const float4 x = *reinterpret_cast<const float4*>(sb + (size_t)l * S::size + S::mat(2) + (r + a) * D + c);
            racc[a][0] += x.x; racc[a][1] += x.y; racc[a][2] += x.z; racc[a][3] += x.w;
        }
    // cross terms, from the last segment backwards
    for (int j = NS - 2; j >= 0; --j) {
        const float* cl = sb + (size_t)(j + 1) * S::size;
        const float* sj = sb + (size_t)j * S::size;
        for (int f = tid; f < D * D; f += PX_NT) {
            Cs[f] = (j == NS - 2 ? 0.f : Cs[f]) + cl[S::mat(1) + f];
            Sj[(f / D) * (D + 4) + f % D] = sj[S::mat(0) + f];
        }
        if (tid < D) ms[tid] = (j == NS - 2 ? 0.f : ms[tid]) + cl[S::vec(0) + tid];
        __syncthreads();
        for (int k = 0; k < D; ++k) {
            const float4 cv = *reinterpret_cast<const float4*>(Cs + k * D + c);
            for (int a = 0; a < 4; ++a) {
                const float sv = Sj[(r + a) * (D + 4) + k];
                racc[a][0] = fmaf(sv, cv.x, racc[a][0]);
                racc[a][1] = fmaf(sv, cv.y, racc[a][1]);
                racc[a][2] = fmaf(sv, cv.z, racc[a][2]);
                racc[a][3] = fmaf(sv, cv.w, racc[a][3]);
            }
        }
        if (tid < D)
            for (int k = 0; k < D; ++k) rv = fmaf(Sj[tid * (D + 4) + k], ms[k], rv);
        __syncthreads();
    }
    for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4*>(out + S::mat(2) + (r + a) * D + c) = make_float4(racc[a][0], racc[a][1], racc[a][2], racc[a][3]);
    if (tid < D) out[S::vec(1) + tid] = rv;
    for (int e = S::vec(0) + 2 * D + tid; e < S::size; e += PX_NT) out[e] = 0.f;
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

int next_pow2(int n) {
    int p = 1;
    while (p < n) p *= 2;
    return p;
}

std::atomic<int> g_segment_chunks{0};   // 0 = automatic

}  // namespace

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

bool make_map_out(CUtensorMap* map, float* base, int T, int BH) {
    EncodeTiled fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)T * D * 4};
    const cuuint32_t box[3] = {32, (cuuint32_t)C, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

Plan plan(int BH, int T, int slots, int seg_chunks) {
    Plan pl;
    pl.NC = (T + C - 1) / C;
    // Costs in chunk-times.  One walk over CTAs of `len` chunks takes (waves of CTAs) x (len +
    // about one chunk of set-up); the prefix kernels take about one per summary slot of a head.
    auto cost = [&](long long ctas, int len) { return ((ctas + slots - 1) / slots) * (long long)(len + 1); };
    // Summaries are needed for the chunks before the last output segment; shorter summary
    // segments shorten the summary walk but lengthen the prefix.
    auto summary_cost = [&](int nch, int& len_out) -> long long {
        const int ncsum = ((pl.NC + nch - 1) / nch - 1) * nch;
        len_out = nch;
        if (ncsum == 0) return 0;
        long long best = -1;
        for (int len = nch; len >= 1; len /= 2) {
            const long long c = cost((long long)BH * (ncsum / len), len) + ncsum / len;
            if (best < 0 || c < best) {
                best = c;
                len_out = len;
            }
        }
        return best;
    };
    if (seg_chunks > 0) {
        pl.NCH = seg_chunks;
    } else {
        long long best = -1;                 // ties: the longer output segment
        for (int nch = 1; nch <= 16; nch *= 2) {
            int len;
            const long long c = cost((long long)BH * ((pl.NC + nch - 1) / nch), nch) + summary_cost(nch, len);
            if (best < 0 || c <= best) {
                best = c;
                pl.NCH = nch;
            }
            if (nch >= pl.NC) break;
        }
    }
    pl.NS = (pl.NC + pl.NCH - 1) / pl.NCH;
    summary_cost(pl.NCH, pl.NCHs);
    pl.NSf = (pl.NS - 1) * pl.NCH / pl.NCHs;
    pl.ratio = pl.NCH / pl.NCHs;
    pl.NSp = next_pow2(pl.NSf + 1);
    return pl;
}

cudaError_t launch_prefix(const float* sums, float* pre, int NS, int NSp, int BH, cudaStream_t st, bool left_vec) {
    k_prefix_run<<<dim3((D * D + D + PX_NT - 1) / PX_NT, BH), PX_NT, 0, st>>>(sums, pre, NS, NSp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_prefix_cross<<<dim3(NS, BH), PX_NT, 0, st>>>(sums, pre, NSp, left_vec ? 1 : 0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_prefix_sum<<<dim3((D * D + D + PX_NT - 1) / PX_NT, BH), PX_NT, 0, st>>>(pre, NS, NSp);
    return cudaGetLastError();
}

// Segment length of the state walk: every chunk of every head is summarised, in segments of
// `len` chunks, one CTA each; the same makespan model as plan(): waves x (len + 1) chunk-times,
// plus about one per segment for the per-head combine.
static int state_segment_chunks(int BH, int T) {
    const int NC = (T + C - 1) / C;
    int best_len = 1;
    long long best = -1;
    for (int len = 1; len <= 16; len *= 2) {
        const long long ns = (NC + len - 1) / len;
        const long long c = ((BH * ns + kSMs - 1) / kSMs) * (len + 1) + ns;
        if (best < 0 || c < best) {
            best = c;
            best_len = len;
        }
        if (len >= NC) break;
    }
    return best_len;
}

size_t state_workspace_bytes(int BH, int T) {
    const int len = state_segment_chunks(BH, T);
    const int NS = ((T + C - 1) / C + len - 1) / len;
    return sizeof(float) * (size_t)BH * next_pow2(NS) * simt_layout::size;
}

cudaError_t state(const void* q, const void* k, const void* v, int BH, int T, void* ws, int* status, float* state_out,
                  cudaStream_t st) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, T, BH) || !make_map(&mk, k, T, BH) || !make_map(&mv, v, T, BH) ||
        !make_map_out(&mo, state_out, 1, 1))
        return cudaErrorInvalidValue;
    const int len = state_segment_chunks(BH, T);
    const int NS = ((T + C - 1) / C + len - 1) / len;
    Params sprm{};
    sprm.T = T; sprm.BH = BH; sprm.NCH = len; sprm.NS = NS; sprm.NSp = next_pow2(NS); sprm.ratio = 1;
    sprm.fold = 0; sprm.eps = 0.f; sprm.norm = 0;
    sprm.sums = static_cast<float*>(ws);
    sprm.pre = nullptr;
    sprm.o = nullptr;
    sprm.status = status;
    cudaError_t e;
    if ((e = set_smem(k_walk<SUMMARY>, SMEM_BYTES)) != cudaSuccess) return e;
    k_walk<SUMMARY><<<dim3(NS, BH), NTH, SMEM_BYTES, st>>>(mq, mk, mv, mo, sprm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_state_total<<<BH, PX_NT, 0, st>>>(sprm.sums, NS, sprm.NSp, state_out);
    return cudaGetLastError();
}

size_t chunk_prefix_floats(int BH, int T) {
    return (size_t)BH * next_pow2((T + C - 1) / C) * simt_layout::size;
}

cudaError_t chunk_prefixes(const void* q, const void* k, const void* v, int BH, int T, float* sums, float* pre,
                           int* status, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, T, BH) || !make_map(&mk, k, T, BH) || !make_map(&mv, v, T, BH) ||
        !make_map_out(&mo, pre, 1, 1))
        return cudaErrorInvalidValue;
    const int NS = (T + C - 1) / C;          // one chunk per summary segment
    Params sprm{};
    sprm.T = T; sprm.BH = BH; sprm.NCH = 1; sprm.NS = NS; sprm.NSp = next_pow2(NS); sprm.ratio = 1;
    sprm.sums = sums;
    sprm.status = status;
    cudaError_t e;
    if ((e = set_smem(k_walk<SUMMARY>, SMEM_BYTES)) != cudaSuccess) return e;
    k_walk<SUMMARY><<<dim3(NS, BH), NTH, SMEM_BYTES, st>>>(mq, mk, mv, mo, sprm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_prefix(sums, pre, NS, sprm.NSp, BH, st);
}

bool set_segment_chunks(int chunks) {
    if (chunks != 0 && chunks != 1 && chunks != 2 && chunks != 4 && chunks != 8 && chunks != 16) return false;
    g_segment_chunks.store(chunks);
    return true;
}

int segment_chunks() { return g_segment_chunks.load(); }

bool supported(int op, bool norm, bool bf16, int d) {
    if (!bf16 || d != D) return false;
    return op == OP_HLA2 || op == OP_AHLA || op == OP_AHLAD || (op == OP_HLA2D && !norm);
}

bool fits(int op, bool norm, int BH, int T, int seg_chunks) {
    return op != OP_AHLAD || ahla_folds(BH, T, seg_chunks, norm);
}

size_t workspace_bytes(int op, bool norm, int BH, int T, int seg_chunks) {
    if (op == OP_AHLA || op == OP_AHLAD) return ahla_workspace_bytes(BH, T, seg_chunks, norm);
    if (op == OP_HLA2D) return decay_workspace_bytes(BH, T, seg_chunks);
    const Plan pl = plan(BH, T, kSMs, seg_chunks);
    return 2 * sizeof(float) * (size_t)BH * pl.NSp * simt_layout::size;
}

int kernel_launches(int op, bool norm, int BH, int T, int seg_chunks) {
    if (op == OP_HLA2D) return decay_kernel_launches(BH, T, seg_chunks);
    // summary walk, the prefix (up to PH_MAX slots per head: folded into the output walk; else
    // three launches), output walk
    const bool ahla = op == OP_AHLA || op == OP_AHLAD;
    const Plan pl = plan(BH, T, ahla ? ahla_ctas_per_sm(norm) * kSMs : kSMs, seg_chunks);
    return pl.NSf + 1 > PH_MAX ? 5 : 2;     // else the output walker folds the prefix itself
}

cudaError_t forward(int op, bool norm, const void* q, const void* k, const void* v, const float* gamma, float eps,
                    float* o, int BH, int H, int T, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev,
                    int seg_chunks) {
    if (op == OP_AHLA) return ahla_forward(q, k, v, o, BH, H, T, norm, eps, nullptr, ws, status, st, ev, seg_chunks);
    if (op == OP_AHLAD) {
        if (!gamma) return cudaErrorInvalidValue;
        return ahla_forward(q, k, v, o, BH, H, T, norm, eps, gamma, ws, status, st, ev, seg_chunks);
    }
    if (op == OP_HLA2D) return decay_forward(q, k, v, gamma, o, BH, H, T, ws, status, st, ev, seg_chunks);
    if (op != OP_HLA2) return cudaErrorNotSupported;
    if (simt::summary_floats(OP_HLA2, D) != (size_t)simt_layout::size) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, T, BH) || !make_map(&mk, k, T, BH) || !make_map(&mv, v, T, BH) ||
        !make_map_out(&mo, o, T, BH))
        return cudaErrorInvalidValue;
    const Plan pl = plan(BH, T, kSMs, seg_chunks);
    Params prm = {};                         // the output walk
    prm.T = T; prm.BH = BH; prm.NCH = pl.NCH; prm.NS = pl.NS; prm.NSp = pl.NSp; prm.ratio = pl.ratio;
    prm.eps = eps; prm.norm = norm ? 1 : 0;
    prm.sums = static_cast<float*>(ws);
    prm.pre = prm.sums + (size_t)BH * pl.NSp * simt_layout::size;
    prm.o = o;
    prm.status = status;
    prm.fold = pl.NSf + 1 <= PH_MAX ? 1 : 0;  // few slots: each output CTA folds its own prefix
    Params sprm = prm;                       // the summary walk: shorter segments, slots 0 .. NSf - 1
    sprm.NCH = pl.NCHs; sprm.NS = pl.NSf; sprm.ratio = 1; sprm.fold = 0;
    cudaError_t e;
    if ((e = set_smem(k_walk<SUMMARY>, SMEM_BYTES)) !=
        cudaSuccess)
        return e;
    if ((e = set_smem(k_walk<OUTPUT>, SMEM_BYTES)) !=
        cudaSuccess)
        return e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    // one CTA per summary segment, plus the zero slot after them that the prefix kernels read
    // (the folding output walk reads none); the other padding slots are never read
    const int nsum = prm.fold ? (pl.NSf > 0 ? pl.NSf : 1) : pl.NSf + 1;
    k_walk<SUMMARY><<<dim3(nsum, BH), NTH, SMEM_BYTES, st>>>(mq, mk, mv, mo, sprm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    if (!prm.fold && (e = launch_prefix(prm.sums, prm.pre, pl.NSf + 1, pl.NSp, BH, st)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[2], st)) != cudaSuccess) return e;
    if (prm.fold) {
        // launched as a programmatic dependent of the summary walk: its set-up and first loads
        // overlap the summary walk's end (nothing stands between the two launches unless the
        // caller asked for phase events, which then serialise them)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(pl.NS, BH);
        cfg.blockDim = dim3(NTH);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if ((e = cudaLaunchKernelEx(&cfg, k_walk<OUTPUT>, mq, mk, mv, mo, prm)) != cudaSuccess) return e;
    } else {
        k_walk<OUTPUT><<<dim3(pl.NS, BH), NTH, SMEM_BYTES, st>>>(mq, mk, mv, mo, prm);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (ev && (e = cudaEventRecord(ev[3], st)) != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace tc
}  // namespace hla
