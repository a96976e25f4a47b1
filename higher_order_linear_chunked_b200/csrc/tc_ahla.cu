// tcgen05 tensor-core path for the asymmetric HLA forward (AHLA; bf16 inputs, d = dv = 64).
//
// "Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 2 and 4.
// Streaming state after token t: P_t = sum_{s<=t} k_s v_s^T and
// E_t = sum_{s<=t} k_s (q_s^T P_s); the output is o_t = q_t^T E_t.
//
// Per chunk of c = 128 tokens (Q, K, V: 128 x 64 tiles; P0, E0: state carried in):
//     A = L (.) (Q K^T)              (inclusive causal mask)
//     Y = Q P0 + A V                 (row s is q_s^T P_s)
//     O = Q E0 + A Y
//     P0 += K^T V,   E0 += K^T Y
// A segment of chunks walked from the zero state is summarised by (P, E, D = K^T Q);
// two segments combine as (P_A + P_B, E_A + E_B + D_B P_A).  The summary slot holds the
// transposes (P^T, D^T, E^T) in the places of (S, C, R) of the second-order slot: the
// transposed combine, E^T_AB = E^T_A + E^T_B + P^T_A D^T_B, is the second-order one
// (R_AB = R_A + R_B + S_A C_B), so the same factored prefix kernels serve both.
//
// The walker keeps the fp32 state in registers (thread = one row of [P^T ; E^T], half of
// its columns) and its bf16 copy in shared memory right after the K tile, so one MMA of
// N = 256 gives [A | Q P0 | Q E0] at once.  96 KB of shared memory and 256 TMEM columns
// per CTA: two CTAs share an SM, and one's epilogues overlap the other's MMAs.
//
// Ratio-normalised AHLA (the denominator is the same operator with V replaced by a ones
// column: o_t = q_t^T E_t / (q_t^T n_t + eps), n_t = sum_{s<=t} k_s (q_s . mK_s), mK_t =
// sum_{s<=t} k_s) runs the same walk on [V | 1]:
//     [Y | y1] = Q [P0 | mK0] + A [V | 1],   [O | den] = Q [E0 | n0] + A [Y | y1],
//     mK0 += K^T 1,   n0 += K^T y1.
// The ones column and y1 are column 0 of two extra [tok][64] tiles that sit at a fixed
// distance from V and from Y, so the N = 80 products read [V | 1] and [Y | y1] as one
// operand; the state increments (1^T K ; y1^T K) come from one M = 128 product over the two
// extra tiles stacked (rows 0 and 64 used).  The fp32 vectors mK0, n0 live in the registers
// of the threads of TMEM lanes 0 and 64, their bf16 copies in row 0 of two 16-row K-major
// tiles that give Q mK0 and Q n0 from N = 16 products.  The segment summary carries (mK, n)
// in its two vector slots; two segments combine as (mK_A + mK_B, n_A + n_B + D_B mK_A).
// The wider accumulators take 512 TMEM columns: one CTA per SM.
//
// With per-head decay (every state multiplied by gamma before each token's update) the chunk
// algebra takes the decayed masked scores At[tau][j] = g^(tau-j) A[tau][j], the row weights
// Gam = diag(g^(tau+1)) and Lam = diag(g^(len-1-tau)), and rho = g^len:
//     Y = Gam Q P0 + At V,   O = Gam Q E0 + At Y,   P0 = rho P0 + K^T Lam V,   E0 = rho E0 + K^T Lam Y
// (the normaliser's vectors likewise).  The weights are applied in fp32 before each operand's
// one rounding to bf16: At in the A epilogue, Gam on the fp32 accumulators Q P0 and Q E0 in
// TMEM, Lam on a copy of K that takes the state tile's place while the state is not read.
// A segment summary carries rho = g^length in its scalar slot; the fold weights summary l
// by the product of the later summaries' rho (the decayed combine, unrolled).
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

constexpr int ANT = 256;                 // 8 warps, two per TMEM lane quadrant
constexpr int kCtasPerSM = 2;

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t AS_V = 0;             // V  [tok][feat]
constexpr uint32_t AS_Q = AS_V + TILE;   // Q, then Y  [tok][feat]
constexpr uint32_t AS_K = AS_Q + TILE;   // K  [tok][feat]
constexpr uint32_t AS_ST = AS_K + TILE;  // [P0^T ; E0^T] K-major [128 n][64 k], directly after K
constexpr uint32_t AS_A = AS_ST + TILE;  // O staging (output walk); set-up: the carried-in state
constexpr uint32_t AS_BAR = AS_A + 2 * TILE;
constexpr uint32_t AS_TOTAL = AS_BAR + 64;
constexpr uint32_t ASMEM_BYTES = AS_TOTAL + 1024;   // + alignment slack
// ratio-normalised only
constexpr uint32_t AS_ONES = AS_A + 2 * TILE;   // [tok][64], column 0 = 1 (the rest 0)
constexpr uint32_t AS_Y1 = AS_ONES + TILE;      // [tok][64], column 0 = y1 (the rest 0)
constexpr uint32_t AS_NM = AS_Y1 + TILE;        // K-major [16][64]: row 0 = mK0^T (the rest 0)
constexpr uint32_t AS_NN = AS_NM + 2048;        // K-major [16][64]: row 0 = n0^T (the rest 0)
constexpr uint32_t AS_VEC = AS_NN + 2048;       // set-up: the carried-in mK0, n0 (fp32)
constexpr uint32_t AS_BAR_N = AS_VEC + 512;
constexpr uint32_t ASMEM_BYTES_N = AS_BAR_N + 64 + 1024;
template <bool NORM> constexpr uint32_t asmem_bytes() { return NORM ? ASMEM_BYTES_N : ASMEM_BYTES; }

// TMEM columns (fp32, 128 lanes).
constexpr uint32_t TA_A = 0;      // A (128); then the masked A as bf16 pairs at columns 0-31
                                  // (tokens 0-63) and 96-127 (tokens 64-127), the state
                                  // increment [dP^T ; dE^T] between them (TA_INC, 64)
constexpr uint32_t TA_INC = 32;
constexpr uint32_t TA_Y = 128;    // Q P0, then Y (64)
constexpr uint32_t TA_O = 192;    // output walk: Q E0, then O (64)
constexpr uint32_t TA_D = 192;    // summary walk: lanes 0-63 D^T of the segment (64)
constexpr uint32_t TA_COLS = 256;
// ratio-normalised: A and the increment as above
constexpr uint32_t TN_Y = 128;    // [Q P0 | Q mK0], then [Y | y1] (80)
constexpr uint32_t TN_O = 224;    // output walk: [Q E0 | Q n0], then [O | den] (80); summary: lanes 0-63 D^T
constexpr uint32_t TN_V = 320;    // [1^T K ; y1^T K]: lanes 0 and 64 (64)
constexpr uint32_t TN_COLS = 512;

enum Mode { SUMMARY = 0, OUTPUT = 1 };

// Threads: warp w reads TMEM lane quadrant (w & 3), i.e. tile rows 32 (w & 3) .. + 31,
// and half (w >> 2) of each tile's columns.  Thread 0 also issues the TMA loads and MMAs.
//
// Rounds of MMAs per chunk n, each followed by an epilogue:
//   R1: [A | Q P0 | Q E0] = Q [K ; P0^T ; E0^T]^T      -> E1: A masked to bf16 pairs in TMEM
//   R2: Y += A V  (summary: also D^T += Q^T K)          -> E2: Y to bf16 (over Q)
//   R3: O += A Y  (output only), [dP^T ; dE^T] = [V^T ; Y^T] K
//                                                      -> E3: state += increment, to bf16;
//                                                             O staged over A; next loads
// The staged O goes to HBM by TMA bulk stores while the next chunk's R1 runs.
template <int MODE, bool NORM, bool DECAY>
__global__ void __launch_bounds__(ANT, NORM ? 1 : kCtasPerSM)
k_ahla_walk(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + (NORM ? AS_BAR_N : AS_BAR));
    constexpr uint32_t TY = NORM ? TN_Y : TA_Y, TO = NORM ? TN_O : TA_O, TD = NORM ? TN_O : TA_D;
    constexpr uint32_t TCOLS = NORM ? TN_COLS : TA_COLS;
    uint64_t* bar_mma = bar_load + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;                     // TMEM lane = tile row
    const int seg = blockIdx.x, bh = blockIdx.y;
    using S = simt_layout;
    float* slot = MODE == OUTPUT ? p.pre + ((size_t)bh * p.NSp + seg * p.ratio) * S::size
                                 : p.sums + ((size_t)bh * p.NSp + seg) * S::size;
    // Programmatic dependent launch: the output walk may be scheduled once every summary CTA
    // has started; its CTAs that fold summaries wait for this grid's completion first.
    if (MODE == SUMMARY && tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (seg >= p.NS) {                                    // padding slots: identity (zeros, rho = 1)
        if (MODE == SUMMARY) {
            float4* s4 = reinterpret_cast<float4*>(slot);
            for (int e = tid; e < S::size / 4; e += ANT)
                s4[e] = make_float4(DECAY && e == S::vec(2) / 4 ? 1.f : 0.f, 0.f, 0.f, 0.f);
        }
        return;
    }
    // decay: g = gamma of the head, lg = log2(g) (g = 1: every weight is 1)
    const float g = DECAY ? p.gamma[bh % p.H] : 1.f;
    const float lg = DECAY ? log2f(g) : 0.f;
    const int chunk0 = seg * p.NCH;
    const int nch = min(p.NCH, (p.T + C - 1) / C - chunk0);

    if (tid == 0) {
        ptx::mbar_init(bar_load, 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    int loads_issued = 0;                                 // thread 0's count of chunk loads
    auto issue_load = [&](int n) {
        const int t0 = (chunk0 + n) * C;
        ptx::mbar_arrive_expect_tx(bar_load, 3 * TILE);
        ptx::tma_load_3d(sm + AS_Q, &tq, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + AS_K, &tk, bar_load, 0, t0, bh);
        ptx::tma_load_3d(sm + AS_V, &tv, bar_load, 0, t0, bh);
        ++loads_issued;
    };
    if (tid == 0) issue_load(0);
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, TCOLS);
        ptx::tmem_relinquish();
    }

    // Ratio-normalised: the ones tile (column 0 = 1), the y1 tile and the two vector tiles start
    // as zeros; only column 0 / row 0 of them is written later.  The threads of TMEM lanes 0
    // and 64 (vrow) hold half of the fp32 vectors mK0 and n0 each.
    const bool vrow = NORM && lane == 0 && (quad & 1) == 0;
    float st2[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) st2[i] = 0.f;
    float* vecs = reinterpret_cast<float*>(sm + AS_VEC);    // set-up: carried-in mK0 | n0
    if (NORM) {
        uint4* z = reinterpret_cast<uint4*>(sm + AS_ONES);
        for (int e = tid; e < (int)(2 * TILE + 4096) / 16; e += ANT) {
            // ones tile: 16-byte chunk e is token e / 8, physical chunk e % 8, which holds the
            // columns of logical chunk (e % 8) ^ (token % 8); logical chunk 0 starts at column 0
            uint4 u = make_uint4(0u, 0u, 0u, 0u);
            if (e < (int)TILE / 16 && ((e ^ (e >> 3)) & 7) == 0) u.x = 0x3F80u;   // bf16 1.0
            z[e] = u;
        }
    }
    // This thread's part of the fp32 state: row `row` of [P^T ; E^T], columns half*32 .. +31.
    float st[32];
    if (MODE == OUTPUT) {
        // the carried-in prefix (P^T, E^T) through shared memory: coalesced loads, rows
        // swizzled by 16-byte chunk, then every thread takes its row
        float* stage = reinterpret_cast<float*>(sm + AS_A);   // P^T [64][64] | E^T [64][64]
        // the summaries are read below: wait for the summary walk (a no-op without a
        // programmatic dependency); segment 0 reads none
        if (p.fold && seg > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        if (p.fold) {
            // n = seg * ratio slots: P0^T = sum_l P^T_l and
            // E0^T = sum_l E^T_l + sum_{m < n-1} P^T_m Dsuf^T(m+1), Dsuf^T(m) = sum_{m <= l < n} D^T_l
            // (the factored prefix, cross terms grouped by their P factor), while the first
            // loads are in flight.
            const int n = seg * p.ratio;
            const float* sb = p.sums + (size_t)bh * p.NSp * S::size;
            float* Cs = reinterpret_cast<float*>(sm + AS_ST);  // Dsuf^T [64][64] (the state tile comes later)
            float* Sm = stage + D * D;                         // P^T_m (the E^T half, for now)
            const int r = 4 * (tid >> 4), c = 4 * (tid & 15);  // this thread's 4 x 4 of E0^T
            float racc[4][4];
            float4 sacc[4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) racc[a][b] = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) sacc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            float macc = 0.f, nacc = 0.f;                      // normalised: mK0, n0 (column tid)
            // decay: summary l enters with weight w_l = prod_{l < m < n} rho_m
            float wl = 1.f;
            for (int l = n - 1; l >= 0; --l) {
                const float* sl = sb + (size_t)l * S::size;
                if (NORM && tid < D) {
                    macc = fmaf(wl, sl[S::vec(0) + tid], macc);
                    nacc = fmaf(wl, sl[S::vec(1) + tid], nacc);
                }
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float4 x = *reinterpret_cast<const float4*>(sl + S::mat(2) + (r + a) * D + c);
                    racc[a][0] = fmaf(wl, x.x, racc[a][0]); racc[a][1] = fmaf(wl, x.y, racc[a][1]);
                    racc[a][2] = fmaf(wl, x.z, racc[a][2]); racc[a][3] = fmaf(wl, x.w, racc[a][3]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 x = reinterpret_cast<const float4*>(sl + S::mat(0))[tid + ANT * i];
                    sacc[i] = make_float4(fmaf(wl, x.x, sacc[i].x), fmaf(wl, x.y, sacc[i].y), fmaf(wl, x.z, sacc[i].z),
                                          fmaf(wl, x.w, sacc[i].w));
                }
                if (DECAY) wl *= sl[S::vec(2)];
            }
            float wm = DECAY && n >= 1 ? sb[(size_t)(n - 1) * S::size + S::vec(2)] : 1.f;   // w_{n-2}
            for (int m = n - 2; m >= 0; --m) {
                const float* cl = sb + (size_t)(m + 1) * S::size;
                const float* smp = sb + (size_t)m * S::size;
                for (int f = tid; f < D * D / 4; f += ANT) {
                    const float4 x = reinterpret_cast<const float4*>(cl + S::mat(1))[f];
                    const float4 o = m == n - 2 ? make_float4(0.f, 0.f, 0.f, 0.f) : reinterpret_cast<float4*>(Cs)[f];
                    reinterpret_cast<float4*>(Cs)[f] = make_float4(o.x + x.x, o.y + x.y, o.z + x.z, o.w + x.w);
                    float4 pm = reinterpret_cast<const float4*>(smp + S::mat(0))[f];
                    if (DECAY) pm = make_float4(wm * pm.x, wm * pm.y, wm * pm.z, wm * pm.w);
                    reinterpret_cast<float4*>(Sm)[f] = pm;     // w_m P^T_m
                }
                __syncthreads();
                if (NORM && tid < D) {                         // n0 += w_m D_suf(m+1) mK_m
                    const float* mk = smp + S::vec(0);
                    float t = 0.f;
                    for (int k = 0; k < D; ++k) t = fmaf(mk[k], Cs[k * D + tid], t);
                    nacc = fmaf(wm, t, nacc);
                }
                if (DECAY) wm *= smp[S::vec(2)];
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
                __syncthreads();
            }
            if (NORM && tid < D) {
                vecs[tid] = macc;
                vecs[D + tid] = nacc;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int f = tid + ANT * i, rr = f >> 4, ch = (f & 15) ^ (rr & 7);
                reinterpret_cast<float4*>(stage)[rr * 16 + ch] = sacc[i];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int i = r + a, j = c + b;
                    stage[D * D + i * D + ((((j >> 2) ^ (i & 7)) << 2) | (j & 3))] = racc[a][b];
                }
        } else {
            const float4* p4 = reinterpret_cast<const float4*>(slot + S::mat(0));
            const float4* e4 = reinterpret_cast<const float4*>(slot + S::mat(2));
            if (NORM && tid < D) {
                vecs[tid] = slot[S::vec(0) + tid];
                vecs[D + tid] = slot[S::vec(1) + tid];
            }
            float4 xp[4], xe[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xp[i] = p4[tid + ANT * i];
                xe[i] = e4[tid + ANT * i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int f = tid + ANT * i, rr = f >> 4, ch = (f & 15) ^ (rr & 7);
                reinterpret_cast<float4*>(stage)[rr * 16 + ch] = xp[i];
                reinterpret_cast<float4*>(stage + D * D)[rr * 16 + ch] = xe[i];
            }
        }
        __syncthreads();
        const int r = row & 63;
        const float4* src = reinterpret_cast<const float4*>(stage + (row >> 6) * D * D) + r * 16;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 x = src[(half * 8 + j) ^ (r & 7)];
            st[4 * j] = x.x; st[4 * j + 1] = x.y; st[4 * j + 2] = x.z; st[4 * j + 3] = x.w;
        }
        if (vrow) {
#pragma unroll
            for (int i = 0; i < 32; ++i) st2[i] = vecs[(quad >> 1) * D + half * 32 + i];
            st_row32(sm + (quad ? AS_NN : AS_NM), 0, half * 32, st2);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) st[i] = 0.f;
    }
    st_row32(sm + AS_ST, row, half * 32, st);
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;

    const uint32_t sbase = ptx::smem_u32(sm);
    constexpr uint32_t I_R1 = ptx::idesc_bf16(128, (MODE == OUTPUT && !NORM) ? 256 : 192, false, false);
    constexpr uint32_t I_N64_KK = ptx::idesc_bf16(128, 64, false, false);
    constexpr uint32_t I_N16_KK = ptx::idesc_bf16(128, 16, false, false);
    constexpr uint32_t I_NV_KM = ptx::idesc_bf16(128, NORM ? 80 : 64, false, true);   // [V | 1], [Y | y1]
    constexpr uint32_t I_N64_MM = ptx::idesc_bf16(128, 64, true, true);
    auto k1 = [](uint64_t d0, int s) { return d0 + (uint64_t)(s * 2); };                         // +32 B
    auto mn = [](uint64_t d0, int s) { return d0 + (uint64_t)(s * 128); };                       // +2048 B
    // Operand descriptors (built where they are used: only thread 0 issues MMAs).
    //   Q [K ; P0^T ; E0^T]^T : K-major Q and K-major B rows K, then P0^T, E0^T
    //   A V, A Y              : K-major A (two atoms), MN-major V / Y
    //   [V^T ; Y^T] K, [Q^T ; K^T] K : stacked MN-major A operands, MN-major K
    auto issue_r1 = [&]() {
        const uint64_t dQ = kdesc(sbase + AS_Q, 0), dKS = kdesc(sbase + AS_K, 0);
        for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TA_A, k1(dQ, s), k1(dKS, s), I_R1, s > 0);
        if (NORM) {                          // Q mK0 -> y1 column; output: Q E0, Q n0 -> den column
            const uint64_t dNM = kdesc(sbase + AS_NM, 0);
            for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TY + 64, k1(dQ, s), k1(dNM, s), I_N16_KK, s > 0);
            if (MODE == OUTPUT) {
                const uint64_t dE = kdesc(sbase + AS_ST + 64 * 128, 0), dNN = kdesc(sbase + AS_NN, 0);
                for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TO, k1(dQ, s), k1(dE, s), I_N64_KK, s > 0);
                for (int s = 0; s < 4; ++s) ptx::umma_bf16(tmem + TO + 64, k1(dQ, s), k1(dNN, s), I_N16_KK, s > 0);
            }
        }
    };
    // masked A as bf16 pairs: K-step s (tokens 16 s .. 16 s + 15)
    auto a_pairs = [&](int s) { return tmem + TA_A + (s < 4 ? 8 * s : 96 + 8 * (s - 4)); };
    auto issue_r2 = [&](int n) {
        const uint64_t dVm = mdesc(sbase + AS_V, NORM ? AS_ONES - AS_V : TILE, 0);
        for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TY, a_pairs(s), mn(dVm, s), I_NV_KM, 1);
        if (MODE == SUMMARY) {   // lanes 0-63: D^T += Q^T K (lanes 64-127 take K^T K, unused)
            const uint64_t dQK = mdesc(sbase + AS_Q, AS_K - AS_Q, 0), dKm = mdesc(sbase + AS_K, TILE, 0);
            for (int s = 0; s < 8; ++s)
                ptx::umma_bf16(tmem + TD, mn(dQK, s), mn(dKm, s), I_N64_MM, (n > 0 || s > 0) ? 1u : 0u);
        }
    };
    auto issue_r3 = [&]() {
        // the increments' B operand: K, or with decay Lam K (staged over the state tile)
        const uint64_t dKm = mdesc(sbase + (DECAY ? AS_ST : AS_K), TILE, 0);
        if (MODE == OUTPUT) {
            const uint64_t dYm = mdesc(sbase + AS_Q, NORM ? AS_Y1 - AS_Q : TILE, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16_ts(tmem + TO, a_pairs(s), mn(dYm, s), I_NV_KM, 1);
        }
        const uint64_t dVY = mdesc(sbase + AS_V, AS_Q - AS_V, 0);
        for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + TA_INC, mn(dVY, s), mn(dKm, s), I_N64_MM, s > 0);
        if (NORM) {                          // [1^T K ; y1^T K] at lanes 0 and 64
            const uint64_t dOY = mdesc(sbase + AS_ONES, AS_Y1 - AS_ONES, 0);
            for (int s = 0; s < 8; ++s) ptx::umma_bf16(tmem + TN_V, mn(dOY, s), mn(dKm, s), I_N64_MM, s > 0);
        }
    };

    uint32_t mma_phase = 0;
    bool ok = true;                          // agreed by the whole block
    bool issuer_ok = true;                   // thread 0's load waits since the last agreement
    // Thread 0 commits the MMAs issued so far and waits for them (bounded); the block agrees,
    // on that and on thread 0's own load waits.
    auto commit_wait = [&]() -> bool {
        bool good = true;
        ptx::tc_fence_before();
        if (tid == 0) {
            ptx::umma_commit(bar_mma);
            good = ptx::mbar_wait(bar_mma, mma_phase) && issuer_ok;
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

    // 32 fp32 columns of this lane -> 16 bf16 pairs in TMEM (column 2i in the low half); on
    // the diagonal block the columns past this lane's token are cleared; nullptr: zeros.
    auto st_pairs = [&](uint32_t tcol, const float* x, bool diag) {
        uint32_t r[16];
        if (x == nullptr) {
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = 0u;
        } else if (diag) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                r[i] = ptx::pack_bf16(2 * i > lane ? 0.f : x[2 * i], 2 * i + 1 > lane ? 0.f : x[2 * i + 1]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = ptx::pack_bf16(x[2 * i], x[2 * i + 1]);
        }
        ptx::tmem_st16u(tmem + lane_base + tcol, r);
    };
    // E1: A (masked, inclusive diagonal) -> bf16 pairs, in place: this warp reads its token
    // blocks b0 = 2 half and b0 + 1 (columns 64 half .. +63) and writes their pairs to columns
    // 96 half .. +31, which it has read itself.  Blocks above the diagonal (b > quad) become
    // zeros (the A of every chunk overwrites them).
    // decay weights g^(tau - j) on this lane's token block b (tau = row): below the diagonal
    // g^(tau - j1) g^(j1 - j) with j1 the block's last token (both exponents >= 0); on it
    // g^(lane - i) for i <= lane (the rest is masked)
    auto weigh = [&](float (&x)[32], int b) {
        if (b < quad) {
            float w = exp2f((float)(row - 32 * b - 31) * lg);
#pragma unroll
            for (int i = 31; i >= 0; --i) {
                x[i] *= w;
                w *= g;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] *= exp2f((float)max(lane - i, 0) * lg);
        }
    };
    // fp32 TMEM columns [col, col + 16) of this lane times sc, in place
    auto scale16 = [&](uint32_t col, float sc) {
        float v[16];
        ptx::tmem_ld16(tmem + lane_base + col, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] *= sc;
        ptx::tmem_st16(tmem + lane_base + col, v);
    };
    auto epi1 = [&](int n) {
        const int b0 = 2 * half;
        const uint32_t pc = TA_A + 96 * half;
        float v0[32], v1[32];
        if (b0 + 1 <= quad) {
            if (DECAY) {
                // one block at a time (registers), in an order in which no pair store lands on
                // fp32 columns not yet read: half 0 stores to columns 0-31 (block 0 first), half 1
                // to columns 96-127 (block 3 first)
                if (half == 0) {
                    ptx::tmem_ld32(tmem + lane_base + TA_A + 32 * b0, v0);
                    weigh(v0, b0);
                    st_pairs(pc, v0, false);
                    ptx::tmem_ld32(tmem + lane_base + TA_A + 32 * (b0 + 1), v1);
                    weigh(v1, b0 + 1);
                    st_pairs(pc + 16, v1, b0 + 1 == quad);
                } else {
                    ptx::tmem_ld32(tmem + lane_base + TA_A + 32 * (b0 + 1), v1);
                    weigh(v1, b0 + 1);
                    st_pairs(pc + 16, v1, b0 + 1 == quad);
                    ptx::tmem_ld32(tmem + lane_base + TA_A + 32 * b0, v0);
                    weigh(v0, b0);
                    st_pairs(pc, v0, false);
                }
            } else {
                ptx::tmem_ld32x2(tmem + lane_base + TA_A + 32 * b0, tmem + lane_base + TA_A + 32 * (b0 + 1), v0, v1);
                st_pairs(pc, v0, false);
                st_pairs(pc + 16, v1, b0 + 1 == quad);
            }
        } else if (b0 == quad) {
            ptx::tmem_ld32(tmem + lane_base + TA_A + 32 * b0, v0);
            if (DECAY) weigh(v0, b0);
            st_pairs(pc, v0, true);
            st_pairs(pc + 16, nullptr, false);
        } else {
            st_pairs(pc, nullptr, false);
            st_pairs(pc + 16, nullptr, false);
        }
        if (DECAY) {
            // Gam on Q P0 (and Q mK0), and in the output walk on Q E0 (and Q n0)
            const float gr = exp2f((float)(row + 1) * lg);
            scale16(TY + half * 32, gr);
            scale16(TY + half * 32 + 16, gr);
            if (NORM && half == 0) scale16(TY + 64, gr);
            if (MODE == OUTPUT) {
                scale16(TO + half * 32, gr);
                scale16(TO + half * 32 + 16, gr);
                if (NORM && half == 0) scale16(TO + 64, gr);
            }
            // Lam K over the state tile (R1 has read the state; E3 rewrites it): this lane's row,
            // half of its 16-byte chunks; rows past the sequence are zero
            const int len = min(C, p.T - (chunk0 + n) * C);
            const float lam = row < len ? exp2f((float)(len - 1 - row) * lg) : 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t off = row * 128 + ((((half * 4 + j) ^ row) & 7) << 4);
                uint4 u = *reinterpret_cast<const uint4*>(sm + AS_K + off);
                uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
                    w[e] = ptx::pack_bf16(lam * f.x, lam * f.y);
                }
                *reinterpret_cast<uint4*>(sm + AS_ST + off) = u;
            }
        }
        ptx::tmem_st_wait();
    };
    // E2: Y -> AS_Q (the Q tile is no longer read)
    auto epi2 = [&]() {
        float v[32];
        ptx::tmem_ld32(tmem + lane_base + TY + half * 32, v);
        st_row32(sm + AS_Q, row, half * 32, v);
        if (NORM && half == 0) {             // y1 -> column 0 of the y1 tile
            float w[16];
            ptx::tmem_ld16(tmem + lane_base + TY + 64, w);
            *reinterpret_cast<bf16*>(sm + AS_Y1 + row * 128 + ((row & 7) << 4)) = __float2bfloat16_rn(w[0]);
        }
    };
    // E3: state += increment, its bf16 copy -> AS_ST; O of the chunk (fp32) staged over the
    // A tile as two [128 rows][32 cols] boxes in the 128B-swizzled TMA layout
    auto epi3 = [&](int n) {
        float v[32];
        const float rho = DECAY ? exp2f((float)min(C, p.T - (chunk0 + n) * C) * lg) : 1.f;
        ptx::tmem_ld32(tmem + lane_base + TA_INC + half * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) st[i] = fmaf(rho, st[i], v[i]);
        if (MODE == OUTPUT || row < 64) st_row32(sm + AS_ST, row, half * 32, st);
        if (NORM && (quad & 1) == 0) {       // lanes 0 and 64: mK0 += K^T 1, n0 += K^T y1
            ptx::tmem_ld32(tmem + lane_base + TN_V + half * 32, v);
            if (lane == 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) st2[i] = fmaf(rho, st2[i], v[i]);
                if (quad == 0 || MODE == OUTPUT) st_row32(sm + (quad ? AS_NN : AS_NM), 0, half * 32, st2);
            }
        }
        if (MODE == OUTPUT) {
            ptx::tmem_ld32(tmem + lane_base + TO + half * 32, v);
            if (NORM) {
                float w[16];
                ptx::tmem_ld16(tmem + lane_base + TO + 64, w);
                const float scale = 1.f / (w[0] + p.eps);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= scale;
            }
            float4* box = reinterpret_cast<float4*>(sm + AS_A + half * (C * 128) + row * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                box[j ^ (row & 7)] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
    };
    // Thread 0: store the staged O of chunk n (rows past T are clipped by the tensor map).
    auto store_o = [&](int n) {
        const int t0 = (chunk0 + n) * C;
        ptx::tma_store_3d(&to, sm + AS_A, 0, t0, bh);
        ptx::tma_store_3d(&to, sm + AS_A + C * 128, 32, t0, bh);
        ptx::bulk_commit();
    };

    // ---- the walk
    // ok changes only where the block agrees, so every thread runs the same barriers.
    for (int n = 0; n < nch && ok; ++n) {
        if (tid == 0) {
            if (MODE == OUTPUT && n > 0) store_o(n - 1);
            issuer_ok = ptx::mbar_wait(bar_load, n & 1);
            if (issuer_ok) {
                ptx::tc_fence_after();
                issue_r1();
            }
        }
        if (!commit_wait()) { ok = false; break; }          // loads and R1 done
        epi1(n);
        sync_for_mma();
        if (tid == 0) issue_r2(n);
        if (!commit_wait()) { ok = false; break; }          // R2 done
        epi2();
        sync_for_mma();
        if (tid == 0) {
            issue_r3();
            if (MODE == OUTPUT) ptx::bulk_wait_read();      // the O staging is free for E3 again
        }
        if (!commit_wait()) { ok = false; break; }          // R3 done: Q/Y, K, V free
        if (tid == 0 && n + 1 < nch) issue_load(n + 1);
        epi3(n);
        sync_for_mma();
    }
    if (MODE == OUTPUT && ok && tid == 0) store_o(nch - 1);

    // ---- summary: stage (P^T, D^T, E^T) in shared memory, then coalesced stores
    if (MODE == SUMMARY && ok) {
        float* stg = reinterpret_cast<float*>(sm + AS_V);  // 48 KB over V, Q, K (all MMAs done)
        auto put_row = [&](int m, int rr, const float (&x)[32]) {
            float4* dst = reinterpret_cast<float4*>(stg + S::mat(m) + rr * D);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                dst[(half * 8 + j) ^ (rr & 7)] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
        };
        if (quad < 2) {
            float v[32];
            put_row(0, row, st);                                   // P^T
            ptx::tmem_ld32(tmem + lane_base + TD + half * 32, v);
            put_row(1, row, v);                                    // D^T
        } else {
            put_row(2, row - 64, st);                              // E^T
        }
        __syncthreads();
        float4* out4 = reinterpret_cast<float4*>(slot);
        const float4* st4 = reinterpret_cast<const float4*>(stg);
        for (int f = tid; f < 3 * D * D / 4; f += ANT) {
            const int rr = (f >> 4) & (D - 1);
            out4[f] = st4[(f & ~15) | ((f & 15) ^ (rr & 7))];
        }
        // decay: rho of the segment = g^(its length)
        const float rho_seg = DECAY ? exp2f((float)min(nch * C, p.T - chunk0 * C) * lg) : 0.f;
        for (int f = (NORM ? S::vec(2) : S::vec(0)) / 4 + tid; f < S::size / 4; f += ANT)
            out4[f] = make_float4(DECAY && f == S::vec(2) / 4 ? rho_seg : 0.f, 0.f, 0.f, 0.f);
        if (vrow) {                          // (mK, n) of the segment
#pragma unroll
            for (int i = 0; i < 32; ++i) slot[S::vec(quad >> 1) + half * 32 + i] = st2[i];
        }
    }
    if (MODE == OUTPUT && tid == 0) ptx::bulk_wait_all();  // O stores done before the CTA exits
    if (!ok && tid == 0) {
        set_status(p.status, DEV_TIMEOUT);
        // let a load and MMAs already in flight land before TMEM and smem are released
        if (loads_issued > 0) ptx::mbar_wait(bar_load, (loads_issued - 1) & 1, 100000000ull);
        ptx::umma_commit(bar_mma);
        ptx::mbar_wait(bar_mma, mma_phase, 100000000ull);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, TCOLS);
}

}  // namespace

int ahla_ctas_per_sm(bool norm) { return norm ? 1 : kCtasPerSM; }

size_t ahla_workspace_bytes(int BH, int T, int seg_chunks, bool norm) {
    const Plan pl = plan(BH, T, ahla_ctas_per_sm(norm) * kSMs, seg_chunks);
    return 2 * sizeof(float) * (size_t)BH * pl.NSp * simt_layout::size;
}

bool ahla_folds(int BH, int T, int seg_chunks, bool norm) {
    const Plan pl = plan(BH, T, ahla_ctas_per_sm(norm) * kSMs, seg_chunks);
    return pl.NSf + 1 <= PH_MAX;
}

template <bool NORM, bool DECAY>
static cudaError_t ahla_run(const void* q, const void* k, const void* v, float* o, int BH, int H, int T, float eps,
                            const float* gamma, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev,
                            int seg_chunks) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, T, BH) || !make_map(&mk, k, T, BH) || !make_map(&mv, v, T, BH) ||
        !make_map_out(&mo, o, T, BH))
        return cudaErrorInvalidValue;
    const Plan pl = plan(BH, T, ahla_ctas_per_sm(NORM) * kSMs, seg_chunks);
    Params prm = {};                         // the output walk
    prm.T = T; prm.BH = BH; prm.NCH = pl.NCH; prm.NS = pl.NS; prm.NSp = pl.NSp; prm.ratio = pl.ratio;
    prm.eps = eps; prm.norm = NORM ? 1 : 0;
    prm.sums = static_cast<float*>(ws);
    prm.pre = prm.sums + (size_t)BH * pl.NSp * simt_layout::size;
    prm.o = o;
    prm.status = status;
    prm.gamma = gamma;
    prm.H = H;
    prm.fold = pl.NSf + 1 <= PH_MAX ? 1 : 0;  // few slots: each output CTA folds its own prefix
    // the decayed walk folds its prefix only (the prefix kernels carry no decay)
    if (DECAY && !prm.fold) return cudaErrorNotSupported;
    Params sprm = prm;                       // the summary walk: shorter segments, slots 0 .. NSf - 1
    sprm.NCH = pl.NCHs; sprm.NS = pl.NSf; sprm.ratio = 1; sprm.fold = 0;
    constexpr int SMEM = (int)asmem_bytes<NORM>();
    auto ksum = k_ahla_walk<SUMMARY, NORM, DECAY>;
    auto kout = k_ahla_walk<OUTPUT, NORM, DECAY>;
    cudaError_t e;
    if ((e = set_smem(ksum, SMEM)) != cudaSuccess) return e;
    if ((e = set_smem(kout, SMEM)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    ksum<<<dim3(pl.NSp, BH), ANT, SMEM, st>>>(mq, mk, mv, mo, sprm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    if (!prm.fold && (e = launch_prefix(prm.sums, prm.pre, pl.NSf + 1, pl.NSp, BH, st, NORM)) != cudaSuccess)
        return e;
    if (ev && (e = cudaEventRecord(ev[2], st)) != cudaSuccess) return e;
    if (prm.fold) {
        // a programmatic dependent of the summary walk (see the second-order forward)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(pl.NS, BH);
        cfg.blockDim = dim3(ANT);
        cfg.dynamicSmemBytes = SMEM;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if ((e = cudaLaunchKernelEx(&cfg, kout, mq, mk, mv, mo, prm)) != cudaSuccess) return e;
    } else {
        kout<<<dim3(pl.NS, BH), ANT, SMEM, st>>>(mq, mk, mv, mo, prm);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (ev && (e = cudaEventRecord(ev[3], st)) != cudaSuccess) return e;
    return cudaSuccess;
}

cudaError_t ahla_forward(const void* q, const void* k, const void* v, float* o, int BH, int H, int T, bool norm,
                         float eps, const float* gamma, void* ws, int* status, cudaStream_t st, cudaEvent_t* ev,
                         int seg_chunks) {
    if (gamma) {
        if (norm) return ahla_run<true, true>(q, k, v, o, BH, H, T, eps, gamma, ws, status, st, ev, seg_chunks);
        return ahla_run<false, true>(q, k, v, o, BH, H, T, 0.f, gamma, ws, status, st, ev, seg_chunks);
    }
    if (norm) return ahla_run<true, false>(q, k, v, o, BH, H, T, eps, nullptr, ws, status, st, ev, seg_chunks);
    return ahla_run<false, false>(q, k, v, o, BH, H, T, 0.f, nullptr, ws, status, st, ev, seg_chunks);
}

}  // namespace tc
}  // namespace hla
