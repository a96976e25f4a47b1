// CUDA-core (FFMA, fp32) chunk-parallel path for every HLA op.
//
// "Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 4:
// the sequence is cut into chunks; each chunk's summary is built on its own
// (chunk kernel), an exclusive scan with the semidirect-product combine turns them
// into carried-in prefixes (one block per head folding the summaries in order, in
// one launch; or, for the third order and when three summaries do not fit in shared
// memory, the Blelloch tree, one launch per level), and each chunk's output applies
// its prefix (output kernel).  This path serves
// the fp32 workloads (whose tolerance rules out single-pass TF32 tensor cores),
// every op at d in {32, 64}, and bf16 inputs the tcgen05 path does not cover.
//
// Per chunk (c tokens, local 0-based index; A* = Q K^T, A = L (.) A*):
//   second order   summary  S = K^T K, C = Q^T V, m = Q^T 1,
//                           R = S C - G = K^T (A^T V), r = S m - h = K^T (A^T 1)
//                  combine  R_AB = R_A + R_B + S_A C_B, r_AB = r_A + r_B + S_A m_B
//                  output   W = L (.) (Q S0 Q^T + A A^T), O = Q R0 + W V,
//                           den = Q r0 + W 1 (ratio-normalised)
//   decayed        state (S, C, G, Khat, m, h, rho), rho = gamma^len, Khat = K^T K;
//                  combine and output formulas in combine_into / k_output below
//   AHLA           summary  P = K^T V, Dm = K^T Q, E = K^T (A V);  mK = K^T 1, n = K^T (A 1)
//                  combine  E_AB = E_A + E_B + Dm_B P_A (n likewise, with mK for P);
//                  output   O = Q E0 + A (Q P0 + A V);  ratio-normalised: den = Q n0 + A (Q mK0 + A 1)
//   third order    summary  S, Q2 = Q^T Q, P, X = Q^T (A V), Z = K^T (A^T Q),
//                           F = K^T (A^T (A V));
//                  output   W as above, O = Q F0 + W (Q P0 + A V);  with V replaced by a ones
//                           column: vectors mK, X1, F1 and den = Q F1_0 + W (Q mK0 + A 1)
//   unmasked       summary  S = K^T K, C = Q^T V;  combine S, C add;
//   second order   output   W = L (.) (Q S0 Q^T + A A*^T), O = Q (S0 C0) + W V + (A K) C0
#include <algorithm>

#include <cooperative_groups.h>
#include <type_traits>

#include "common.cuh"
#include "simt.h"
#include "tc.h"

namespace hla {
namespace simt {

constexpr int C = 64;        // chunk length
constexpr int LDC = C + 1;   // padded row stride of c x c tiles in shared memory
constexpr int NT = 256;      // threads per block

template <int D>
struct Dim {
    static constexpr int LD = D + 1;  // padded row stride of c x D / D x D tiles
};

// Programmatic dependent launch between the kernels of one forward: a kernel lets the next one
// launch as soon as all of its CTAs have started (pdl_release), and the next one waits for its
// completion (pdl_wait) before it reads what that kernel wrote; loads of the forward's inputs go
// before the wait.  Both are no-ops for a kernel launched without the attribute.  A pointer read
// after the wait carries no __restrict__: with it the compiler may take the data as fixed for the
// whole kernel and move a batch of its loads above the wait, before the earlier kernel is done.
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
static cudaError_t launch_dep(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------------------
// Summary layout: NMAT matrices D x D, then NVEC vectors D, then one scalar.
// ---------------------------------------------------------------------------
template <int OP, int D>
struct Sum {
    static constexpr int DD = D * D;
    static constexpr int NMAT = (OP == OP_HLA3 || OP == OP_HLA3D) ? 6 : OP == OP_HLA2D ? 4 : OP == OP_HLA2U ? 2 : 3;
    static constexpr int NVEC = (OP == OP_HLA2 || OP == OP_HLA2D || OP == OP_AHLA || OP == OP_AHLAD) ? 2
                                : (OP == OP_HLA3 || OP == OP_HLA3D) ? 3 : 0;
    static constexpr int VEC0 = NMAT * DD;
    static constexpr int SCAL = VEC0 + NVEC * D;
    static constexpr int SIZE = (SCAL + 4 + 31) / 32 * 32;
    __host__ __device__ static constexpr int mat(int i) { return i * DD; }
    __host__ __device__ static constexpr int vec(int i) { return VEC0 + i * D; }
};
// Matrix / vector slots.
//   OP_HLA2 : S=0 C=1 R=2 ; m=0 r=1
//   OP_HLA2D: S=0 C=1 G=2 Khat=3 ; m=0 h=1 ; scalar rho
//   OP_AHLA : P=0 E=1 Dm=2 ; mK=0 n=1            (the ratio-normaliser's P and E: V -> ones)
//   OP_HLA3 : S=0 Q2=1 P=2 F=3 X=4 Z=5 ; mK=0 X1=1 F1=2   (likewise for P, X, F)
//   OP_HLA2U: S=0 C=1
//   OP_AHLAD: as OP_AHLA (Dm undecayed) ; scalar rho
//   OP_HLA3D: as OP_HLA3 (Q2 weighted by gamma^position, X and Z undecayed sums) ; scalar rho

size_t summary_floats(int op, int d) {
    switch (op) {
    case OP_HLA2: return d == 32 ? Sum<OP_HLA2, 32>::SIZE : Sum<OP_HLA2, 64>::SIZE;
    case OP_HLA2D: return d == 32 ? Sum<OP_HLA2D, 32>::SIZE : Sum<OP_HLA2D, 64>::SIZE;
    case OP_AHLA: return d == 32 ? Sum<OP_AHLA, 32>::SIZE : Sum<OP_AHLA, 64>::SIZE;
    case OP_HLA3: return d == 32 ? Sum<OP_HLA3, 32>::SIZE : Sum<OP_HLA3, 64>::SIZE;
    case OP_HLA2U: return d == 32 ? Sum<OP_HLA2U, 32>::SIZE : Sum<OP_HLA2U, 64>::SIZE;
    case OP_AHLAD: return d == 32 ? Sum<OP_AHLAD, 32>::SIZE : Sum<OP_AHLAD, 64>::SIZE;
    case OP_HLA3D: return d == 32 ? Sum<OP_HLA3D, 32>::SIZE : Sum<OP_HLA3D, 64>::SIZE;
    }
    return 0;
}

// the ops whose summaries carry rho = gamma^length (identity: 1)
__host__ __device__ constexpr bool decayed_op(int op) { return op == OP_HLA2D || op == OP_AHLAD || op == OP_HLA3D; }

// ---------------------------------------------------------------------------
// Block-cooperative small matrix products in shared/global memory.
//   out(m,n) = init(m,n) + sum_k a1(m,k) b1(k,n) [+ sum_k a2(m,k) b2(k,n) ...]
// Thread owns the R x R outputs (tm + i*M/R, tn + j*N/R), R = 4 unless a caller spreads a small
// product over more threads: a() reads are broadcasts within a warp, b() reads walk consecutive
// n (conflict-free).
// ---------------------------------------------------------------------------
struct Zero {
    __device__ float operator()(int, int) const { return 0.f; }
};

template <int M, int N, int K1, int K2, int K3, int R = 4, class A1, class B1, class A2, class B2, class A3,
          class B3, class FI, class FS>
__device__ __forceinline__ void mm3(A1 a1, B1 b1, A2 a2, B2 b2, A3 a3, B3 b3, FI init, FS store) {
    static_assert(M % R == 0 && N % R == 0, "tile");
    constexpr int RM = M / R, RN = N / R;
    for (int tile = threadIdx.x; tile < RM * RN; tile += blockDim.x) {
        const int tm = tile / RN, tn = tile % RN;
        float acc[R][R];
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int j = 0; j < R; ++j) acc[i][j] = init(tm + i * RM, tn + j * RN);
#pragma unroll 4
        for (int kk = 0; kk < K1; ++kk) {
            float av[R], bv[R];
#pragma unroll
            for (int i = 0; i < R; ++i) av[i] = a1(tm + i * RM, kk);
#pragma unroll
            for (int j = 0; j < R; ++j) bv[j] = b1(kk, tn + j * RN);
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int j = 0; j < R; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
#pragma unroll 4
        for (int kk = 0; kk < K2; ++kk) {
            float av[R], bv[R];
#pragma unroll
            for (int i = 0; i < R; ++i) av[i] = a2(tm + i * RM, kk);
#pragma unroll
            for (int j = 0; j < R; ++j) bv[j] = b2(kk, tn + j * RN);
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int j = 0; j < R; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
#pragma unroll 4
        for (int kk = 0; kk < K3; ++kk) {
            float av[R], bv[R];
#pragma unroll
            for (int i = 0; i < R; ++i) av[i] = a3(tm + i * RM, kk);
#pragma unroll
            for (int j = 0; j < R; ++j) bv[j] = b3(kk, tn + j * RN);
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int j = 0; j < R; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int j = 0; j < R; ++j) store(tm + i * RM, tn + j * RN, acc[i][j]);
    }
}

template <int M, int N, int K, class A1, class B1, class FI, class FS>
__device__ __forceinline__ void mm(A1 a, B1 b, FI init, FS store) {
    mm3<M, N, K, 0, 0>(a, b, a, b, a, b, init, store);
}

template <int M, int N, int K1, int K2, class A1, class B1, class A2, class B2, class FI, class FS>
__device__ __forceinline__ void mm2(A1 a1, B1 b1, A2 a2, B2 b2, FI init, FS store) {
    mm3<M, N, K1, K2, 0>(a1, b1, a2, b2, a1, b1, init, store);
}

// Row-major shared tile accessors.
struct Tile {                      // element (r, c) of a tile with row stride ld
    const float* p;
    int ld;
    __device__ float operator()(int r, int c) const { return p[r * ld + c]; }
};
struct TileT {                     // transposed view: element (r, c) = tile[c][r]
    const float* p;
    int ld;
    __device__ float operator()(int r, int c) const { return p[c * ld + r]; }
};
struct GTile {                  // element (r, c) of a row-major matrix in global memory
    const float* p;
    int ld;
    __device__ float operator()(int r, int c) const { return p[r * ld + c]; }
};
struct Put {                    // plain store into a tile
    float* p;
    int ld;
    __device__ void operator()(int r, int c, float x) const { p[r * ld + c] = x; }
};

// Load `rows` chunk rows (zero beyond T) of a [T][D] head slice into a padded fp32 tile.
template <int D, typename TIn>
__device__ __forceinline__ void load_rows(float* dst, const TIn* src, int t0, int T) {
    constexpr int LD = Dim<D>::LD, PER = C * D / NT;
    static_assert(C * D % NT == 0, "whole tiles per pass");
    if constexpr (PER > 8) {                 // d = 64: one value at a time (keeps the registers of
        for (int e = threadIdx.x; e < C * D; e += blockDim.x) {     // the kernels around it)
            const int t = t0 + e / D;
            dst[(e / D) * LD + e % D] = (t < T) ? to_f32(src[(size_t)t * D + e % D]) : 0.f;
        }
    } else {                                 // d = 32: all loads of the tile in flight, then the stores
        float x[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = threadIdx.x + i * NT, t = t0 + e / D;
            x[i] = (t < T) ? to_f32(src[(size_t)t * D + e % D]) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = threadIdx.x + i * NT;
            dst[(e / D) * LD + e % D] = x[i];
        }
    }
}

// Load a D x D matrix (global, dense) into a padded tile; `scale` applied.
template <int D>
__device__ __forceinline__ void load_mat(float* dst, const float* src) {
    constexpr int LD = Dim<D>::LD;
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) dst[(e / D) * LD + (e % D)] = src[e];
}

// NM row-major D x D matrices from global memory into padded shared tiles, by a block of NT
// threads: every load is issued before the first store, so one memory latency covers them all
// (a store waits for its load, and a warp issues in order).
// At d = 64 (16 values a thread per matrix) the matrices go one after the other, which keeps
// the registers of the kernels around them.
template <int D, int NM>
__device__ __forceinline__ void load_mats(float* const (&dst)[NM], const float* const (&src)[NM]) {
    constexpr int LD = Dim<D>::LD, PER = D * D / NT;
    static_assert(D * D % NT == 0, "whole matrices per pass");
    constexpr int G = PER * NM <= 24 ? NM : 1;          // matrices per batch of loads
#pragma unroll
    for (int m0 = 0; m0 < NM; m0 += G) {
        float x[G][PER];
#pragma unroll
        for (int m = 0; m < G; ++m)
#pragma unroll
            for (int i = 0; i < PER; ++i) x[m][i] = src[m0 + m][threadIdx.x + i * NT];
#pragma unroll
        for (int m = 0; m < G; ++m)
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = threadIdx.x + i * NT;
                dst[m0 + m][(e / D) * LD + (e % D)] = x[m][i];
            }
    }
}

__device__ __forceinline__ float gpow(float g, int n) {  // gamma^n, n >= 0
    return n == 0 ? 1.f : powf(g, (float)n);
}

// Identity element of each op's combine: zeros, rho = 1.
template <int OP, int D>
__device__ void write_identity(float* out) {
    using S = Sum<OP, D>;
    for (int e = threadIdx.x; e < S::SIZE; e += blockDim.x) out[e] = (decayed_op(OP) && e == S::SCAL) ? 1.f : 0.f;
}

// ---------------------------------------------------------------------------
// Chunk kernel: one block per (chunk, head); writes the chunk's summary.
// Slots NC..NCp-1 (scan padding) receive the identity.
// ---------------------------------------------------------------------------
template <int OP, int D, typename TIn>
__global__ void __launch_bounds__(NT) k_summary(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                const TIn* __restrict__ v, const float* __restrict__ gamma,
                                                int H, int T, int NC, int NCp, float* __restrict__ sums) {
    using S = Sum<OP, D>;
    constexpr int LD = Dim<D>::LD;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    pdl_release();
    float* out = sums + ((size_t)bh * NCp + chunk) * S::SIZE;
    if (chunk >= NC) {
        write_identity<OP, D>(out);
        return;
    }
    extern __shared__ float sm[];
    float* Qs = sm;
    float* Ks = Qs + C * LD;
    float* Vs = Ks + C * LD;
    float* As = Vs + C * LD;      // C x LDC
    float* Ys = As + C * LDC;     // C x LD
    float* Y2 = Ys + C * LD;      // C x LD
    float* us = Y2 + C * LD;      // C
    float* lam = us + C;          // C  (decay weights)
    float* gpw = lam + C;         // C + 1: gamma^j
    const size_t head = (size_t)bh * T * D;
    const int t0 = chunk * C;
    load_rows<D>(Qs, q + head, t0, T);
    load_rows<D>(Ks, k + head, t0, T);
    load_rows<D>(Vs, v + head, t0, T);
    float g = 1.f;
    const int len = min(C, T - t0);      // tokens in this chunk (the last one may be short)
    if (decayed_op(OP)) {
        // gamma^(len - 1 - tau): decayed to the chunk's own last token, so that the summary of
        // a short last chunk is the state after the sequence's last token (the streaming state)
        g = gamma[bh % H];
        for (int j = threadIdx.x; j < C; j += blockDim.x) lam[j] = j < len ? gpow(g, len - 1 - j) : 0.f;
        for (int j = threadIdx.x; j <= C; j += blockDim.x) gpw[j] = gpow(g, j);
    }
    __syncthreads();
    // A* = Q K^T (masked to A = L (.) A* except for the decayed second order, which needs both
    // parts; the decayed AHLA / third order keep At = gamma^(t-j) A_tj)
    if (OP != OP_HLA2U)
        mm<C, C, D>(Tile{Qs, LD}, TileT{Ks, LD}, Zero{}, [&](int r, int c, float x) {
            if (OP == OP_AHLAD || OP == OP_HLA3D) As[r * LDC + c] = c <= r ? gpw[r - c] * x : 0.f;
            else As[r * LDC + c] = (OP == OP_HLA2D || c <= r) ? x : 0.f;
        });
    __syncthreads();

    auto store_mat = [&](int slot) {
        return [=](int r, int c, float x) { out[S::mat(slot) + r * D + c] = x; };
    };

    if (OP == OP_HLA2) {
        mm<D, D, C>(TileT{Ks, LD}, Tile{Ks, LD}, Zero{}, store_mat(0));        // S = K^T K
        mm<D, D, C>(TileT{Qs, LD}, Tile{Vs, LD}, Zero{}, store_mat(1));        // C = Q^T V
        mm<C, D, C>(TileT{As, LDC}, Tile{Vs, LD}, Zero{}, Put{Ys, LD});        // Y = A^T V
        for (int i = threadIdx.x; i < C; i += blockDim.x) {              // u = A^T 1
            float s = 0.f;
            for (int j = 0; j < C; ++j) s += As[j * LDC + i];
            us[i] = s;
        }
        __syncthreads();
        mm<D, D, C>(TileT{Ks, LD}, Tile{Ys, LD}, Zero{}, store_mat(2));        // R = K^T Y
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float sm_ = 0.f, sr = 0.f;
            for (int i = 0; i < C; ++i) {
                sm_ += Qs[i * LD + a];
                sr += Ks[i * LD + a] * us[i];
            }
            out[S::vec(0) + a] = sm_;                                    // m = Q^T 1
            out[S::vec(1) + a] = sr;                                     // r = K^T (A^T 1)
        }
    } else if (OP == OP_HLA2D) {
        // S = K^T diag(lam) K, C = Q^T diag(lam) V, Khat = K^T K
        mm<D, D, C>([&](int r, int c) { return Ks[c * LD + r] * lam[c]; }, Tile{Ks, LD}, Zero{}, store_mat(0));
        mm<D, D, C>([&](int r, int c) { return Qs[c * LD + r] * lam[c]; }, Tile{Vs, LD}, Zero{}, store_mat(1));
        mm<D, D, C>(TileT{Ks, LD}, Tile{Ks, LD}, Zero{}, store_mat(3));
        // Y_G[i] = sum_{j<i} (q_j.k_i) lam_j v_j ;  u_i = sum_{j<i} (q_j.k_i) lam_j
        auto ug = [&](int i, int j) { return j < i ? As[j * LDC + i] * lam[j] : 0.f; };
        mm<C, D, C>(ug, Tile{Vs, LD}, Zero{}, Put{Ys, LD});
        for (int i = threadIdx.x; i < C; i += blockDim.x) {
            float s = 0.f;
            for (int j = 0; j < i; ++j) s += As[j * LDC + i] * lam[j];
            us[i] = s;
        }
        __syncthreads();
        mm<D, D, C>(TileT{Ks, LD}, Tile{Ys, LD}, Zero{}, store_mat(2));        // G = K^T Y_G
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float sm_ = 0.f, sh = 0.f;
            for (int i = 0; i < C; ++i) {
                sm_ += Qs[i * LD + a] * lam[i];
                sh += Ks[i * LD + a] * us[i];
            }
            out[S::vec(0) + a] = sm_;                                    // m
            out[S::vec(1) + a] = sh;                                     // h = K^T u
        }
        if (threadIdx.x == 0) out[S::SCAL] = gpow(g, len);               // rho = gamma^len
    } else if (OP == OP_HLA2U) {
        mm<D, D, C>(TileT{Ks, LD}, Tile{Ks, LD}, Zero{}, store_mat(0));        // S = K^T K
        mm<D, D, C>(TileT{Qs, LD}, Tile{Vs, LD}, Zero{}, store_mat(1));        // C = Q^T V
    } else if (OP == OP_AHLAD) {
        // As = At.  P = K^T Lam V, Dm = K^T Q, Y = At V, E = K^T Lam Y; mK = K^T Lam 1, n = K^T Lam (At 1)
        auto kl = [&](int r, int c) { return Ks[c * LD + r] * lam[c]; };               // (K^T Lam)[r][c]
        mm<D, D, C>(kl, Tile{Vs, LD}, Zero{}, store_mat(0));
        mm<D, D, C>(TileT{Ks, LD}, Tile{Qs, LD}, Zero{}, store_mat(2));
        mm<C, D, C>(Tile{As, LDC}, Tile{Vs, LD}, Zero{}, Put{Ys, LD});
        __syncthreads();
        mm<D, D, C>(kl, Tile{Ys, LD}, Zero{}, store_mat(1));
        for (int i = threadIdx.x; i < C; i += blockDim.x) {
            float s = 0.f;
            for (int j = 0; j <= i; ++j) s += As[i * LDC + j];
            us[i] = s;
        }
        __syncthreads();
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float sm_ = 0.f, sn = 0.f;
            for (int i = 0; i < C; ++i) {
                sm_ += Ks[i * LD + a] * lam[i];
                sn += Ks[i * LD + a] * lam[i] * us[i];
            }
            out[S::vec(0) + a] = sm_;
            out[S::vec(1) + a] = sn;
        }
        if (threadIdx.x == 0) out[S::SCAL] = gpow(g, len);
    } else if (OP == OP_HLA3D) {
        // As = At.  S = K^T Lam K, Q2 = Q^T Gam Q (Gam = gamma^(tau+1)), P = K^T Lam V, Y = At V,
        // X = Q^T Y, Z = K^T (At^T Q), F = K^T (At^T Lam Y); vectors with V -> 1
        auto kl = [&](int r, int c) { return Ks[c * LD + r] * lam[c]; };
        mm<D, D, C>(kl, Tile{Ks, LD}, Zero{}, store_mat(0));
        mm<D, D, C>([&](int r, int c) { return Qs[c * LD + r] * gpw[c + 1]; }, Tile{Qs, LD}, Zero{}, store_mat(1));
        mm<D, D, C>(kl, Tile{Vs, LD}, Zero{}, store_mat(2));
        mm<C, D, C>(Tile{As, LDC}, Tile{Vs, LD}, Zero{}, Put{Ys, LD});
        mm<C, D, C>(TileT{As, LDC}, Tile{Qs, LD}, Zero{}, Put{Y2, LD});
        __syncthreads();
        mm<D, D, C>(TileT{Qs, LD}, Tile{Ys, LD}, Zero{}, store_mat(4));
        mm<D, D, C>(TileT{Ks, LD}, Tile{Y2, LD}, Zero{}, store_mat(5));
        __syncthreads();
        mm<C, D, C>(TileT{As, LDC}, [&](int r, int c) { return lam[r] * Ys[r * LD + c]; }, Zero{}, Put{Y2, LD});
        __syncthreads();
        mm<D, D, C>(TileT{Ks, LD}, Tile{Y2, LD}, Zero{}, store_mat(3));
        for (int i = threadIdx.x; i < C; i += blockDim.x) {              // u = At 1
            float s = 0.f;
            for (int j = 0; j <= i; ++j) s += As[i * LDC + j];
            us[i] = s;
        }
        __syncthreads();
        float* ws_ = Y2;                                                  // w = At^T Lam u (C floats)
        for (int i = threadIdx.x; i < C; i += blockDim.x) {
            float s = 0.f;
            for (int r = i; r < C; ++r) s += As[r * LDC + i] * lam[r] * us[r];
            ws_[i] = s;
        }
        __syncthreads();
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float sm_ = 0.f, sx = 0.f, sf = 0.f;
            for (int i = 0; i < C; ++i) {
                sm_ += Ks[i * LD + a] * lam[i];
                sx += Qs[i * LD + a] * us[i];
                sf += Ks[i * LD + a] * ws_[i];
            }
            out[S::vec(0) + a] = sm_;                                    // mK = K^T Lam 1
            out[S::vec(1) + a] = sx;                                     // X1 = Q^T (At 1)
            out[S::vec(2) + a] = sf;                                     // F1 = K^T (At^T Lam At 1)
        }
        if (threadIdx.x == 0) out[S::SCAL] = gpow(g, len);
    } else if (OP == OP_AHLA) {
        mm<D, D, C>(TileT{Ks, LD}, Tile{Vs, LD}, Zero{}, store_mat(0));        // P = K^T V
        mm<D, D, C>(TileT{Ks, LD}, Tile{Qs, LD}, Zero{}, store_mat(2));        // Dm = K^T Q
        mm<C, D, C>(Tile{As, LDC}, Tile{Vs, LD}, Zero{}, Put{Ys, LD});         // Y = A V
        __syncthreads();
        mm<D, D, C>(TileT{Ks, LD}, Tile{Ys, LD}, Zero{}, store_mat(1));        // E = K^T Y
        for (int i = threadIdx.x; i < C; i += blockDim.x) {              // u = A 1
            float s = 0.f;
            for (int j = 0; j <= i; ++j) s += As[i * LDC + j];
            us[i] = s;
        }
        __syncthreads();
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float sm_ = 0.f, sn = 0.f;
            for (int i = 0; i < C; ++i) {
                sm_ += Ks[i * LD + a];
                sn += Ks[i * LD + a] * us[i];
            }
            out[S::vec(0) + a] = sm_;                                    // mK = K^T 1
            out[S::vec(1) + a] = sn;                                     // n = K^T (A 1)
        }
    } else {  // OP_HLA3
        mm<D, D, C>(TileT{Ks, LD}, Tile{Ks, LD}, Zero{}, store_mat(0));        // S
        mm<D, D, C>(TileT{Qs, LD}, Tile{Qs, LD}, Zero{}, store_mat(1));        // Q2
        mm<D, D, C>(TileT{Ks, LD}, Tile{Vs, LD}, Zero{}, store_mat(2));        // P
        mm<C, D, C>(Tile{As, LDC}, Tile{Vs, LD}, Zero{}, Put{Ys, LD});         // Yl = A V
        mm<C, D, C>(TileT{As, LDC}, Tile{Qs, LD}, Zero{}, Put{Y2, LD});        // A^T Q
        __syncthreads();
        mm<D, D, C>(TileT{Qs, LD}, Tile{Ys, LD}, Zero{}, store_mat(4));        // X = Q^T Yl
        mm<D, D, C>(TileT{Ks, LD}, Tile{Y2, LD}, Zero{}, store_mat(5));        // Z = K^T (A^T Q)
        __syncthreads();
        mm<C, D, C>(TileT{As, LDC}, Tile{Ys, LD}, Zero{}, Put{Y2, LD});        // A^T Yl
        __syncthreads();
        mm<D, D, C>(TileT{Ks, LD}, Tile{Y2, LD}, Zero{}, store_mat(3));        // F = K^T (A^T Yl)
        // the same with V replaced by ones: u = A 1, w = A^T u
        for (int i = threadIdx.x; i < C; i += blockDim.x) {
            float s = 0.f;
            for (int j = 0; j <= i; ++j) s += As[i * LDC + j];
            us[i] = s;
        }
        __syncthreads();
        float* ws_ = lam;                                                 // C floats, unused here
        for (int i = threadIdx.x; i < C; i += blockDim.x) {
            float s = 0.f;
            for (int r = i; r < C; ++r) s += As[r * LDC + i] * us[r];
            ws_[i] = s;
        }
        __syncthreads();
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float sm_ = 0.f, sx = 0.f, sf = 0.f;
            for (int i = 0; i < C; ++i) {
                sm_ += Ks[i * LD + a];
                sx += Qs[i * LD + a] * us[i];
                sf += Ks[i * LD + a] * ws_[i];
            }
            out[S::vec(0) + a] = sm_;                                    // mK = K^T 1
            out[S::vec(1) + a] = sx;                                     // X1 = Q^T (A 1)
            out[S::vec(2) + a] = sf;                                     // F1 = K^T (A^T (A 1))
        }
    }
}

// ---------------------------------------------------------------------------
// Scan kernel: one Blelloch level; one block per (pair, head).
//   up-sweep:   X[R] = X[L] o X[R]
//   down-sweep: X[L], X[R] = X[R], X[R] o X[L]   (root: X[R] read as identity)
// combine(A, B) summarises "A then B".
// ---------------------------------------------------------------------------
template <int OP, int D>
__device__ void combine_into(const float* A, const float* B, float* out, float* tmp) {
    using S = Sum<OP, D>;
    constexpr int DD = D * D;
    auto G = [](const float* p, int slot) { return Tile{p + S::mat(slot), D}; };
    auto add2 = [&](int slot) {
        for (int e = threadIdx.x; e < DD; e += blockDim.x) out[S::mat(slot) + e] = A[S::mat(slot) + e] + B[S::mat(slot) + e];
    };
    auto dst = [&](int slot) {
        return [=](int r, int c, float x) { out[S::mat(slot) + r * D + c] = x; };
    };
    if (OP == OP_HLA2) {
        add2(0);
        add2(1);
        mm<D, D, D>(G(A, 0), G(B, 1),
                    [&](int r, int c) { return A[S::mat(2) + r * D + c] + B[S::mat(2) + r * D + c]; }, dst(2));
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float s = 0.f;
            for (int b = 0; b < D; ++b) s += A[S::mat(0) + a * D + b] * B[S::vec(0) + b];
            out[S::vec(0) + a] = A[S::vec(0) + a] + B[S::vec(0) + a];
            out[S::vec(1) + a] = A[S::vec(1) + a] + B[S::vec(1) + a] + s;
        }
    } else if (OP == OP_HLA2D) {
        const float rb = B[S::SCAL];
        for (int e = threadIdx.x; e < DD; e += blockDim.x) {
            out[S::mat(0) + e] = rb * A[S::mat(0) + e] + B[S::mat(0) + e];
            out[S::mat(1) + e] = rb * A[S::mat(1) + e] + B[S::mat(1) + e];
            out[S::mat(3) + e] = A[S::mat(3) + e] + B[S::mat(3) + e];
        }
        mm<D, D, D>([&](int r, int c) { return rb * B[S::mat(3) + r * D + c]; }, G(A, 1),
                    [&](int r, int c) { return rb * A[S::mat(2) + r * D + c] + B[S::mat(2) + r * D + c]; },
                    dst(2));
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float s = 0.f;
            for (int b = 0; b < D; ++b) s += B[S::mat(3) + a * D + b] * A[S::vec(0) + b];
            out[S::vec(0) + a] = rb * A[S::vec(0) + a] + B[S::vec(0) + a];
            out[S::vec(1) + a] = rb * A[S::vec(1) + a] + B[S::vec(1) + a] + rb * s;
        }
        if (threadIdx.x == 0) out[S::SCAL] = A[S::SCAL] * rb;
    } else if (OP == OP_HLA2U) {
        add2(0);
        add2(1);
    } else if (OP == OP_AHLAD) {
        // P = rb P_A + P_B, E = rb E_A + E_B + rb Dm_B P_A, Dm adds; vectors alike (n gets rb Dm_B mK_A)
        const float rb = B[S::SCAL];
        for (int e = threadIdx.x; e < DD; e += blockDim.x) {
            out[S::mat(0) + e] = rb * A[S::mat(0) + e] + B[S::mat(0) + e];
            out[S::mat(2) + e] = A[S::mat(2) + e] + B[S::mat(2) + e];
        }
        mm<D, D, D>([&](int r, int c) { return rb * B[S::mat(2) + r * D + c]; }, G(A, 0),
                    [&](int r, int c) { return rb * A[S::mat(1) + r * D + c] + B[S::mat(1) + r * D + c]; }, dst(1));
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float s = 0.f;
            for (int b = 0; b < D; ++b) s += B[S::mat(2) + a * D + b] * A[S::vec(0) + b];
            out[S::vec(0) + a] = rb * A[S::vec(0) + a] + B[S::vec(0) + a];
            out[S::vec(1) + a] = rb * A[S::vec(1) + a] + B[S::vec(1) + a] + rb * s;
        }
        if (threadIdx.x == 0) out[S::SCAL] = A[S::SCAL] * rb;
    } else if (OP == OP_HLA3D) {
        // S = rb S_A + S_B, P = rb P_A + P_B, Q2 = Q2_A + ra Q2_B, Z = Z_A + Z_B + S_A Q2_B,
        // X = X_A + X_B + Q2_B P_A, F = rb F_A + F_B + rb (S_A Q2_B P_A + S_A X_B + Z_B P_A)
        const float ra = A[S::SCAL], rb = B[S::SCAL];
        mm<D, D, D>(G(A, 0), G(B, 1), Zero{}, [&](int r, int c, float x) { tmp[r * D + c] = x; });   // S_A Q2_B
        __syncthreads();
        for (int e = threadIdx.x; e < DD; e += blockDim.x) {
            out[S::mat(0) + e] = rb * A[S::mat(0) + e] + B[S::mat(0) + e];
            out[S::mat(1) + e] = A[S::mat(1) + e] + ra * B[S::mat(1) + e];
            out[S::mat(2) + e] = rb * A[S::mat(2) + e] + B[S::mat(2) + e];
            out[S::mat(5) + e] = A[S::mat(5) + e] + B[S::mat(5) + e] + tmp[e];
        }
        mm<D, D, D>(G(B, 1), G(A, 2),
                    [&](int r, int c) { return A[S::mat(4) + r * D + c] + B[S::mat(4) + r * D + c]; }, dst(4));
        auto rbt = [&](const float* p, int slot) {
            return [=](int r, int c) { return rb * p[S::mat(slot) + r * D + c]; };
        };
        mm3<D, D, D, D, D>([&](int r, int c) { return rb * tmp[r * D + c]; }, G(A, 2), rbt(A, 0), G(B, 4), rbt(B, 5),
                           G(A, 2),
                           [&](int r, int c) { return rb * A[S::mat(3) + r * D + c] + B[S::mat(3) + r * D + c]; },
                           dst(3));
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float sx = 0.f, sf = 0.f;
            for (int b = 0; b < D; ++b) {
                const float mk = A[S::vec(0) + b];
                sx += B[S::mat(1) + a * D + b] * mk;
                sf += tmp[a * D + b] * mk + A[S::mat(0) + a * D + b] * B[S::vec(1) + b] + B[S::mat(5) + a * D + b] * mk;
            }
            out[S::vec(0) + a] = rb * A[S::vec(0) + a] + B[S::vec(0) + a];
            out[S::vec(1) + a] = A[S::vec(1) + a] + B[S::vec(1) + a] + sx;
            out[S::vec(2) + a] = rb * A[S::vec(2) + a] + B[S::vec(2) + a] + rb * sf;
        }
        if (threadIdx.x == 0) out[S::SCAL] = ra * rb;
    } else if (OP == OP_AHLA) {
        add2(0);
        add2(2);
        mm<D, D, D>(G(B, 2), G(A, 0),
                    [&](int r, int c) { return A[S::mat(1) + r * D + c] + B[S::mat(1) + r * D + c]; }, dst(1));
        for (int a = threadIdx.x; a < D; a += blockDim.x) {          // n_AB = n_A + n_B + Dm_B mK_A
            float s = 0.f;
            for (int b = 0; b < D; ++b) s += B[S::mat(2) + a * D + b] * A[S::vec(0) + b];
            out[S::vec(0) + a] = A[S::vec(0) + a] + B[S::vec(0) + a];
            out[S::vec(1) + a] = A[S::vec(1) + a] + B[S::vec(1) + a] + s;
        }
    } else {  // OP_HLA3
        // tmp = S_A Q2_B
        mm<D, D, D>(G(A, 0), G(B, 1), Zero{}, [&](int r, int c, float x) { tmp[r * D + c] = x; });
        __syncthreads();
        add2(0);
        add2(1);
        add2(2);
        for (int e = threadIdx.x; e < DD; e += blockDim.x) out[S::mat(5) + e] = A[S::mat(5) + e] + B[S::mat(5) + e] + tmp[e];
        mm<D, D, D>(G(B, 1), G(A, 2),
                    [&](int r, int c) { return A[S::mat(4) + r * D + c] + B[S::mat(4) + r * D + c]; }, dst(4));
        mm3<D, D, D, D, D>(Tile{tmp, D}, G(A, 2), G(A, 0), G(B, 4), G(B, 5), G(A, 2),
                           [&](int r, int c) { return A[S::mat(3) + r * D + c] + B[S::mat(3) + r * D + c]; },
                           dst(3));
        // vectors (P -> mK, X -> X1, F -> F1): X1_AB = X1_A + X1_B + Q2_B mK_A,
        // F1_AB = F1_A + F1_B + (S_A Q2_B) mK_A + S_A X1_B + Z_B mK_A
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            float sx = 0.f, sf = 0.f;
            for (int b = 0; b < D; ++b) {
                const float mk = A[S::vec(0) + b];
                sx += B[S::mat(1) + a * D + b] * mk;
                sf += tmp[a * D + b] * mk + A[S::mat(0) + a * D + b] * B[S::vec(1) + b] + B[S::mat(5) + a * D + b] * mk;
            }
            out[S::vec(0) + a] = A[S::vec(0) + a] + B[S::vec(0) + a];
            out[S::vec(1) + a] = A[S::vec(1) + a] + B[S::vec(1) + a] + sx;
            out[S::vec(2) + a] = A[S::vec(2) + a] + B[S::vec(2) + a] + sf;
        }
    }
}

template <int OP, int D>
__global__ void __launch_bounds__(NT) k_scan_level(float* sums, int NCp, int step, int down, int root) {
    using S = Sum<OP, D>;
    pdl_release();
    pdl_wait();
    extern __shared__ float sm[];
    float* As = sm;
    float* Bs = As + S::SIZE;
    float* tmp = Bs + S::SIZE;
    const int pair = blockIdx.x, bh = blockIdx.y;
    const int L = pair * 2 * step + step - 1, R = pair * 2 * step + 2 * step - 1;
    float* base = sums + (size_t)bh * NCp * S::SIZE;
    float* XL = base + (size_t)L * S::SIZE;
    float* XR = base + (size_t)R * S::SIZE;
    if (!down) {
        for (int e = threadIdx.x; e < S::SIZE; e += blockDim.x) {
            As[e] = XL[e];
            Bs[e] = XR[e];
        }
        __syncthreads();
        combine_into<OP, D>(As, Bs, XR, tmp);
    } else {
        // A = parent prefix (X[R], identity at the root), B = left subtree total (X[L])
        if (root) write_identity<OP, D>(As);
        else
            for (int e = threadIdx.x; e < S::SIZE; e += blockDim.x) As[e] = XR[e];
        for (int e = threadIdx.x; e < S::SIZE; e += blockDim.x) Bs[e] = XL[e];
        __syncthreads();
        for (int e = threadIdx.x; e < S::SIZE; e += blockDim.x) XL[e] = As[e];
        combine_into<OP, D>(As, Bs, XR, tmp);
    }
}

template <int OP, int D>
__global__ void k_identity(float* sums, int NCp) {
    using S = Sum<OP, D>;
    pdl_release();
    pdl_wait();
    write_identity<OP, D>(sums + (size_t)blockIdx.x * NCp * S::SIZE);
}

// ---------------------------------------------------------------------------
// Exclusive scan as a left-to-right fold, one block per head: slot l becomes the combine of
// slots 0 .. l-1 (the same prefixes as the Blelloch tree, combined in sequence order).  Each
// summary is read once and each prefix written once, in one launch; the next summary is
// loaded into registers while the current combine runs.  Used when three summaries and the
// combine's scratch fit in shared memory, except for the third order: its combine is five
// d x d x d products, and with few heads the serial fold measured slower than the tree
// (2 x 8 heads, 64 chunks, d = 32: 0.426 ms against 0.166 ms).  Otherwise the per-level
// tree below serves.
// ---------------------------------------------------------------------------
template <int OP, int D>
constexpr size_t fold_smem() { return sizeof(float) * (3 * (size_t)Sum<OP, D>::SIZE + (size_t)D * D); }
template <int OP, int D>
constexpr bool fold_fits() { return OP != OP_HLA3 && OP != OP_HLA3D && fold_smem<OP, D>() <= 227 * 1024; }

template <int OP, int D>
__global__ void __launch_bounds__(NT) k_scan_fold(float* sums, int NC, int NCp) {
    using S = Sum<OP, D>;
    constexpr int N4 = S::SIZE / 4, PER = (N4 + NT - 1) / NT;
    pdl_release();
    pdl_wait();
    extern __shared__ float4 sm4[];
    float* acc = reinterpret_cast<float*>(sm4);          // prefix of slots 0 .. l-1
    float* other = acc + S::SIZE;
    float* cur = other + S::SIZE;                          // summary l
    float* tmp = cur + S::SIZE;                            // D x D scratch of the combine
    float4* base4 = reinterpret_cast<float4*>(sums + (size_t)blockIdx.x * NCp * S::SIZE);
    write_identity<OP, D>(acc);
    float4 nx[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = threadIdx.x + i * NT;
        if (e < N4) nx[i] = base4[e];
    }
    for (int l = 0; l < NC; ++l) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = threadIdx.x + i * NT;
            if (e < N4) reinterpret_cast<float4*>(cur)[e] = nx[i];
        }
        __syncthreads();                                   // cur = summary l, acc = prefix l
        float4* slot = base4 + (size_t)l * N4;             // read already: becomes the prefix
        for (int e = threadIdx.x; e < N4; e += NT) slot[e] = reinterpret_cast<const float4*>(acc)[e];
        if (l + 1 < NC) {
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = threadIdx.x + i * NT;
                if (e < N4) nx[i] = slot[N4 + e];
            }
        }
        combine_into<OP, D>(acc, cur, other, tmp);         // prefix l+1 = prefix l o summary l
        __syncthreads();
        float* t = acc;
        acc = other;
        other = t;
    }
}

// ---------------------------------------------------------------------------
// Third order: the exclusive prefix in factored form.  The combine's cross terms depend on the
// earlier operand only through S, P and m^K, which add plainly, so unrolled over the chunks
//     S0(n) = sum_{l<n} S_l,   P0(n) = sum_{l<n} P_l,   mK0(n) = sum_{l<n} mK_l,
//     F0(n) = sum_{l<n} (F_l + S0(l) Q2_l P0(l) + S0(l) X_l + Z_l P0(l)),
//     F1_0(n) = sum_{l<n} (F1_l + S0(l) Q2_l mK0(l) + S0(l) X1_l + Z_l mK0(l)),
// which are all the output kernel reads.  Three launches, each parallel over chunks or elements:
// plain exclusive sums of S, P, mK in place; the corrected F_l, F1_l per chunk; their exclusive
// sums in place.  The result equals the Blelloch tree's up to the order of fp32 additions.
// With decay (OP_HLA3D) the combine scales the earlier operand's S, P, mK, F, F1 by the later
// one's rho and its cross terms by rho too, while Q2, X, Z enter only as the chunk's own; so
// the sums become decayed running sums (run = rho_l run + y_l) and the corrected terms
// F_l + rho_l (...), with the same three launches.
// ---------------------------------------------------------------------------
template <int OP, int D>
__global__ void __launch_bounds__(NT) k_hla3_prefix_plain(float* sums, int NC, int NCp, int which) {
    using S = Sum<OP, D>;
    pdl_release();
    pdl_wait();
    const int e = blockIdx.x * NT + threadIdx.x;
    int off;
    if (which == 0) {                        // S, P and mK
        if (e >= 2 * D * D + D) return;
        off = e < D * D ? S::mat(0) + e : e < 2 * D * D ? S::mat(2) + (e - D * D) : S::vec(0) + (e - 2 * D * D);
    } else {                                 // the corrected F and F1
        if (e >= D * D + D) return;
        off = e < D * D ? S::mat(3) + e : S::vec(2) + (e - D * D);
    }
    float* p = sums + (size_t)blockIdx.y * NCp * S::SIZE + off;
    const float* rho = sums + (size_t)blockIdx.y * NCp * S::SIZE + S::SCAL;
    float run = 0.f;
    constexpr int B = 32;                    // B loads in flight, then the dependent adds
    for (int l0 = 0; l0 < NC; l0 += B) {
        float y[B], r[B];
#pragma unroll
        for (int i = 0; i < B; ++i)
            if (l0 + i < NC) {
                y[i] = p[(size_t)(l0 + i) * S::SIZE];
                r[i] = OP == OP_HLA3D ? rho[(size_t)(l0 + i) * S::SIZE] : 1.f;
            }
#pragma unroll
        for (int i = 0; i < B; ++i)
            if (l0 + i < NC) {
                p[(size_t)(l0 + i) * S::SIZE] = run;
                run = OP == OP_HLA3D ? fmaf(r[i], run, y[i]) : run + y[i];
            }
    }
}

template <int OP, int D>
__global__ void __launch_bounds__(NT) k_hla3_prefix_cross(float* sums, int NCp) {
    using S = Sum<OP, D>;
    pdl_release();
    pdl_wait();
    constexpr int LD = Dim<D>::LD;
    extern __shared__ float smx[];
    float* S0 = smx;
    float* P0 = S0 + D * LD;
    float* SQ = P0 + D * LD;
    float* Q2 = SQ + D * LD;
    float* Xs = Q2 + D * LD;
    float* Zs = Xs + D * LD;
    float* mk = Zs + D * LD;
    float* x1 = mk + D;
    float* slot = sums + ((size_t)blockIdx.y * NCp + blockIdx.x) * S::SIZE;
    // S0(l) and P0(l) (the plain prefixes, in place), the chunk's Q2, X, Z
    load_mats<D, 5>({S0, Q2, P0, Xs, Zs}, {slot + S::mat(0), slot + S::mat(1), slot + S::mat(2), slot + S::mat(4),
                                          slot + S::mat(5)});
    for (int a = threadIdx.x; a < D; a += blockDim.x) {
        mk[a] = slot[S::vec(0) + a];
        x1[a] = slot[S::vec(1) + a];
    }
    __syncthreads();
    constexpr int R = D * D >= 16 * NT ? 4 : 2;       // 2 x 2 per thread at d = 32: every thread works
    mm3<D, D, D, 0, 0, R>(Tile{S0, LD}, Tile{Q2, LD}, Tile{S0, LD}, Tile{Q2, LD}, Tile{S0, LD}, Tile{Q2, LD},
                          Zero{}, Put{SQ, LD});                                  // S0 Q2
    __syncthreads();
    float* F = slot + S::mat(3);
    const float rho = OP == OP_HLA3D ? slot[S::SCAL] : 1.f;
    // F += rho ((S0 Q2) P0 + S0 X + Z P0)
    mm3<D, D, D, D, D, R>(Tile{SQ, LD}, Tile{P0, LD}, Tile{S0, LD}, Tile{Xs, LD}, Tile{Zs, LD}, Tile{P0, LD}, Zero{},
                          [&](int r, int c, float x) { F[r * D + c] = fmaf(rho, x, F[r * D + c]); });
    for (int a = threadIdx.x; a < D; a += blockDim.x) {
        float s = 0.f;
        for (int b = 0; b < D; ++b) s += SQ[a * LD + b] * mk[b] + S0[a * LD + b] * x1[b] + Zs[a * LD + b] * mk[b];
        slot[S::vec(2) + a] = fmaf(rho, s, slot[S::vec(2) + a]);
    }
}

template <int OP, int D>
static cudaError_t hla3_factored_prefix(float* sums, int NC, int NCp, int BH, cudaStream_t st) {
    auto kp = k_hla3_prefix_plain<OP, D>;
    cudaError_t e = launch_dep(kp, dim3((2 * D * D + D + NT - 1) / NT, BH), dim3(NT), 0, st, sums, NC, NCp, 0);
    if (e != cudaSuccess) return e;
    const int smem = (int)(sizeof(float) * (6 * D * Dim<D>::LD + 2 * D));
    auto kc = k_hla3_prefix_cross<OP, D>;
    if ((e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    if ((e = launch_dep(kc, dim3(NC, BH), dim3(NT), (size_t)smem, st, sums, NCp)) != cudaSuccess) return e;
    return launch_dep(kp, dim3((D * D + D + NT - 1) / NT, BH), dim3(NT), 0, st, sums, NC, NCp, 1);
}

// ---------------------------------------------------------------------------
// Output kernel: one block per (chunk, head); applies the chunk's prefix.
// ---------------------------------------------------------------------------
template <int OP, bool NORM, int D, typename TIn>
__global__ void __launch_bounds__(NT) k_output(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                               const TIn* __restrict__ v, const float* __restrict__ gamma,
                                               float eps, int H, int T, int NCp, const float* sums,
                                               float* __restrict__ o) {
    using S = Sum<OP, D>;
    constexpr int LD = Dim<D>::LD;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    const float* pre = sums + ((size_t)bh * NCp + chunk) * S::SIZE;
    extern __shared__ float sm[];
    float* Qs = sm;
    float* Ks = Qs + C * LD;
    float* Vs = Ks + C * LD;
    float* As = Vs + C * LD;      // C x LDC
    float* Ws = As + C * LDC;     // C x LDC
    float* Ps = Ws + C * LDC;     // C x LD
    float* Ys = Ps + C * LD;      // C x LD
    float* M0 = Ys + C * LD;      // D x LD  (prefix matrices)
    float* M1 = M0 + D * LD;
    float* M2 = M1 + D * LD;
    float* vec = M2 + D * LD;     // 2 D
    float* den = vec + 2 * D;     // C
    float* gp = den + C;          // C + 1
    const size_t head = (size_t)bh * T * D;
    const int t0 = chunk * C;
    load_rows<D>(Qs, q + head, t0, T);
    load_rows<D>(Ks, k + head, t0, T);
    load_rows<D>(Vs, v + head, t0, T);
    pdl_wait();                              // the prefixes below come from the scan
    float g = 1.f;
    if (OP == OP_HLA2) {
        load_mats<D, 2>({M0, M1}, {pre + S::mat(0), pre + S::mat(2)});       // S0, R0
        for (int a = threadIdx.x; a < D; a += blockDim.x) vec[a] = pre[S::vec(1) + a];  // r0
    } else if (OP == OP_HLA2D) {
        load_mats<D, 3>({M0, M1, M2}, {pre + S::mat(0), pre + S::mat(1), pre + S::mat(2)});   // S0, C0, G0
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            vec[a] = pre[S::vec(0) + a];      // m0
            vec[D + a] = pre[S::vec(1) + a];  // h0
        }
        g = gamma[bh % H];
        for (int j = threadIdx.x; j <= C; j += blockDim.x) gp[j] = gpow(g, j);
    } else if (OP == OP_HLA2U) {
        load_mats<D, 2>({M0, M1}, {pre + S::mat(0), pre + S::mat(1)});       // S0, C0
    } else if (OP == OP_AHLA || OP == OP_AHLAD) {
        load_mats<D, 2>({M0, M1}, {pre + S::mat(0), pre + S::mat(1)});       // P0, E0
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            vec[a] = pre[S::vec(0) + a];      // mK0
            vec[D + a] = pre[S::vec(1) + a];  // n0
        }
    } else {
        load_mats<D, 3>({M0, M1, M2}, {pre + S::mat(0), pre + S::mat(2), pre + S::mat(3)});   // S0, P0, F0
        for (int a = threadIdx.x; a < D; a += blockDim.x) {
            vec[a] = pre[S::vec(0) + a];      // mK0
            vec[D + a] = pre[S::vec(2) + a];  // F1_0
        }
    }
    if (OP == OP_AHLAD || OP == OP_HLA3D) {
        g = gamma[bh % H];
        for (int j = threadIdx.x; j <= C; j += blockDim.x) gp[j] = gpow(g, j);
    }
    __syncthreads();
    mm<C, C, D>(Tile{Qs, LD}, TileT{Ks, LD}, Zero{}, [&](int r, int c, float x) {
        As[r * LDC + c] = (OP == OP_HLA2D || OP == OP_HLA2U || c <= r) ? x : 0.f;
    });
    if (OP == OP_HLA2 || OP == OP_HLA3 || OP == OP_HLA3D || OP == OP_HLA2U)
        mm<C, D, D>(Tile{Qs, LD}, Tile{M0, LD}, Zero{}, Put{Ps, LD});                      // P = Q S0
    if (OP == OP_HLA2U)
        mm<D, D, D>(Tile{M0, LD}, Tile{M1, LD}, Zero{}, Put{M2, LD});                      // S0 C0
    if (OP == OP_HLA2D)
        mm<C, D, D>(Tile{Qs, LD}, Tile{M0, LD}, Zero{}, [&](int r, int c, float x) {         // P~ = Gamma Q S0
            Ps[r * LD + c] = gp[r + 1] * x;
        });
    __syncthreads();

    const size_t obase = ((size_t)bh * T + t0) * D;
    auto emit = [&](int r, int c, float x) {
        if (t0 + r < T) o[obase + (size_t)r * D + c] = NORM ? x / (den[r] + eps) : x;
    };

    if (OP == OP_HLA2) {
        // W = L (.) (P Q^T + A A^T)
        mm2<C, C, D, C>(Tile{Ps, LD}, TileT{Qs, LD}, Tile{As, LDC}, TileT{As, LDC}, Zero{},
                        [&](int r, int c, float x) { Ws[r * LDC + c] = c <= r ? x : 0.f; });
        __syncthreads();
        if (NORM) {
            for (int r = threadIdx.x; r < C; r += blockDim.x) {
                float s = 0.f;
                for (int a = 0; a < D; ++a) s += Qs[r * LD + a] * vec[a];
                for (int j = 0; j <= r; ++j) s += Ws[r * LDC + j];
                den[r] = s;
            }
            __syncthreads();
        }
        mm2<C, D, D, C>(Tile{Qs, LD}, Tile{M1, LD}, Tile{Ws, LDC}, Tile{Vs, LD}, Zero{}, emit);   // O = Q R0 + W V
    } else if (OP == OP_HLA2D) {
        // W_tj = [j<=t] g^(t-j) ( g^(t+1) (P Q^T)_tj + sum_{i<=t} A*_ti A*_ji (g^(t-i) - [i>j]) )
        //      = [j<=t] g^(t-j) ( (P~ Q^T) + (A~ A*^T) - (A U^T) )_tj
        auto At = [&](int r, int c) { return c <= r ? gp[r - c] * As[r * LDC + c] : 0.f; };   // A~
        auto Am = [&](int r, int c) { return c <= r ? -As[r * LDC + c] : 0.f; };            // -A
        auto Ut = [&](int kk, int n) { return kk > n ? As[n * LDC + kk] : 0.f; };           // U^T
        mm3<C, C, D, C, C>(Tile{Ps, LD}, TileT{Qs, LD}, At, TileT{As, LDC}, Am, Ut, Zero{},
                           [&](int r, int c, float x) { Ws[r * LDC + c] = c <= r ? gp[r - c] * x : 0.f; });
        // Z' = P~ + (A~ - A) K
        mm<C, D, C>([&](int r, int c) { return c <= r ? (gp[r - c] - 1.f) * As[r * LDC + c] : 0.f; },
                    Tile{Ks, LD}, Tile{Ps, LD}, Put{Ys, LD});
        __syncthreads();
        if (NORM) {
            for (int r = threadIdx.x; r < C; r += blockDim.x) {
                float s = 0.f, zm = 0.f, qh = 0.f;
                for (int j = 0; j <= r; ++j) s += Ws[r * LDC + j];
                for (int a = 0; a < D; ++a) {
                    zm += Ys[r * LD + a] * vec[a];
                    qh += Qs[r * LD + a] * vec[D + a];
                }
                den[r] = s + gp[r + 1] * (zm - qh);
            }
            __syncthreads();
        }
        // O = W V + Gamma Z' C0 - Gamma Q G0
        mm3<C, D, C, D, D>(Tile{Ws, LDC}, Tile{Vs, LD},
                           [&](int r, int c) { return gp[r + 1] * Ys[r * LD + c]; }, Tile{M1, LD},
                           [&](int r, int c) { return -gp[r + 1] * Qs[r * LD + c]; }, Tile{M2, LD}, Zero{}, emit);
    } else if (OP == OP_HLA2U) {
        // As holds A* = Q K^T unmasked; A = L (.) A*.
        auto Am = [&](int r, int c) { return c <= r ? As[r * LDC + c] : 0.f; };
        // W = L (.) (P Q^T + A A*^T): the pair weight summed over every key up to the query's token
        mm2<C, C, D, C>(Tile{Ps, LD}, TileT{Qs, LD}, Am, TileT{As, LDC}, Zero{},
                        [&](int r, int c, float x) { Ws[r * LDC + c] = c <= r ? x : 0.f; });
        mm<C, D, C>(Am, Tile{Ks, LD}, Zero{}, Put{Ys, LD});                                    // Y = A K
        __syncthreads();
        // O = Q (S0 C0) + W V + Y C0
        mm3<C, D, D, C, D>(Tile{Qs, LD}, Tile{M2, LD}, Tile{Ws, LDC}, Tile{Vs, LD}, Tile{Ys, LD}, Tile{M1, LD},
                           Zero{}, emit);
    } else if (OP == OP_AHLA) {
        mm2<C, D, D, C>(Tile{Qs, LD}, Tile{M0, LD}, Tile{As, LDC}, Tile{Vs, LD}, Zero{}, Put{Ys, LD});   // Y = Q P0 + A V
        __syncthreads();
        if (NORM) {     // y1 = Q mK0 + A 1 (in gp), den = Q n0 + A y1
            for (int r = threadIdx.x; r < C; r += blockDim.x) {
                float s = 0.f;
                for (int a = 0; a < D; ++a) s += Qs[r * LD + a] * vec[a];
                for (int j = 0; j <= r; ++j) s += As[r * LDC + j];
                gp[r] = s;
            }
            __syncthreads();
            for (int r = threadIdx.x; r < C; r += blockDim.x) {
                float s = 0.f;
                for (int a = 0; a < D; ++a) s += Qs[r * LD + a] * vec[D + a];
                for (int j = 0; j <= r; ++j) s += As[r * LDC + j] * gp[j];
                den[r] = s;
            }
            __syncthreads();
        }
        mm2<C, D, D, C>(Tile{Qs, LD}, Tile{M1, LD}, Tile{As, LDC}, Tile{Ys, LD}, Zero{}, emit);          // O = Q E0 + A Y
    } else if (OP == OP_AHLAD || OP == OP_HLA3D) {
        // Gam = diag(gamma^(tau+1)) (the carried state decays by one step per token of the chunk
        // up to and including tau), At_tj = gamma^(t-j) A_tj:
        //   AHLA:  Y = Gam Q P0 + At V,  O = Gam Q E0 + At Y
        //   third: Y = Gam Q P0 + At V,  W = L (.) (Gam P Q^T + At A^T),  O = Gam Q F0 + W Y
        auto At = [&](int r, int c) { return c <= r ? gp[r - c] * As[r * LDC + c] : 0.f; };
        auto GQ = [&](int r, int c) { return gp[r + 1] * Qs[r * LD + c]; };
        const float* Pm = OP == OP_AHLAD ? M0 : M1;                                            // P0
        const float* Em = OP == OP_AHLAD ? M1 : M2;                                            // E0 / F0
        mm2<C, D, D, C>(GQ, Tile{Pm, LD}, At, Tile{Vs, LD}, Zero{}, Put{Ys, LD});
        if (OP == OP_HLA3D)
            mm2<C, C, D, C>([&](int r, int c) { return gp[r + 1] * Ps[r * LD + c]; }, TileT{Qs, LD}, At,
                            TileT{As, LDC}, Zero{}, [&](int r, int c, float x) { Ws[r * LDC + c] = c <= r ? x : 0.f; });
        __syncthreads();
        if (NORM) {     // y1 = Gam Q mK0 + At 1 (in Ps column 0), den = Gam Q n0 + At y1 (F1_0, W y1)
            for (int r = threadIdx.x; r < C; r += blockDim.x) {
                float s = 0.f;
                for (int a = 0; a < D; ++a) s += Qs[r * LD + a] * vec[a];
                s *= gp[r + 1];
                for (int j = 0; j <= r; ++j) s += gp[r - j] * As[r * LDC + j];
                den[r] = s;                                  // y1, for now
            }
            __syncthreads();
            float* y1 = Ps;                                  // P is not read again
            for (int r = threadIdx.x; r < C; r += blockDim.x) y1[r * LD] = den[r];
            __syncthreads();
            for (int r = threadIdx.x; r < C; r += blockDim.x) {
                float s = 0.f;
                for (int a = 0; a < D; ++a) s += Qs[r * LD + a] * vec[D + a];
                s *= gp[r + 1];
                for (int j = 0; j <= r; ++j)
                    s += (OP == OP_AHLAD ? gp[r - j] * As[r * LDC + j] : Ws[r * LDC + j]) * y1[j * LD];
                den[r] = s;
            }
            __syncthreads();
        }
        if (OP == OP_AHLAD) mm2<C, D, D, C>(GQ, Tile{Em, LD}, At, Tile{Ys, LD}, Zero{}, emit);
        else mm2<C, D, D, C>(GQ, Tile{Em, LD}, Tile{Ws, LDC}, Tile{Ys, LD}, Zero{}, emit);
    } else {  // OP_HLA3
        mm2<C, C, D, C>(Tile{Ps, LD}, TileT{Qs, LD}, Tile{As, LDC}, TileT{As, LDC}, Zero{},
                        [&](int r, int c, float x) { Ws[r * LDC + c] = c <= r ? x : 0.f; });
        mm2<C, D, D, C>(Tile{Qs, LD}, Tile{M1, LD}, Tile{As, LDC}, Tile{Vs, LD}, Zero{}, Put{Ys, LD});   // Y = Q P0 + A V
        __syncthreads();
        if (NORM) {     // y1 = Q mK0 + A 1 (in gp), den = Q F1_0 + W y1
            for (int r = threadIdx.x; r < C; r += blockDim.x) {
                float s = 0.f;
                for (int a = 0; a < D; ++a) s += Qs[r * LD + a] * vec[a];
                for (int j = 0; j <= r; ++j) s += As[r * LDC + j];
                gp[r] = s;
            }
            __syncthreads();
            for (int r = threadIdx.x; r < C; r += blockDim.x) {
                float s = 0.f;
                for (int a = 0; a < D; ++a) s += Qs[r * LD + a] * vec[D + a];
                for (int j = 0; j <= r; ++j) s += Ws[r * LDC + j] * gp[j];
                den[r] = s;
            }
            __syncthreads();
        }
        mm2<C, D, D, C>(Tile{Qs, LD}, Tile{M2, LD}, Tile{Ws, LDC}, Tile{Ys, LD}, Zero{}, emit);          // O = Q F0 + W Y
    }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
static int next_pow2(int n) {
    int p = 1;
    while (p < n) p *= 2;
    return p;
}

template <int D>
static size_t summary_smem() {
    constexpr int LD = Dim<D>::LD;
    return sizeof(float) * (size_t)(3 * C * LD + C * LDC + 2 * C * LD + 3 * C + 1);
}
template <int D>
static size_t output_smem() {
    constexpr int LD = Dim<D>::LD;
    return sizeof(float) * (size_t)(3 * C * LD + 2 * C * LDC + 2 * C * LD + 3 * D * LD + 2 * D + 2 * C + 1);
}
template <int OP, int D>
static size_t scan_smem() {
    return sizeof(float) * (size_t)(2 * Sum<OP, D>::SIZE + D * D);
}


size_t workspace_floats(int op, int d, int BH, int T) {
    const int NC = (T + C - 1) / C;
    return (size_t)BH * next_pow2(NC) * summary_floats(op, d);
}

// Blelloch exclusive scan over NCp (a power of two) summaries per head, in place:
// log2(NCp) up-sweep launches, then log2(NCp) down-sweep launches (the first one
// reads the root as the identity).  One block per (pair, head) per level.
template <int OP, int D>
static cudaError_t scan_levels(float* sums, int NCp, int BH, cudaStream_t st) {
    auto kl = k_scan_level<OP, D>;
    const size_t s2 = scan_smem<OP, D>();
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kl, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2)) != cudaSuccess) return e;
    if (NCp == 1) return launch_dep(k_identity<OP, D>, dim3(BH), dim3(NT), 0, st, sums, NCp);
    for (int step = 1; step < NCp; step *= 2)
        if ((e = launch_dep(kl, dim3(NCp / (2 * step), BH), dim3(NT), s2, st, sums, NCp, step, 0, 0)) != cudaSuccess)
            return e;
    for (int step = NCp / 2; step >= 1; step /= 2)
        if ((e = launch_dep(kl, dim3(NCp / (2 * step), BH), dim3(NT), s2, st, sums, NCp, step, 1,
                            step == NCp / 2 ? 1 : 0)) != cudaSuccess)
            return e;
    return cudaSuccess;
}

cudaError_t scan(int op, int d, float* sums, int NCp, int BH, cudaStream_t st) {
    switch (op) {
    case OP_HLA2: return d == 32 ? scan_levels<OP_HLA2, 32>(sums, NCp, BH, st) : scan_levels<OP_HLA2, 64>(sums, NCp, BH, st);
    case OP_HLA2D: return d == 32 ? scan_levels<OP_HLA2D, 32>(sums, NCp, BH, st) : scan_levels<OP_HLA2D, 64>(sums, NCp, BH, st);
    case OP_AHLA: return d == 32 ? scan_levels<OP_AHLA, 32>(sums, NCp, BH, st) : scan_levels<OP_AHLA, 64>(sums, NCp, BH, st);
    case OP_HLA3: return d == 32 ? scan_levels<OP_HLA3, 32>(sums, NCp, BH, st) : scan_levels<OP_HLA3, 64>(sums, NCp, BH, st);
    case OP_HLA2U: return d == 32 ? scan_levels<OP_HLA2U, 32>(sums, NCp, BH, st) : scan_levels<OP_HLA2U, 64>(sums, NCp, BH, st);
    case OP_AHLAD: return d == 32 ? scan_levels<OP_AHLAD, 32>(sums, NCp, BH, st) : scan_levels<OP_AHLAD, 64>(sums, NCp, BH, st);
    case OP_HLA3D: return d == 32 ? scan_levels<OP_HLA3D, 32>(sums, NCp, BH, st) : scan_levels<OP_HLA3D, 64>(sums, NCp, BH, st);
    }
    return cudaErrorInvalidValue;
}

int scan_launches(int NCp) {
    int levels = 0;
    for (int p = 1; p < NCp; p *= 2) ++levels;
    return NCp == 1 ? 1 : 2 * levels;
}

// The plain third order with fp32 inputs and d = 32 takes the tcgen05 summary and output kernels.
template <int OP, bool NORM, int D, typename TIn>
constexpr bool tc_third_order() {
    return OP == OP_HLA3 && !NORM && D == 32 && std::is_same<TIn, float>::value;
}
// So does the plain second order with fp32 inputs at d = 32, up to tc::hla2f_max_chunks()
// 128-token chunks per head (its output CTAs fold the summaries themselves).
template <int OP, bool NORM, int D, typename TIn>
constexpr bool tc_second_order_f32() {
    return OP == OP_HLA2 && !NORM && D == 32 && std::is_same<TIn, float>::value;
}
static bool tc_second_order_f32_fits(int T) { return (T + 127) / 128 <= tc::hla2f_max_chunks(); }

template <int OP, bool NORM, int D, typename TIn>
static cudaError_t run(const void* q, const void* k, const void* v, const float* gamma, float eps, float* o,
                       int BH, int H, int T, float* sums, int* status, cudaStream_t st, cudaEvent_t* ev,
                       bool allow_tc) {
    if (allow_tc && tc_second_order_f32<OP, NORM, D, TIn>() && tc_second_order_f32_fits(T))
        return tc::hla2f_forward((const float*)q, (const float*)k, (const float*)v, sums, Sum<OP, D>::SIZE, o, BH, T,
                                 status, st, ev);
    if (allow_tc && tc_third_order<OP, NORM, D, TIn>()) {
        // the plain third order with fp32 inputs at d = 32: summaries and output on the tensor
        // cores over 128-token chunks, the factored prefix between them on the CUDA cores
        const int NC2 = (T + 127) / 128;
        cudaError_t e;
        if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
        if ((e = tc::hla3_summaries((const float*)q, (const float*)k, (const float*)v, sums, NC2, Sum<OP, D>::SIZE, BH,
                                    T, status, st)) != cudaSuccess)
            return e;
        if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
        if ((e = hla3_factored_prefix<OP, D>(sums, NC2, NC2, BH, st)) != cudaSuccess) return e;
        if (ev && (e = cudaEventRecord(ev[2], st)) != cudaSuccess) return e;
        if ((e = tc::hla3_output((const float*)q, (const float*)k, (const float*)v, sums, NC2, Sum<OP, D>::SIZE, o, BH,
                                 T, status, st)) != cudaSuccess)
            return e;
        if (ev && (e = cudaEventRecord(ev[3], st)) != cudaSuccess) return e;
        return cudaSuccess;
    }
    const int NC = (T + C - 1) / C;
    const int NCp = next_pow2(NC);
    auto ks = k_summary<OP, D, TIn>;
    auto ko = k_output<OP, NORM, D, TIn>;
    const size_t s1 = summary_smem<D>(), s3 = output_smem<D>();
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ko, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    ks<<<dim3(NCp, BH), NT, s1, st>>>((const TIn*)q, (const TIn*)k, (const TIn*)v, gamma, H, T, NC, NCp, sums);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    if (OP == OP_HLA3 || OP == OP_HLA3D) {
        if ((e = hla3_factored_prefix<OP, D>(sums, NC, NCp, BH, st)) != cudaSuccess) return e;
    } else if (fold_fits<OP, D>()) {
        auto kf = k_scan_fold<OP, D>;
        if ((e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fold_smem<OP, D>())) !=
            cudaSuccess)
            return e;
        if ((e = launch_dep(kf, dim3(BH), dim3(NT), fold_smem<OP, D>(), st, sums, NC, NCp)) != cudaSuccess) return e;
    } else if ((e = scan_levels<OP, D>(sums, NCp, BH, st)) != cudaSuccess) {
        return e;
    }
    if (ev && (e = cudaEventRecord(ev[2], st)) != cudaSuccess) return e;
    if ((e = launch_dep(ko, dim3(NC, BH), dim3(NT), s3, st, (const TIn*)q, (const TIn*)k, (const TIn*)v, gamma, eps, H,
                        T, NCp, (const float*)sums, o)) != cudaSuccess)
        return e;
    if (ev && (e = cudaEventRecord(ev[3], st)) != cudaSuccess) return e;
    return cudaSuccess;
}

template <typename TIn, int D>
static cudaError_t dispatch_op(int op, bool norm, const void* q, const void* k, const void* v, const float* gamma,
                               float eps, float* o, int BH, int H, int T, float* sums, int* status, cudaStream_t st,
                               cudaEvent_t* ev, bool allow_tc) {
    switch (op) {
    case OP_HLA2:
        return norm ? run<OP_HLA2, true, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc)
                    : run<OP_HLA2, false, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
    case OP_HLA2D:
        return norm ? run<OP_HLA2D, true, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc)
                    : run<OP_HLA2D, false, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
    case OP_AHLA:
        return norm ? run<OP_AHLA, true, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc)
                    : run<OP_AHLA, false, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
    case OP_HLA3:
        return norm ? run<OP_HLA3, true, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc)
                    : run<OP_HLA3, false, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
    case OP_HLA2U: return run<OP_HLA2U, false, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
    case OP_AHLAD:
        return norm ? run<OP_AHLAD, true, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc)
                    : run<OP_AHLAD, false, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
    case OP_HLA3D:
        return norm ? run<OP_HLA3D, true, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc)
                    : run<OP_HLA3D, false, D, TIn>(q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
    }
    return cudaErrorInvalidValue;
}

cudaError_t forward(int op, bool norm, bool bf16, int d, const void* q, const void* k, const void* v,
                    const float* gamma, float eps, float* o, int BH, int H, int T, float* sums, int* status,
                    cudaStream_t st, cudaEvent_t* ev, bool allow_tc) {
    if (bf16) {
        if (d == 32)
            return dispatch_op<__nv_bfloat16, 32>(op, norm, q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev,
                                                  allow_tc);
        return dispatch_op<__nv_bfloat16, 64>(op, norm, q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev,
                                              allow_tc);
    }
    if (d == 32)
        return dispatch_op<float, 32>(op, norm, q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
    return dispatch_op<float, 64>(op, norm, q, k, v, gamma, eps, o, BH, H, T, sums, status, st, ev, allow_tc);
}

static bool uses_fold(int op, int d) {
    switch (op) {
    case OP_HLA2: return d == 32 ? fold_fits<OP_HLA2, 32>() : fold_fits<OP_HLA2, 64>();
    case OP_HLA2D: return d == 32 ? fold_fits<OP_HLA2D, 32>() : fold_fits<OP_HLA2D, 64>();
    case OP_AHLA: return d == 32 ? fold_fits<OP_AHLA, 32>() : fold_fits<OP_AHLA, 64>();
    case OP_HLA3: return d == 32 ? fold_fits<OP_HLA3, 32>() : fold_fits<OP_HLA3, 64>();
    case OP_HLA2U: return d == 32 ? fold_fits<OP_HLA2U, 32>() : fold_fits<OP_HLA2U, 64>();
    case OP_AHLAD: return d == 32 ? fold_fits<OP_AHLAD, 32>() : fold_fits<OP_AHLAD, 64>();
    case OP_HLA3D: return d == 32 ? fold_fits<OP_HLA3D, 32>() : fold_fits<OP_HLA3D, 64>();
    }
    return false;
}

int kernel_launches(int op, bool norm, bool bf16, int d, int T) {
    if (op == OP_HLA2 && !norm && !bf16 && d == 32 && tc_second_order_f32_fits(T)) return 2;   // tcgen05, folded prefix
    if (op == OP_HLA3 || op == OP_HLA3D) return 2 + 3;   // the factored prefix (decayed or not)
    return 2 + (uses_fold(op, d) ? 1 : scan_launches(next_pow2((T + C - 1) / C)));
}

// ---------------------------------------------------------------------------
// Streaming state.  A head's state after t tokens is the summary of those t
// tokens in the layout above (the state the recurrence reaches from zero, with
// the maps the combine needs), so the chunk kernel and the up-sweep of the scan
// export it and the step kernel below advances it one token at a time.
// ---------------------------------------------------------------------------

// Copy the root of each head's up-sweep tree (slot NCp-1: every chunk combined) out.
template <int OP, int D>
__global__ void __launch_bounds__(NT) k_copy_root(const float* __restrict__ sums, int NCp, float* __restrict__ state) {
    using S = Sum<OP, D>;
    const float* src = sums + ((size_t)blockIdx.x * NCp + NCp - 1) * S::SIZE;
    float* dst = state + (size_t)blockIdx.x * S::SIZE;
    for (int e = threadIdx.x; e < S::SIZE; e += blockDim.x) dst[e] = src[e];
}

template <int OP, int D, typename TIn>
static cudaError_t state_run(const void* q, const void* k, const void* v, const float* gamma, int BH, int H, int T,
                             float* sums, float* state, cudaStream_t st) {
    const int NC = (T + C - 1) / C;
    const int NCp = next_pow2(NC);
    auto ks = k_summary<OP, D, TIn>;
    auto kl = k_scan_level<OP, D>;
    const size_t s1 = summary_smem<D>(), s2 = scan_smem<OP, D>();
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kl, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2)) != cudaSuccess) return e;
    ks<<<dim3(NCp, BH), NT, s1, st>>>((const TIn*)q, (const TIn*)k, (const TIn*)v, gamma, H, T, NC, NCp, sums);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    for (int step = 1; step < NCp; step *= 2) {            // up-sweep only: the root ends as the total
        kl<<<dim3(NCp / (2 * step), BH), NT, s2, st>>>(sums, NCp, step, 0, 0);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    k_copy_root<OP, D><<<BH, NT, 0, st>>>(sums, NCp, state);
    return cudaGetLastError();
}

template <typename TIn, int D>
static cudaError_t state_op(int op, const void* q, const void* k, const void* v, const float* gamma, int BH, int H,
                            int T, float* sums, float* state, cudaStream_t st) {
    switch (op) {
    case OP_HLA2: return state_run<OP_HLA2, D, TIn>(q, k, v, gamma, BH, H, T, sums, state, st);
    case OP_HLA2D: return state_run<OP_HLA2D, D, TIn>(q, k, v, gamma, BH, H, T, sums, state, st);
    case OP_AHLA: return state_run<OP_AHLA, D, TIn>(q, k, v, gamma, BH, H, T, sums, state, st);
    case OP_HLA3: return state_run<OP_HLA3, D, TIn>(q, k, v, gamma, BH, H, T, sums, state, st);
    case OP_HLA2U: return state_run<OP_HLA2U, D, TIn>(q, k, v, gamma, BH, H, T, sums, state, st);
    case OP_AHLAD: return state_run<OP_AHLAD, D, TIn>(q, k, v, gamma, BH, H, T, sums, state, st);
    case OP_HLA3D: return state_run<OP_HLA3D, D, TIn>(q, k, v, gamma, BH, H, T, sums, state, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t state(int op, bool bf16, int d, const void* q, const void* k, const void* v, const float* gamma, int BH,
                  int H, int T, float* sums, float* state_out, cudaStream_t st) {
    if (bf16) {
        if (d == 32) return state_op<__nv_bfloat16, 32>(op, q, k, v, gamma, BH, H, T, sums, state_out, st);
        return state_op<__nv_bfloat16, 64>(op, q, k, v, gamma, BH, H, T, sums, state_out, st);
    }
    if (d == 32) return state_op<float, 32>(op, q, k, v, gamma, BH, H, T, sums, state_out, st);
    return state_op<float, 64>(op, q, k, v, gamma, BH, H, T, sums, state_out, st);
}

int state_launches(int T) {
    int levels = 0;
    for (int p = 1; p < next_pow2((T + C - 1) / C); p *= 2) ++levels;
    return 2 + levels;                                       // chunk kernel, up-sweep levels, copy
}

// One token per head: the recurrence's update, on the summary layout, in fp32.
//   second order (R-form)  S += k k^T;  C += q v^T;  m += q;  z = S q;  R += z v^T;  r += z;
//                          o = q^T R  (ratio-normalised: / (q . r + eps))
//   decayed                w = g (k^T C), s = g (k . m);  S = g S + k k^T;  C = g C + q v^T;
//                          G = g G + k w^T;  m = g m + q;  h = g h + s k;  Khat += k k^T;
//                          rho *= g;  x = q^T S;  o = x^T C - q^T G  (/ (x . m - q . h + eps))
//   AHLA                   P += k v^T;  Dm += k q^T;  y = q^T P;  E += k y^T;  o = q^T E;
//                          mK += k;  n += (q . mK) k;  ratio-normalised: o / (q . n + eps)
//                          (decayed: P, E, mK, n scaled by g first, Dm not; rho *= g)
//   third order            S += k k^T;  P += k v^T;  Q2 += q q^T;  a = S q;  b = q^T P;
//                          F += a b^T;  X += q b^T;  Z += a q^T;  o = q^T F;  mK += k;
//                          F1 += (q . mK) a;  X1 += (q . mK) q;  ratio-normalised: / (q . F1 + eps)
//                          (decayed: S, P, F, mK, F1 scaled by g first; Q2 += rho g q q^T;
//                          X, Z, X1 not; rho *= g: the combine with the token's own summary)
//   unmasked               S += k k^T;  C += q v^T;  o = (q^T S) C
// S is symmetric, so every product with a vector reads matrix columns: thread j of a group
// walks rows i, and four groups of D threads split the rows (partial sums in shared memory).
// The head's state is staged in shared memory (every load in flight at once), updated there
// and written back once: one read and one write of the state per step.
template <int D>
__device__ __forceinline__ void col_dot(const float* __restrict__ M, const float* x, float* part, float* out) {
    const int j = threadIdx.x % D, g = threadIdx.x / D;       // NT / D groups
    constexpr int G = NT / D, RPG = D / G;
    float acc = 0.f;
#pragma unroll 4
    for (int i = g * RPG; i < (g + 1) * RPG; ++i) acc = fmaf(x[i], M[i * D + j], acc);
    part[g * D + j] = acc;
    __syncthreads();
    if (threadIdx.x < D) {
        float t = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) t += part[h * D + threadIdx.x];
        out[threadIdx.x] = t;
    }
    __syncthreads();
}

template <int OP, bool NORM, int D, typename TIn>
__global__ void __launch_bounds__(NT) k_step(float* __restrict__ state, const TIn* __restrict__ q,
                                             const TIn* __restrict__ k, const TIn* __restrict__ v,
                                             const float* __restrict__ gamma, float eps, int H, float* __restrict__ o) {
    using S = Sum<OP, D>;
    constexpr int DD = D * D;
    constexpr int N4 = S::SIZE / 4, PER = (N4 + NT - 1) / NT;
    __shared__ float qs[D], ks[D], vs[D], a[D], b[D], part[NT];
    __shared__ float scal[2];
    extern __shared__ float4 st4[];
    const int bh = blockIdx.x, tid = threadIdx.x;
    float4* gst = reinterpret_cast<float4*>(state + (size_t)bh * S::SIZE);
    // asynchronous 16-byte copies (no registers held): all of them in flight, then one wait
    for (int i = 0; i < PER; ++i) {
        const int e = tid + i * NT;
        if (e < N4) {
            const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(st4 + e));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(gst + e) : "memory");
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    float* st = reinterpret_cast<float*>(st4);
    if (tid < D) {
        qs[tid] = to_f32(q[(size_t)bh * D + tid]);
        ks[tid] = to_f32(k[(size_t)bh * D + tid]);
        vs[tid] = to_f32(v[(size_t)bh * D + tid]);
    }
    __syncthreads();
    if (OP == OP_HLA2) {
        float* Sm = st + S::mat(0); float* Cm = st + S::mat(1); float* Rm = st + S::mat(2);
        float* m = st + S::vec(0); float* r = st + S::vec(1);
        for (int e = tid; e < DD; e += NT) {
            const int i = e / D, j = e % D;
            Sm[e] = fmaf(ks[i], ks[j], Sm[e]);
            Cm[e] = fmaf(qs[i], vs[j], Cm[e]);
        }
        if (tid < D) m[tid] += qs[tid];
        __syncthreads();
        col_dot<D>(Sm, qs, part, a);                            // a = z = S q
        for (int e = tid; e < DD; e += NT) Rm[e] = fmaf(a[e / D], vs[e % D], Rm[e]);
        if (tid < D) r[tid] += a[tid];
        __syncthreads();
        col_dot<D>(Rm, qs, part, b);                            // b = q^T R
        if (tid < D) {
            float den = 1.f;
            if (NORM) {
                float t = 0.f;
                for (int i = 0; i < D; ++i) t = fmaf(qs[i], r[i], t);
                den = t + eps;
            }
            o[(size_t)bh * D + tid] = NORM ? b[tid] / den : b[tid];
        }
    } else if (OP == OP_HLA2D) {
        const float g = gamma[bh % H];
        float* Sm = st + S::mat(0); float* Cm = st + S::mat(1); float* Gm = st + S::mat(2); float* Kh = st + S::mat(3);
        float* m = st + S::vec(0); float* h = st + S::vec(1);
        col_dot<D>(Cm, ks, part, a);                            // a = k^T C (before the update)
        if (tid == 0) {
            float t = 0.f;
            for (int i = 0; i < D; ++i) t = fmaf(ks[i], m[i], t);
            scal[0] = g * t;                                    // s = g (k . m)
        }
        __syncthreads();
        for (int e = tid; e < DD; e += NT) {
            const int i = e / D, j = e % D;
            const float kk = ks[i] * ks[j];
            Sm[e] = fmaf(g, Sm[e], kk);
            Cm[e] = fmaf(g, Cm[e], qs[i] * vs[j]);
            Gm[e] = fmaf(g, Gm[e], ks[i] * (g * a[j]));
            Kh[e] += kk;
        }
        if (tid < D) {
            m[tid] = fmaf(g, m[tid], qs[tid]);
            h[tid] = fmaf(g, h[tid], scal[0] * ks[tid]);
        }
        if (tid == 0) st[S::SCAL] *= g;
        __syncthreads();
        col_dot<D>(Sm, qs, part, b);                            // b = x = q^T S
        // o_j = sum_i x_i C[i][j] - q_i G[i][j]
        {
            const int j = tid % D, gi = tid / D;
            constexpr int G = NT / D, RPG = D / G;
            float acc = 0.f;
            for (int i = gi * RPG; i < (gi + 1) * RPG; ++i) acc += b[i] * Cm[i * D + j] - qs[i] * Gm[i * D + j];
            part[gi * D + j] = acc;
        }
        __syncthreads();
        if (tid < D) {
            float t = 0.f;
            for (int hh = 0; hh < NT / D; ++hh) t += part[hh * D + tid];
            float den = 1.f;
            if (NORM) {
                float x = 0.f;
                for (int i = 0; i < D; ++i) x += b[i] * m[i] - qs[i] * h[i];
                den = x + eps;
            }
            o[(size_t)bh * D + tid] = NORM ? t / den : t;
        }
    } else if (OP == OP_HLA2U) {
        float* Sm = st + S::mat(0); float* Cm = st + S::mat(1);
        for (int e = tid; e < DD; e += NT) {
            const int i = e / D, j = e % D;
            Sm[e] = fmaf(ks[i], ks[j], Sm[e]);
            Cm[e] = fmaf(qs[i], vs[j], Cm[e]);
        }
        __syncthreads();
        col_dot<D>(Sm, qs, part, a);                            // a = q^T S
        col_dot<D>(Cm, a, part, b);                             // b = (q^T S) C
        if (tid < D) o[(size_t)bh * D + tid] = b[tid];
    } else if (OP == OP_AHLA || OP == OP_AHLAD) {
        // decayed: P, E, mK, n scaled by g before the update, D undecayed, rho *= g
        const float g = OP == OP_AHLAD ? gamma[bh % H] : 1.f;
        float* P = st + S::mat(0); float* E = st + S::mat(1); float* Dm = st + S::mat(2);
        for (int e = tid; e < DD; e += NT) {
            const int i = e / D, j = e % D;
            P[e] = fmaf(ks[i], vs[j], g * P[e]);
            Dm[e] = fmaf(ks[i], qs[j], Dm[e]);
            E[e] *= g;
        }
        float* mK = st + S::vec(0); float* n = st + S::vec(1);
        if (tid < D) {
            mK[tid] = fmaf(g, mK[tid], ks[tid]);
            n[tid] *= g;
        }
        if (OP == OP_AHLAD && tid == 0) st[S::SCAL] *= g;
        __syncthreads();
        col_dot<D>(P, qs, part, a);                             // a = y = q^T P
        if (tid == 0) {
            float t = 0.f;
            for (int i = 0; i < D; ++i) t = fmaf(qs[i], mK[i], t);
            scal[0] = t;                                        // y1 = q . mK
        }
        for (int e = tid; e < DD; e += NT) E[e] = fmaf(ks[e / D], a[e % D], E[e]);
        __syncthreads();
        if (tid < D) n[tid] = fmaf(ks[tid], scal[0], n[tid]);
        __syncthreads();
        col_dot<D>(E, qs, part, b);                             // b = q^T E
        if (tid < D) {
            float den = 1.f;
            if (NORM) {
                float t = 0.f;
                for (int i = 0; i < D; ++i) t = fmaf(qs[i], n[i], t);
                den = t + eps;
            }
            o[(size_t)bh * D + tid] = NORM ? b[tid] / den : b[tid];
        }
    } else {                                                    // OP_HLA3, OP_HLA3D
        // decayed: S, P, F, mK, F1 scaled by g before the update; Q2 gains the token with weight
        // rho g (its position's), X, Z, X1 undecayed; rho *= g
        const float g = OP == OP_HLA3D ? gamma[bh % H] : 1.f;
        const float wq = OP == OP_HLA3D ? st[S::SCAL] * g : 1.f;
        float* Sm = st + S::mat(0); float* Q2 = st + S::mat(1); float* P = st + S::mat(2);
        float* F = st + S::mat(3); float* X = st + S::mat(4); float* Z = st + S::mat(5);
        __syncthreads();                                        // every thread has read rho
        for (int e = tid; e < DD; e += NT) {
            const int i = e / D, j = e % D;
            Sm[e] = fmaf(ks[i], ks[j], g * Sm[e]);
            P[e] = fmaf(ks[i], vs[j], g * P[e]);
            Q2[e] = fmaf(wq * qs[i], qs[j], Q2[e]);
            F[e] *= g;
        }
        float* mK = st + S::vec(0); float* X1 = st + S::vec(1); float* F1 = st + S::vec(2);
        if (tid < D) {
            mK[tid] = fmaf(g, mK[tid], ks[tid]);
            F1[tid] *= g;
        }
        if (OP == OP_HLA3D && tid == 0) st[S::SCAL] = wq;
        __syncthreads();
        col_dot<D>(Sm, qs, part, a);                            // a = S q
        col_dot<D>(P, qs, part, b);                             // b = q^T P
        if (tid == 0) {
            float t = 0.f;
            for (int i = 0; i < D; ++i) t = fmaf(qs[i], mK[i], t);
            scal[0] = t;                                        // b1 = q . mK
        }
        for (int e = tid; e < DD; e += NT) {
            const int i = e / D, j = e % D;
            F[e] = fmaf(a[i], b[j], F[e]);
            X[e] = fmaf(qs[i], b[j], X[e]);
            Z[e] = fmaf(a[i], qs[j], Z[e]);
        }
        __syncthreads();
        if (tid < D) {
            F1[tid] = fmaf(a[tid], scal[0], F1[tid]);
            X1[tid] = fmaf(qs[tid], scal[0], X1[tid]);
        }
        __syncthreads();
        col_dot<D>(F, qs, part, a);                             // a = q^T F
        if (tid < D) {
            float den = 1.f;
            if (NORM) {
                float t = 0.f;
                for (int i = 0; i < D; ++i) t = fmaf(qs[i], F1[i], t);
                den = t + eps;
            }
            o[(size_t)bh * D + tid] = NORM ? a[tid] / den : a[tid];
        }
    }
    __syncthreads();
    for (int e = tid; e < N4; e += NT) gst[e] = st4[e];
}

// The same step for the second-order family (R-form, decayed, unmasked) with a head's state
// split by rows over a cluster of STEP_CL CTAs, so that a step's DRAM round trip is spread over
// STEP_CL times more SMs.  Every row-local part of the update stays in its CTA:
//   S_i += k_i k,  C_i += q_i v,  z_i = S_i . q  (S symmetric: S q reads row i),  R_i += z_i v;
// only sums over the rows cross CTAs: the output o_j = sum_i q_i R_ij (second order),
// sum_i x_i C_ij - q_i G_ij (decayed), sum_i x_i C_ij (unmasked), their denominators, and the
// decayed form's a = k^T C and k . m taken before its update.  Each such sum is one partial
// vector per CTA, which the CTA writes into slot `rank` of every CTA's shared memory (distributed
// shared memory stores); after one cluster barrier each CTA adds its slots locally.  No CTA
// touches another's shared memory after the last barrier, so none waits for the others to leave.
constexpr int STEP_CL = 8;    // CTAs per head
constexpr int STEP_NT = 128;  // threads per CTA: a float4 of each owned matrix row slice per thread

template <int OP, bool NORM, int D, typename TIn>
__global__ void __cluster_dims__(STEP_CL, 1, 1) __launch_bounds__(STEP_NT)
    k_step_rows(float* __restrict__ state, const TIn* __restrict__ q, const TIn* __restrict__ k,
                const TIn* __restrict__ v, const float* __restrict__ gamma, float eps, int H, float* __restrict__ o) {
    using S = Sum<OP, D>;
    constexpr int ROWS = D / STEP_CL;        // rows of every matrix this CTA owns
    constexpr int LPR = D / 4;               // threads per row, one float4 each
    constexpr int ACT = ROWS * LPR;          // threads that own a float4 of every matrix
    constexpr int NM = S::NMAT;
    static_assert(ACT <= STEP_NT && 32 % LPR == 0, "row slice layout");
    __shared__ float qs[D], ks[D], vs[D], full[D + 1];
    __shared__ float prod[ROWS][D + 1];      // per-row terms of a sum over rows
    __shared__ float red[2][STEP_CL][D + 1]; // every CTA's partial sums, two rounds
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = static_cast<int>(cl.block_rank());
    const int bh = blockIdx.x / STEP_CL, tid = threadIdx.x;
    const int rl = tid / LPR, j0 = 4 * (tid % LPR), i = rank * ROWS + rl;
    const bool act = tid < ACT, lead = act && (tid % LPR) == 0;
    float* st = state + (size_t)bh * S::SIZE;

    float4 M[NM];
    float vec0 = 0.f, vec1 = 0.f;
    if (act) {
#pragma unroll
        for (int m = 0; m < NM; ++m) M[m] = *reinterpret_cast<const float4*>(st + S::mat(m) + i * D + j0);
        if (S::NVEC > 0 && lead) {
            vec0 = st[S::vec(0) + i];
            vec1 = st[S::vec(1) + i];
        }
    }
    if (tid < D) {
        qs[tid] = to_f32(q[(size_t)bh * D + tid]);
        ks[tid] = to_f32(k[(size_t)bh * D + tid]);
        vs[tid] = to_f32(v[(size_t)bh * D + tid]);
    }
    __syncthreads();

    // Sum over the cluster's rows of prod[.][0 .. n): this CTA's rows, stored into slot `rank` of
    // red[buf] in every CTA of the cluster; one cluster barrier; the slots added into full[0 .. n).
    auto cluster_sum = [&](int buf, int n) {
        __syncthreads();
        for (int t = tid; t < n; t += STEP_NT) {
            float a = 0.f;
#pragma unroll
            for (int r = 0; r < ROWS; ++r) a += prod[r][t];
#pragma unroll
            for (int r = 0; r < STEP_CL; ++r) cl.map_shared_rank(&red[buf][rank][0], r)[t] = a;
        }
        cl.sync();
        for (int t = tid; t < n; t += STEP_NT) {
            float a = 0.f;
#pragma unroll
            for (int r = 0; r < STEP_CL; ++r) a += red[buf][r][t];
            full[t] = a;
        }
        __syncthreads();
    };
    auto row_dot = [&](const float4& x) {          // row i of a matrix . q, over the row's LPR threads
        float a = x.x * qs[j0] + x.y * qs[j0 + 1] + x.z * qs[j0 + 2] + x.w * qs[j0 + 3];
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        return a;
    };
    const float4 k4 = make_float4(ks[j0], ks[j0 + 1], ks[j0 + 2], ks[j0 + 3]);
    const float4 v4 = make_float4(vs[j0], vs[j0 + 1], vs[j0 + 2], vs[j0 + 3]);
    auto axpy = [](float4& y, float a, const float4& x) {
        y.x = fmaf(a, x.x, y.x); y.y = fmaf(a, x.y, y.y); y.z = fmaf(a, x.z, y.z); y.w = fmaf(a, x.w, y.w);
    };
    auto put = [&](float4 x) {
        prod[rl][j0] = x.x; prod[rl][j0 + 1] = x.y; prod[rl][j0 + 2] = x.z; prod[rl][j0 + 3] = x.w;
    };
    float qi = 0.f, ki = 0.f;
    if (act) { qi = qs[i]; ki = ks[i]; }
    int nred = D;                                   // length of the final sum (D + 1 with a denominator)

    if (OP == OP_HLA2) {                            // S=0 C=1 R=2 ; m r
        float z = 0.f;
        if (act) {
            axpy(M[0], ki, k4);
            axpy(M[1], qi, v4);
            z = row_dot(M[0]);
            axpy(M[2], z, v4);
            vec0 += qi;
            vec1 += z;
            put(make_float4(qi * M[2].x, qi * M[2].y, qi * M[2].z, qi * M[2].w));
            if (NORM && lead) prod[rl][D] = qi * vec1;
        }
        nred = NORM ? D + 1 : D;
    } else if (OP == OP_HLA2U) {                    // S=0 C=1
        if (act) {
            axpy(M[0], ki, k4);
            axpy(M[1], qi, v4);
            const float x = row_dot(M[0]);
            put(make_float4(x * M[1].x, x * M[1].y, x * M[1].z, x * M[1].w));
        }
    } else {                                        // OP_HLA2D: S=0 C=1 G=2 Khat=3 ; m h ; rho
        const float g = gamma[bh % H];
        if (act) {                                  // a = k^T C and k . m, before the update
            put(make_float4(ki * M[1].x, ki * M[1].y, ki * M[1].z, ki * M[1].w));
            if (lead) prod[rl][D] = ki * vec0;
        }
        cluster_sum(0, D + 1);
        if (act) {
            const float4 a4 = make_float4(g * full[j0], g * full[j0 + 1], g * full[j0 + 2], g * full[j0 + 3]);
            const float sg = g * full[D];
            M[0] = make_float4(fmaf(g, M[0].x, ki * k4.x), fmaf(g, M[0].y, ki * k4.y), fmaf(g, M[0].z, ki * k4.z),
                               fmaf(g, M[0].w, ki * k4.w));
            M[1] = make_float4(fmaf(g, M[1].x, qi * v4.x), fmaf(g, M[1].y, qi * v4.y), fmaf(g, M[1].z, qi * v4.z),
                               fmaf(g, M[1].w, qi * v4.w));
            M[2] = make_float4(fmaf(g, M[2].x, ki * a4.x), fmaf(g, M[2].y, ki * a4.y), fmaf(g, M[2].z, ki * a4.z),
                               fmaf(g, M[2].w, ki * a4.w));
            M[3].x += ki * k4.x; M[3].y += ki * k4.y; M[3].z += ki * k4.z; M[3].w += ki * k4.w;
            vec0 = fmaf(g, vec0, qi);
            vec1 = fmaf(g, vec1, sg * ki);
            const float x = row_dot(M[0]);
            put(make_float4(x * M[1].x - qi * M[2].x, x * M[1].y - qi * M[2].y, x * M[1].z - qi * M[2].z,
                            x * M[1].w - qi * M[2].w));
            if (NORM && lead) prod[rl][D] = x * vec0 - qi * vec1;
        }
        if (rank == 0 && tid == 0) st[S::SCAL] *= g;
        nred = NORM ? D + 1 : D;
    }
    if (act) {
#pragma unroll
        for (int m = 0; m < NM; ++m) *reinterpret_cast<float4*>(st + S::mat(m) + i * D + j0) = M[m];
        if (S::NVEC > 0 && lead) {
            st[S::vec(0) + i] = vec0;
            st[S::vec(1) + i] = vec1;
        }
    }
    cluster_sum(1, nred);
    constexpr int OC = D / STEP_CL;                 // output columns written by this CTA
    if (tid < OC) {
        const int j = rank * OC + tid;
        o[(size_t)bh * D + j] = NORM ? full[j] / (full[D] + eps) : full[j];
    }
}

template <int OP, bool NORM, int D, typename TIn>
static cudaError_t step_rows_launch(float* st_, const void* q, const void* k, const void* v, const float* gamma,
                                    float eps, int BH, int H, float* o, cudaStream_t st) {
    k_step_rows<OP, NORM, D, TIn><<<BH * STEP_CL, STEP_NT, 0, st>>>(st_, (const TIn*)q, (const TIn*)k,
                                                                    (const TIn*)v, gamma, eps, H, o);
    return cudaGetLastError();
}

template <int OP, bool NORM, int D, typename TIn>
static cudaError_t step_launch(float* st_, const void* q, const void* k, const void* v, const float* gamma,
                               float eps, int BH, int H, float* o, cudaStream_t st) {
    auto kf = k_step<OP, NORM, D, TIn>;
    const int smem = Sum<OP, D>::SIZE * (int)sizeof(float);     // the head's state
    cudaError_t e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kf<<<BH, NT, smem, st>>>(st_, (const TIn*)q, (const TIn*)k, (const TIn*)v, gamma, eps, H, o);
    return cudaGetLastError();
}

template <typename TIn, int D>
static cudaError_t step_op(int op, bool norm, float* st_, const void* q, const void* k, const void* v,
                           const float* gamma, float eps, int BH, int H, float* o, cudaStream_t st) {
    switch (op) {
    case OP_HLA2:
        return norm ? step_rows_launch<OP_HLA2, true, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st)
                    : step_rows_launch<OP_HLA2, false, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st);
    case OP_HLA2D:
        return norm ? step_rows_launch<OP_HLA2D, true, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st)
                    : step_rows_launch<OP_HLA2D, false, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st);
    case OP_AHLA:
        return norm ? step_launch<OP_AHLA, true, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st)
                    : step_launch<OP_AHLA, false, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st);
    case OP_HLA3:
        return norm ? step_launch<OP_HLA3, true, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st)
                    : step_launch<OP_HLA3, false, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st);
    case OP_HLA2U: return step_rows_launch<OP_HLA2U, false, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st);
    case OP_AHLAD:
        return norm ? step_launch<OP_AHLAD, true, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st)
                    : step_launch<OP_AHLAD, false, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st);
    case OP_HLA3D:
        return norm ? step_launch<OP_HLA3D, true, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st)
                    : step_launch<OP_HLA3D, false, D, TIn>(st_, q, k, v, gamma, eps, BH, H, o, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t step(int op, bool norm, bool bf16, int d, float* state_io, const void* q, const void* k, const void* v,
                 const float* gamma, float eps, int BH, int H, float* o, cudaStream_t st) {
    if (bf16) {
        if (d == 32) return step_op<__nv_bfloat16, 32>(op, norm, state_io, q, k, v, gamma, eps, BH, H, o, st);
        return step_op<__nv_bfloat16, 64>(op, norm, state_io, q, k, v, gamma, eps, BH, H, o, st);
    }
    if (d == 32) return step_op<float, 32>(op, norm, state_io, q, k, v, gamma, eps, BH, H, o, st);
    return step_op<float, 64>(op, norm, state_io, q, k, v, gamma, eps, BH, H, o, st);
}



// ===========================================================================
// Backward pass of the masked second-order output (no decay, not normalised).
//
// "Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 4 and
// Contribuciones 2: the page offers the exact scan as the basis of exact parallel training but
// prints no gradient.  These kernels differentiate the chunk algebra of the forward: for chunk c
// (Q, K, V, dO: its 64-row tiles; S0, R0: the state carried in, the forward scan's exclusive
// prefix; dS', dR': the adjoints of the state it hands on)
//     A = L (.) Q K^T,  P = Q S0,  W = L (.) (P Q^T + A A^T),  Z = P + A K,
//     O = Q R0 + W V,   S0' = S0 + K^T K,   R0' = R0 + Z^T V,
// reverse mode gives
//     dW = L (.) dO V^T,   dV = W^T dO + Z dR',   dZ = V dR'^T,   dP = dZ + dW Q,
//     dA = L (.) (dZ K^T + (dW + dW^T) A),
//     dQ = dO R0^T + dW^T P + dP S0^T + dA K,   dK = K (dS' + dS'^T) + A^T dZ + dA^T Q,
// and the adjoints handed back, dR = dR' + Q^T dO and dS = dS' + Q^T dP.  Unrolled over the
// chunks after c they are suffix sums:
//     dR'(c) = sum_{m > c} Q_m^T dO_m,
//     dS'(c) = sum_{m > c} (U_m + C_m dR'(m)^T),   U_m = Q_m^T (dW_m Q_m),  C_m = Q_m^T V_m,
// so every chunk runs in parallel apart from two element-wise suffix sums:
//   the forward's chunk summaries and scan (S0, R0 per chunk);
//   k_bwd_chunk: Y = Q^T dO, U, C per chunk;  k_bwd_suffix: dR' in place of Y;
//   k_bwd_cross: X = U + C dR'^T in place of U;  k_bwd_suffix: dS' in place of X;
//   k_bwd_out: dQ, dK, dV of every chunk.
// Everything in fp32 on the CUDA cores; bf16 inputs are widened on load.
// ===========================================================================
template <int D>
struct Bwd {
    static constexpr int DD = D * D;
    static constexpr int SIZE = 3 * DD;       // per chunk: [Y | dR'], [U | X | dS'], C
};

// The (dW + dW^T) view of a masked c x c tile.
struct SymTile {
    const float* p;
    int ld;
    __device__ float operator()(int r, int c) const { return p[r * ld + c] + p[c * ld + r]; }
};
// Global row-major D x D matrix views.
struct GMat {
    const float* p;
    int ld;
    __device__ float operator()(int r, int c) const { return p[r * ld + c]; }
};
struct GMatT {
    const float* p;
    int ld;
    __device__ float operator()(int r, int c) const { return p[c * ld + r]; }
};
// Store into a tile with the causal mask (column > row written as 0).
struct PutMasked {
    float* p;
    int ld;
    __device__ void operator()(int r, int c, float x) const { p[r * ld + c] = c <= r ? x : 0.f; }
};

template <int D, typename TIn>
__global__ void __launch_bounds__(NT) k_bwd_chunk(const TIn* __restrict__ q, const TIn* __restrict__ v,
                                                  const float* __restrict__ dout, int T, int NCp,
                                                  float* __restrict__ bw) {
    constexpr int LD = Dim<D>::LD;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    extern __shared__ float sm[];
    float* Qs = sm;
    float* Vs = Qs + C * LD;
    float* Os = Vs + C * LD;                  // dO
    float* dWs = Os + C * LD;                 // C x LDC
    float* Gs = dWs + C * LDC;                // dW Q
    const size_t head = (size_t)bh * T * D;
    const int t0 = chunk * C;
    load_rows<D>(Qs, q + head, t0, T);
    load_rows<D>(Vs, v + head, t0, T);
    load_rows<D>(Os, dout + head, t0, T);
    __syncthreads();
    float* out = bw + ((size_t)bh * NCp + chunk) * Bwd<D>::SIZE;
    // Y = Q^T dO, C = Q^T V, dW = L (.) dO V^T
    mm<D, D, C>(TileT{Qs, LD}, Tile{Os, LD}, Zero{}, [&](int r, int c, float x) { out[r * D + c] = x; });
    mm<D, D, C>(TileT{Qs, LD}, Tile{Vs, LD}, Zero{}, [&](int r, int c, float x) { out[2 * D * D + r * D + c] = x; });
    mm<C, C, D>(Tile{Os, LD}, TileT{Vs, LD}, Zero{}, PutMasked{dWs, LDC});
    __syncthreads();
    mm<C, D, C>(Tile{dWs, LDC}, Tile{Qs, LD}, Zero{}, Put{Gs, LD});          // dW Q
    __syncthreads();
    mm<D, D, C>(TileT{Qs, LD}, Tile{Gs, LD}, Zero{}, [&](int r, int c, float x) { out[D * D + r * D + c] = x; });
}

// Exclusive suffix sum over a head's NC chunks of matrix slot `slot`, element-wise and in place.
template <int D>
__global__ void __launch_bounds__(NT) k_bwd_suffix(float* __restrict__ bw, int NC, int NCp, int slot) {
    const int e = blockIdx.x * NT + threadIdx.x;
    if (e >= D * D) return;
    float* p = bw + (size_t)blockIdx.y * NCp * Bwd<D>::SIZE + slot * D * D + e;
    float run = 0.f;
    for (int c0 = NC - 1; c0 >= 0; c0 -= 32) {     // 32 independent loads in flight
        float y[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (c0 - i >= 0) y[i] = p[(size_t)(c0 - i) * Bwd<D>::SIZE];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (c0 - i >= 0) {
                p[(size_t)(c0 - i) * Bwd<D>::SIZE] = run;
                run += y[i];
            }
    }
}

// X = U + C dR'^T per chunk, in place of U.
template <int D>
__global__ void __launch_bounds__(NT) k_bwd_cross(float* __restrict__ bw, int NCp, int trans) {
    constexpr int LD = Dim<D>::LD;
    __shared__ float Cs[D * LD], Rs[D * LD];
    float* slot = bw + ((size_t)blockIdx.y * NCp + blockIdx.x) * Bwd<D>::SIZE;
    load_mats<D, 2>({Cs, Rs}, {slot + 2 * D * D, slot});
    __syncthreads();
    float* U = slot + D * D;
    auto acc = [&](int r, int c) { return U[r * D + c]; };
    auto put = [&](int r, int c, float x) { U[r * D + c] = x; };
    if (trans) mm<D, D, D>(Tile{Cs, LD}, TileT{Rs, LD}, acc, put);     // second order: U + C dR'^T
    else mm<D, D, D>(Tile{Cs, LD}, Tile{Rs, LD}, acc, put);            // AHLA: U + M dE'
}

template <int D, typename TIn>
__global__ void __launch_bounds__(NT) k_bwd_out(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                const TIn* __restrict__ v, const float* __restrict__ dout,
                                                int T, int NCp, const float* __restrict__ sums,
                                                const float* __restrict__ bw, float* __restrict__ dq,
                                                float* __restrict__ dk, float* __restrict__ dv) {
    using S = Sum<OP_HLA2, D>;
    constexpr int LD = Dim<D>::LD;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    const float* pre = sums + ((size_t)bh * NCp + chunk) * S::SIZE;          // S0 = mat(0), R0 = mat(2)
    const float* adj = bw + ((size_t)bh * NCp + chunk) * Bwd<D>::SIZE;       // dR' = 0, dS' = 1
    extern __shared__ float sm[];
    float* Qs = sm;
    float* Ks = Qs + C * LD;
    float* Vs = Ks + C * LD;                  // V, later the first three terms of dQ
    float* Os = Vs + C * LD;                  // dO
    float* Ps = Os + C * LD;                  // P
    float* Zs = Ps + C * LD;                  // Z, later dP
    float* As = Zs + C * LD;                  // C x LDC: A
    float* Ws = As + C * LDC;                 // W, later dZ
    float* dWs = Ws + C * LDC;                // dW
    float* dAs = dWs + C * LDC;               // dA
    float* M0 = dAs + C * LDC;                // D x LD: S0, later dS' + dS'^T
    float* M1 = M0 + D * LD;                  // dR', later R0
    const size_t head = (size_t)bh * T * D;
    const int t0 = chunk * C;
    load_rows<D>(Qs, q + head, t0, T);
    load_rows<D>(Ks, k + head, t0, T);
    load_rows<D>(Vs, v + head, t0, T);
    load_rows<D>(Os, dout + head, t0, T);
    load_mat<D>(M0, pre + S::mat(0));
    load_mat<D>(M1, adj);
    __syncthreads();
    mm<C, C, D>(Tile{Qs, LD}, TileT{Ks, LD}, Zero{}, PutMasked{As, LDC});     // A
    mm<C, D, D>(Tile{Qs, LD}, Tile{M0, LD}, Zero{}, Put{Ps, LD});              // P = Q S0
    mm<C, C, D>(Tile{Os, LD}, TileT{Vs, LD}, Zero{}, PutMasked{dWs, LDC});    // dW
    __syncthreads();
    mm2<C, C, D, C>(Tile{Ps, LD}, TileT{Qs, LD}, Tile{As, LDC}, TileT{As, LDC}, Zero{}, PutMasked{Ws, LDC});  // W
    mm<C, D, C>(Tile{As, LDC}, Tile{Ks, LD}, [&](int r, int c) { return Ps[r * LD + c]; }, Put{Zs, LD});   // Z
    __syncthreads();
    // dV = W^T dO + Z dR'
    mm2<C, D, C, D>(TileT{Ws, LDC}, Tile{Os, LD}, Tile{Zs, LD}, Tile{M1, LD}, Zero{},
                    [&](int r, int c, float x) { if (t0 + r < T) dv[head + (size_t)(t0 + r) * D + c] = x; });
    __syncthreads();
    mm<C, D, D>(Tile{Vs, LD}, TileT{M1, LD}, Zero{}, Put{Ws, LD});            // dZ = V dR'^T (over W)
    __syncthreads();
    mm<C, D, C>(Tile{dWs, LDC}, Tile{Qs, LD}, [&](int r, int c) { return Ws[r * LD + c]; }, Put{Zs, LD});  // dP
    mm2<C, C, D, C>(Tile{Ws, LD}, TileT{Ks, LD}, SymTile{dWs, LDC}, Tile{As, LDC}, Zero{}, PutMasked{dAs, LDC});  // dA
    load_mat<D>(M1, pre + S::mat(2));                                         // R0
    __syncthreads();
    // dQ = dO R0^T + dW^T P + dA K (+ dP S0^T below)
    mm3<C, D, D, C, C>(Tile{Os, LD}, TileT{M1, LD}, TileT{dWs, LDC}, Tile{Ps, LD}, Tile{dAs, LDC}, Tile{Ks, LD},
                       Zero{}, Put{Vs, LD});
    __syncthreads();
    mm<C, D, D>(Tile{Zs, LD}, TileT{M0, LD}, [&](int r, int c) { return Vs[r * LD + c]; },
                [&](int r, int c, float x) { if (t0 + r < T) dq[head + (size_t)(t0 + r) * D + c] = x; });
    __syncthreads();
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) {                   // dS' + dS'^T
        const int r = e / D, c = e % D;
        M0[r * LD + c] = adj[D * D + r * D + c] + adj[D * D + c * D + r];
    }
    __syncthreads();
    // dK = K (dS' + dS'^T) + A^T dZ + dA^T Q
    mm3<C, D, D, C, C>(Tile{Ks, LD}, Tile{M0, LD}, TileT{As, LDC}, Tile{Ws, LD}, TileT{dAs, LDC}, Tile{Qs, LD},
                       Zero{}, [&](int r, int c, float x) { if (t0 + r < T) dk[head + (size_t)(t0 + r) * D + c] = x; });
}

template <int D>
static size_t bwd_chunk_smem() {
    return sizeof(float) * (size_t)(4 * C * Dim<D>::LD + C * LDC);
}
template <int D>
static size_t bwd_out_smem() {
    return sizeof(float) * (size_t)(6 * C * Dim<D>::LD + 4 * C * LDC + 2 * D * Dim<D>::LD);
}

size_t backward_workspace_floats(int d, int BH, int T) {
    const int NCp = next_pow2((T + C - 1) / C);
    // forward summaries, adjoint slots, and at d = 64 the 128-token prefixes of the tensor-core path
    return workspace_floats(OP_HLA2, d, BH, T) + (size_t)BH * NCp * 3 * d * d +
           (d == 64 ? tc::chunk_prefix_floats(BH, T) : 0);
}

int backward_launches(bool bf16, int d, int T) {
    // bf16 at d = 64: summary walker, three prefix kernels, chunk terms, two suffix sums, cross
    // term, gradients (128-token chunks); otherwise summaries, the scan, the same adjoint stages
    // (64-token chunks), gradients
    if (bf16 && d == 64) return 4 + 5;
    return kernel_launches(OP_HLA2, false, true, d, T) - 1 + 5;
}

template <int D, typename TIn>
static cudaError_t backward_run(const void* q, const void* k, const void* v, const float* dout, float* dq, float* dk,
                                float* dv, int BH, int T, float* ws, int* status, bool fp32_only, cudaStream_t st) {
    const int NC = (T + C - 1) / C;
    const int NCp = next_pow2(NC);
    float* sums = ws;
    float* bw = ws + workspace_floats(OP_HLA2, D, BH, T);
    cudaError_t e;
    if (D == 64 && sizeof(TIn) == 2 && !fp32_only) {
        // tensor-core path, 128-token chunks throughout: the state entering every chunk (summary
        // walker over one-chunk segments, segment-prefix kernels), the adjoint terms, their
        // suffix sums and cross term (CUDA cores), the gradients
        float* pre = bw + (size_t)BH * NCp * Bwd<D>::SIZE;
        const int NC2 = (T + 127) / 128, NSp2 = next_pow2(NC2);
        if ((e = tc::chunk_prefixes(q, k, v, BH, T, sums, pre, status, st)) != cudaSuccess) return e;
        if ((e = tc::bwd_terms(q, v, dout, bw, BH, T, status, st)) != cudaSuccess) return e;
        const dim3 sg2((D * D + NT - 1) / NT, BH);
        k_bwd_suffix<D><<<sg2, NT, 0, st>>>(bw, NC2, NSp2, 0);                // dR'
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        k_bwd_cross<D><<<dim3(NC2, BH), NT, 0, st>>>(bw, NSp2, 1);             // X = U + C dR'^T
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        k_bwd_suffix<D><<<sg2, NT, 0, st>>>(bw, NC2, NSp2, 1);                // dS'
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        return tc::bwd_out(q, k, v, dout, pre, bw, dq, dk, dv, BH, T, status, st);
    }
    auto ks = k_summary<OP_HLA2, D, TIn>;
    auto kc = k_bwd_chunk<D, TIn>;
    auto ko = k_bwd_out<D, TIn>;
    const size_t s1 = summary_smem<D>(), s2 = bwd_chunk_smem<D>(), s3 = bwd_out_smem<D>();
    if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ko, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3)) != cudaSuccess) return e;
    // the forward's carried states: chunk summaries, then their exclusive scan
    ks<<<dim3(NCp, BH), NT, s1, st>>>((const TIn*)q, (const TIn*)k, (const TIn*)v, nullptr, 1, T, NC, NCp, sums);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (fold_fits<OP_HLA2, D>()) {
        auto kf = k_scan_fold<OP_HLA2, D>;
        if ((e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)fold_smem<OP_HLA2, D>())) != cudaSuccess)
            return e;
        kf<<<BH, NT, fold_smem<OP_HLA2, D>(), st>>>(sums, NC, NCp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else if ((e = scan_levels<OP_HLA2, D>(sums, NCp, BH, st)) != cudaSuccess) {
        return e;
    }
    kc<<<dim3(NC, BH), NT, s2, st>>>((const TIn*)q, (const TIn*)v, dout, T, NCp, bw);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 sg((D * D + NT - 1) / NT, BH);
    k_bwd_suffix<D><<<sg, NT, 0, st>>>(bw, NC, NCp, 0);                       // dR'
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_cross<D><<<dim3(NC, BH), NT, 0, st>>>(bw, NCp, 1);                   // X = U + C dR'^T
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_suffix<D><<<sg, NT, 0, st>>>(bw, NC, NCp, 1);                       // dS'
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ko<<<dim3(NC, BH), NT, s3, st>>>((const TIn*)q, (const TIn*)k, (const TIn*)v, dout, T, NCp, sums, bw, dq, dk,
                                     dv);
    return cudaGetLastError();
}

cudaError_t backward(bool bf16, int d, const void* q, const void* k, const void* v, const float* dout, float* dq,
                     float* dk, float* dv, int BH, int T, float* ws, int* status, cudaStream_t st,
                     bool fp32_only);

// ---------------------------------------------------------------------------
// Ratio-normalised second order: o = num / (den + eps), num = W V and den = W 1 (the same operator
// on a ones value column).  With dO given,
//     dnum = dO / (den + eps),   dden_t = -sum_f dO_tf num_tf / (den_t + eps)^2,
// and den_t is column 0 of the operator on an all-ones value tensor, whose gradient with respect
// to q and k, for an output gradient that is dden in column 0 and zero elsewhere, is the ones
// term.  So (dq, dk, dv) = backward(q, k, v; dnum) + (the dq, dk of backward(q, k, 1; [dden, 0..])).
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void k_fill_ones(TIn* __restrict__ x, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        x[i] = TIn(1.f);
}

// One thread per (token, head) row: dnum and the ones term's output gradient (dden in column 0).
template <int D>
__global__ void k_norm_grads(const float* __restrict__ num, const float* __restrict__ den, const float* __restrict__ dout,
                             float eps, size_t rows, float* __restrict__ dnum, float* __restrict__ g1) {
    const size_t r = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const float s = 1.f / (den[r * D] + eps);
    float acc = 0.f;
    for (int f = 0; f < D; ++f) {
        const float g = dout[r * D + f];
        dnum[r * D + f] = g * s;
        acc = fmaf(g, num[r * D + f], acc);
        g1[r * D + f] = 0.f;
    }
    g1[r * D] = -acc * s * s;
}

__global__ void k_add_into(float* __restrict__ a, const float* __restrict__ b, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        a[i] += b[i];
}

size_t backward_normalized_workspace_floats(int d, int BH, int T) {
    const size_t n = (size_t)BH * T * d;
    const size_t inner = std::max(backward_workspace_floats(d, BH, T), workspace_floats(OP_HLA2, d, BH, T));
    // num, the ones operator, the ones (as fp32: big enough for either dtype), dnum, its ones term's
    // output gradient, dq2, dk2, dv2
    return 8 * n + inner;
}

int backward_normalized_launches(bool bf16, int d, int T) {
    // two plain forwards, the ones, the gradient split, two plain backwards, two additions
    // (the two forwards stay on the CUDA cores: the gradient combines them with cancellation)
    return 2 * kernel_launches(OP_HLA2, false, true, d, T) + 1 + 1 + 2 * backward_launches(false, d, T) + 2;
}

cudaError_t backward_normalized(bool bf16, int d, const void* q, const void* k, const void* v, const float* dout,
                                float eps, float* dq, float* dk, float* dv, int BH, int T, float* ws, int* status,
                                cudaStream_t st) {
    const size_t n = (size_t)BH * T * d;
    float* num = ws;
    float* den = num + n;
    float* ones = den + n;
    float* dnum = ones + n;
    float* g1 = dnum + n;
    float* dq2 = g1 + n;
    float* dk2 = dq2 + n;
    float* dv2 = dk2 + n;
    float* inner = dv2 + n;
    const int blocks = 4 * 148;
    cudaError_t e;
    if (bf16) k_fill_ones<__nv_bfloat16><<<blocks, NT, 0, st>>>(reinterpret_cast<__nv_bfloat16*>(ones), n);
    else k_fill_ones<float><<<blocks, NT, 0, st>>>(ones, n);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = forward(OP_HLA2, false, bf16, d, q, k, v, nullptr, 0.f, num, BH, 1, T, inner, status, st, nullptr, false)) !=
        cudaSuccess)
        return e;
    if ((e = forward(OP_HLA2, false, bf16, d, q, k, ones, nullptr, 0.f, den, BH, 1, T, inner, status, st, nullptr, false)) !=
        cudaSuccess)
        return e;
    const size_t rows = (size_t)BH * T;
    if (d == 32) k_norm_grads<32><<<(unsigned)((rows + NT - 1) / NT), NT, 0, st>>>(num, den, dout, eps, rows, dnum, g1);
    else k_norm_grads<64><<<(unsigned)((rows + NT - 1) / NT), NT, 0, st>>>(num, den, dout, eps, rows, dnum, g1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // The two terms of dq and dk nearly cancel where o barely depends on q and k (o = v for a
    // constant v), so both passes keep the fp32 gradient kernel: bf16 operands would leave an
    // error of the size of each term, not of their difference.
    if ((e = backward(bf16, d, q, k, v, dnum, dq, dk, dv, BH, T, inner, status, st, true)) != cudaSuccess) return e;
    if ((e = backward(bf16, d, q, k, ones, g1, dq2, dk2, dv2, BH, T, inner, status, st, true)) != cudaSuccess)
        return e;
    k_add_into<<<blocks, NT, 0, st>>>(dq, dq2, n);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_add_into<<<blocks, NT, 0, st>>>(dk, dk2, n);
    return cudaGetLastError();
}

// ===========================================================================
// Backward pass of the AHLA output (no decay, not normalised).  The forward's chunk algebra:
//     A = L (.) Q K^T,  Y = Q P0 + A V,  O = Q E0 + A Y,  P0' = P0 + K^T V,  E0' = E0 + K^T Y.
// Reverse mode, with dO given and (dP', dE') the adjoints of the state the chunk hands on:
//     dY = A^T dO + K dE',   dA = L (.) (dO Y^T + dY V^T),
//     dQ = dO E0^T + dY P0^T + dA K,   dK = Y dE'^T + V dP'^T + dA^T Q,   dV = K dP' + A^T dY,
// and the adjoints handed back dE = dE' + Q^T dO, dP = dP' + Q^T dY.  Unrolled over the chunks
// after c they are suffix sums, of the same shape as the second order's:
//     dE'(c) = sum_{m>c} Q_m^T dO_m,   dP'(c) = sum_{m>c} (U_m + M_m dE'(m)),
//     U_m = Q_m^T (A_m^T dO_m),   M_m = Q_m^T K_m
// (slot layout [Y = Q^T dO | U | M]; the cross term without the transpose).
// ===========================================================================
template <int D, typename TIn>
__global__ void __launch_bounds__(NT) k_abwd_chunk(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                   const float* __restrict__ dout, int T, int NCp,
                                                   float* __restrict__ bw) {
    constexpr int LD = Dim<D>::LD;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    extern __shared__ float sm[];
    float* Qs = sm;
    float* Ks = Qs + C * LD;
    float* Os = Ks + C * LD;                  // dO
    float* Gs = Os + C * LD;                  // A^T dO
    float* As = Gs + C * LD;                  // C x LDC
    const size_t head = (size_t)bh * T * D;
    const int t0 = chunk * C;
    load_rows<D>(Qs, q + head, t0, T);
    load_rows<D>(Ks, k + head, t0, T);
    load_rows<D>(Os, dout + head, t0, T);
    __syncthreads();
    float* out = bw + ((size_t)bh * NCp + chunk) * Bwd<D>::SIZE;
    mm<C, C, D>(Tile{Qs, LD}, TileT{Ks, LD}, Zero{}, PutMasked{As, LDC});                          // A
    mm<D, D, C>(TileT{Qs, LD}, Tile{Os, LD}, Zero{}, [&](int r, int c, float x) { out[r * D + c] = x; });      // Y
    mm<D, D, C>(TileT{Qs, LD}, Tile{Ks, LD}, Zero{},
                [&](int r, int c, float x) { out[2 * D * D + r * D + c] = x; });                   // M
    __syncthreads();
    mm<C, D, C>(TileT{As, LDC}, Tile{Os, LD}, Zero{}, Put{Gs, LD});                                 // A^T dO
    __syncthreads();
    mm<D, D, C>(TileT{Qs, LD}, Tile{Gs, LD}, Zero{},
                [&](int r, int c, float x) { out[D * D + r * D + c] = x; });                       // U
}

template <int D, typename TIn>
__global__ void __launch_bounds__(NT) k_abwd_out(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                 const TIn* __restrict__ v, const float* __restrict__ dout,
                                                 int T, int NCp, const float* __restrict__ sums,
                                                 const float* __restrict__ bw, float* __restrict__ dq,
                                                 float* __restrict__ dk, float* __restrict__ dv) {
    using S = Sum<OP_AHLA, D>;
    constexpr int LD = Dim<D>::LD;
    const int chunk = blockIdx.x, bh = blockIdx.y;
    const float* pre = sums + ((size_t)bh * NCp + chunk) * S::SIZE;          // P0 = mat(0), E0 = mat(1)
    const float* adj = bw + ((size_t)bh * NCp + chunk) * Bwd<D>::SIZE;       // dE' = 0, dP' = 1
    extern __shared__ float sm[];
    float* Qs = sm;
    float* Ks = Qs + C * LD;
    float* Vs = Ks + C * LD;
    float* Os = Vs + C * LD;                  // dO
    float* Ys = Os + C * LD;                  // Y
    float* dYs = Ys + C * LD;                 // dY
    float* As = dYs + C * LD;                 // C x LDC: A
    float* dAs = As + C * LDC;                // dA
    float* P0 = dAs + C * LDC;                // D x LD
    float* E0 = P0 + D * LD;
    float* dP = E0 + D * LD;
    float* dE = dP + D * LD;
    const size_t head = (size_t)bh * T * D;
    const int t0 = chunk * C;
    load_rows<D>(Qs, q + head, t0, T);
    load_rows<D>(Ks, k + head, t0, T);
    load_rows<D>(Vs, v + head, t0, T);
    load_rows<D>(Os, dout + head, t0, T);
    load_mats<D, 4>({P0, E0, dE, dP}, {pre + S::mat(0), pre + S::mat(1), adj, adj + D * D});
    __syncthreads();
    mm<C, C, D>(Tile{Qs, LD}, TileT{Ks, LD}, Zero{}, PutMasked{As, LDC});                          // A
    __syncthreads();
    mm2<C, D, D, C>(Tile{Qs, LD}, Tile{P0, LD}, Tile{As, LDC}, Tile{Vs, LD}, Zero{}, Put{Ys, LD});   // Y
    mm2<C, D, C, D>(TileT{As, LDC}, Tile{Os, LD}, Tile{Ks, LD}, Tile{dE, LD}, Zero{}, Put{dYs, LD}); // dY
    __syncthreads();
    // dA = L (.) (dO Y^T + dY V^T);  dV = K dP' + A^T dY
    mm2<C, C, D, D>(Tile{Os, LD}, TileT{Ys, LD}, Tile{dYs, LD}, TileT{Vs, LD}, Zero{}, PutMasked{dAs, LDC});
    mm2<C, D, D, C>(Tile{Ks, LD}, Tile{dP, LD}, TileT{As, LDC}, Tile{dYs, LD}, Zero{},
                    [&](int r, int c, float x) { if (t0 + r < T) dv[head + (size_t)(t0 + r) * D + c] = x; });
    __syncthreads();
    // dQ = dO E0^T + dY P0^T + dA K;  dK = Y dE'^T + V dP'^T + dA^T Q
    mm3<C, D, D, D, C>(Tile{Os, LD}, TileT{E0, LD}, Tile{dYs, LD}, TileT{P0, LD}, Tile{dAs, LDC}, Tile{Ks, LD},
                       Zero{}, [&](int r, int c, float x) { if (t0 + r < T) dq[head + (size_t)(t0 + r) * D + c] = x; });
    mm3<C, D, D, D, C>(Tile{Ys, LD}, TileT{dE, LD}, Tile{Vs, LD}, TileT{dP, LD}, TileT{dAs, LDC}, Tile{Qs, LD},
                       Zero{}, [&](int r, int c, float x) { if (t0 + r < T) dk[head + (size_t)(t0 + r) * D + c] = x; });
}

template <int D>
static size_t abwd_chunk_smem() {
    return sizeof(float) * (size_t)(4 * C * Dim<D>::LD + C * LDC);
}
template <int D>
static size_t abwd_out_smem() {
    return sizeof(float) * (size_t)(6 * C * Dim<D>::LD + 2 * C * LDC + 4 * D * Dim<D>::LD);
}

size_t ahla_backward_workspace_floats(int d, int BH, int T) {
    const int NCp = next_pow2((T + C - 1) / C);
    return workspace_floats(OP_AHLA, d, BH, T) + (size_t)BH * NCp * 3 * d * d;
}

int ahla_backward_launches(int d, int T) {
    // summaries, the scan, chunk terms, two suffix sums, cross term, gradients
    return kernel_launches(OP_AHLA, false, true, d, T) - 1 + 5;
}

template <int D, typename TIn>
static cudaError_t ahla_backward_run(const void* q, const void* k, const void* v, const float* dout, float* dq,
                                     float* dk, float* dv, int BH, int T, float* ws, cudaStream_t st) {
    const int NC = (T + C - 1) / C;
    const int NCp = next_pow2(NC);
    float* sums = ws;
    float* bw = ws + workspace_floats(OP_AHLA, D, BH, T);
    auto ks = k_summary<OP_AHLA, D, TIn>;
    auto kc = k_abwd_chunk<D, TIn>;
    auto ko = k_abwd_out<D, TIn>;
    const size_t s1 = summary_smem<D>(), s2 = abwd_chunk_smem<D>(), s3 = abwd_out_smem<D>();
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ko, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3)) != cudaSuccess) return e;
    // the forward's carried states: chunk summaries, then their exclusive scan
    ks<<<dim3(NCp, BH), NT, s1, st>>>((const TIn*)q, (const TIn*)k, (const TIn*)v, nullptr, 1, T, NC, NCp, sums);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (fold_fits<OP_AHLA, D>()) {
        auto kf = k_scan_fold<OP_AHLA, D>;
        if ((e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)fold_smem<OP_AHLA, D>())) != cudaSuccess)
            return e;
        kf<<<BH, NT, fold_smem<OP_AHLA, D>(), st>>>(sums, NC, NCp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else if ((e = scan_levels<OP_AHLA, D>(sums, NCp, BH, st)) != cudaSuccess) {
        return e;
    }
    kc<<<dim3(NC, BH), NT, s2, st>>>((const TIn*)q, (const TIn*)k, dout, T, NCp, bw);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 sg((D * D + NT - 1) / NT, BH);
    k_bwd_suffix<D><<<sg, NT, 0, st>>>(bw, NC, NCp, 0);                       // dE'
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_cross<D><<<dim3(NC, BH), NT, 0, st>>>(bw, NCp, 0);                   // X = U + M dE'
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_suffix<D><<<sg, NT, 0, st>>>(bw, NC, NCp, 1);                       // dP'
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ko<<<dim3(NC, BH), NT, s3, st>>>((const TIn*)q, (const TIn*)k, (const TIn*)v, dout, T, NCp, sums, bw, dq, dk,
                                     dv);
    return cudaGetLastError();
}

cudaError_t ahla_backward(bool bf16, int d, const void* q, const void* k, const void* v, const float* dout, float* dq,
                          float* dk, float* dv, int BH, int T, float* ws, cudaStream_t st) {
    if (bf16) {
        if (d == 32) return ahla_backward_run<32, __nv_bfloat16>(q, k, v, dout, dq, dk, dv, BH, T, ws, st);
        return ahla_backward_run<64, __nv_bfloat16>(q, k, v, dout, dq, dk, dv, BH, T, ws, st);
    }
    if (d == 32) return ahla_backward_run<32, float>(q, k, v, dout, dq, dk, dv, BH, T, ws, st);
    return ahla_backward_run<64, float>(q, k, v, dout, dq, dk, dv, BH, T, ws, st);
}

cudaError_t backward(bool bf16, int d, const void* q, const void* k, const void* v, const float* dout, float* dq,
                     float* dk, float* dv, int BH, int T, float* ws, int* status, cudaStream_t st, bool fp32_only) {
    if (bf16) {
        if (d == 32) return backward_run<32, __nv_bfloat16>(q, k, v, dout, dq, dk, dv, BH, T, ws, status, true, st);
        return backward_run<64, __nv_bfloat16>(q, k, v, dout, dq, dk, dv, BH, T, ws, status, fp32_only, st);
    }
    if (d == 32) return backward_run<32, float>(q, k, v, dout, dq, dk, dv, BH, T, ws, status, true, st);
    return backward_run<64, float>(q, k, v, dout, dq, dk, dv, BH, T, ws, status, true, st);
}

}  // namespace simt
}  // namespace hla
