// tcgen05 layout self-check: one bf16 MMA (M = 128) with K-major / MN-major operands in
// 128-byte-swizzled shared memory, accumulator read back through tcgen05.ld.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tc.h"

namespace hla {
namespace tc {

using bf16 = __nv_bfloat16;

// Place element (row r of the operand's M/N extent, column kk along K) of an R x K operand.
__device__ __forceinline__ uint32_t operand_offset(bool mn_major, int R, int K, int r, int kk) {
    if (!mn_major) return static_cast<uint32_t>((kk / 64) * (R * 128)) + ptx::sw128_offset(r, kk % 64);
    return static_cast<uint32_t>((r / 64) * (K * 128)) + ptx::sw128_offset(kk, r % 64);
}

// Descriptor of K-step s (16 elements) of an R x K operand.
__device__ __forceinline__ uint64_t operand_desc(bool mn_major, uint32_t base, int R, int K, int s) {
    if (!mn_major) return ptx::desc_sw128(base + (s / 4) * (R * 128) + (s % 4) * 32, 16, 1024);
    return ptx::desc_sw128(base + s * 2048, K * 128, 1024);
}

__global__ void __launch_bounds__(128) k_selftest(int cs, const bf16* __restrict__ a, const bf16* __restrict__ b,
                                                   float* __restrict__ d, int N, int K) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int M = (cs & 4) ? 64 : 128;          // bit 2: M = 64 (half-lane-quadrant accumulator)
    const int loff = (cs & 8) ? 16 : 0;         // bit 3: accumulator at TMEM lane offset 16
    const bool a_tm = (cs & 16) != 0;           // bit 4: A read from tensor memory (M = 128, K-major)
    const bool a_mn = (cs & 2) != 0, b_mn = (cs & 1) != 0;
    uint8_t* As = smem;
    uint8_t* Bs = smem + M * K * 2;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    for (int e = tid; e < M * K; e += blockDim.x) {
        int r, kk;
        if (!a_mn) { r = e / K; kk = e % K; } else { kk = e / M; r = e % M; }
        const bf16 x = a_mn ? a[kk * M + r] : a[r * K + kk];
        *reinterpret_cast<bf16*>(As + operand_offset(a_mn, M, K, r, kk)) = x;
    }
    for (int e = tid; e < N * K; e += blockDim.x) {
        int r, kk;
        if (!b_mn) { r = e / K; kk = e % K; } else { kk = e / N; r = e % N; }
        const bf16 x = b_mn ? b[kk * N + r] : b[r * K + kk];
        *reinterpret_cast<bf16*>(Bs + operand_offset(b_mn, N, K, r, kk)) = x;
    }
    ptx::fence_proxy_async();
    if (warp == 0) {
        ptx::tmem_alloc(&tmem_base, 512);
        ptx::tmem_relinquish();
    }
    if (tid == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tbase = tmem_base;
    constexpr uint32_t kAcol = 256;             // A's columns when it is read from tensor memory
    if (a_tm) {
        // row m = lane m: K bf16 values packed two per column from column kAcol on
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t r[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int kk = 2 * (c0 + i);
                const float lo = __bfloat162float(a[m * K + kk]), hi = __bfloat162float(a[m * K + kk + 1]);
                r[i] = ptx::pack_bf16(lo, hi);
            }
            ptx::tmem_st16u(tbase + (static_cast<uint32_t>(warp * 32) << 16) + kAcol + c0, r);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
    }
    if (tid == 0) {
        const uint32_t idesc = ptx::idesc_bf16(M, N, a_mn, b_mn);
        const uint32_t abase = ptx::smem_u32(As), bbase = ptx::smem_u32(Bs);
        const uint32_t dt = tbase + (static_cast<uint32_t>(loff) << 16);
        for (int s = 0; s < K / 16; ++s) {
            if (a_tm)
                ptx::umma_bf16_ts(dt, tbase + kAcol + 8 * s, operand_desc(b_mn, bbase, N, K, s), idesc, s > 0);
            else
                ptx::umma_bf16(dt, operand_desc(a_mn, abase, M, K, s), operand_desc(b_mn, bbase, N, K, s), idesc,
                               s > 0);
        }
        ptx::umma_commit(&bar);
    }
    bool ok = ptx::mbar_wait(&bar, 0);
    if (!ok) ok = ptx::mbar_wait(&bar, 0);  // second bounded wait before touching TMEM
    ptx::tc_fence_after();
    const uint32_t taddr = tbase + (static_cast<uint32_t>(warp * 32) << 16);
    // M = 128: row m in lane m.  M = 64: row m in lane (m % 16) + 32 (m / 16) + loff.
    int m = -1;
    if (M == 128) m = warp * 32 + lane;
    else if (lane >= loff && lane < loff + 16) m = warp * 16 + (lane - loff);
    for (int col = 0; col < N; col += 16) {
        float v[16];
        ptx::tmem_ld16(taddr + col, v);
        if (m >= 0)
            for (int i = 0; i < 16; ++i) d[m * N + col + i] = ok ? v[i] : __int_as_float(0x7fc00000);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) ptx::tmem_dealloc(tbase, 512);
}

// A bounded wait that runs out on purpose: an mbarrier nothing arrives on, waited on with the
// same helper the walkers use.  On the timeout the kernel records DEV_TIMEOUT in the status
// word and frees its TMEM, exactly as the walkers' error path does, then returns normally.
__global__ void __launch_bounds__(64) k_wait_timeout(int* status, unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        ptx::tmem_alloc(&tmem_base, 32);
        ptx::tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    bool ok = true;
    if (threadIdx.x == 0) ok = ptx::mbar_wait(&bar, 0, timeout_ns);
    ok = __syncthreads_and(ok) != 0;
    if (!ok && threadIdx.x == 0) set_status(status, DEV_TIMEOUT);
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) ptx::tmem_dealloc(tmem_base, 32);
}

cudaError_t selftest_wait_timeout(int* status, unsigned timeout_us, cudaStream_t st) {
    k_wait_timeout<<<1, 64, 0, st>>>(status, static_cast<unsigned long long>(timeout_us) * 1000ull);
    return cudaGetLastError();
}

cudaError_t selftest(int layout_case, const void* a, const void* b, float* d, int N, int K, cudaStream_t st) {
    const int smem = 128 * K * 2 + N * K * 2 + 1024;   // A sized for M = 128 in every case
    cudaError_t e = cudaFuncSetAttribute(k_selftest, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_selftest<<<1, 128, smem, st>>>(layout_case, static_cast<const bf16*>(a), static_cast<const bf16*>(b), d, N, K);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace hla
