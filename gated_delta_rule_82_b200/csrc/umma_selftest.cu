// umma_selftest.cu -- one-CTA bf16 GEMM through the library's tcgen05 wrappers.
//
// Exercises exactly the pieces the chunked forward relies on: swizzled K-major and MN-major
// shared-memory tiles written by threads, the shared-memory and instruction descriptors,
// single-thread tcgen05.mma issue, tcgen05.commit to an mbarrier, and the TMEM read-back for
// both M = 128 (row m in lane m) and M = 64 (row m in lane (m % 16) + 32 (m / 16)).
#include "internal.cuh"
#include "tc_sm100.cuh"

namespace ckda {

namespace {

constexpr int kSelftestTmemCols = 512;   // D (N <= 256 columns) + A staged in TMEM (K / 2 columns)

__global__ void __launch_bounds__(128)
umma_selftest_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B,
                     float* __restrict__ D, int M, int N, int K, int b_mn, int a_tmem) {
    // a_tmem: 0 = A from shared memory; 1 = A copied into TMEM by tcgen05.cp; 2 = A written into
    // TMEM by the threads (tcgen05.st: row m in lane m, K elements 2j and 2j + 1 in column j)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;
    uint8_t* sB = base + (size_t)M * K * 2;
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < M * K; e += 128) {
        int m = e / K, kk = e % K;
        *reinterpret_cast<__nv_bfloat16*>(sA + tc::sw128_kmajor(m, kk, M)) = A[e];
    }
    if (!b_mn) {
        for (int e = tid; e < N * K; e += 128) {
            int n = e / K, kk = e % K;
            *reinterpret_cast<__nv_bfloat16*>(sB + tc::sw128_kmajor(n, kk, N)) = B[e];
        }
    } else {
        for (int e = tid; e < N * K; e += 128) {
            int kk = e / N, n = e % N;
            *reinterpret_cast<__nv_bfloat16*>(sB + tc::sw128_mnmajor(kk, n, K)) = B[e];
        }
    }
    tc::fence_proxy_async_smem();
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, kSelftestTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
        abort_flag = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tbase = tmem_base;

    if (!a_tmem && tid == 0) {
        const uint32_t idesc = tc::idesc_bf16_f32(M, N, 0, b_mn);
        const uint32_t a0 = tc::smem_u32(sA), b0 = tc::smem_u32(sB);
        for (int ks = 0; ks < K / 16; ++ks) {
            uint64_t ad = tc::smem_desc_sw128(a0 + (ks >> 2) * M * 128 + (ks & 3) * 32, 16, 1024);
            uint64_t bd = b_mn ? tc::smem_desc_sw128(b0 + ks * 2048, K * 128, 1024)
                               : tc::smem_desc_sw128(b0 + (ks >> 2) * N * 128 + (ks & 3) * 32, 16, 1024);
            tc::mma_bf16(tbase, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bar);
    }
    if (a_tmem == 2) {
        // thread (warp w, lane l) writes row 32 w + l of A, 64 K elements per 32-column store
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < K / 2; c0 += 32) {
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const uint16_t lo = __bfloat16_as_ushort(A[(size_t)m * K + 2 * (c0 + j)]);
                const uint16_t hi = __bfloat16_as_ushort(A[(size_t)m * K + 2 * (c0 + j) + 1]);
                v[j] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            tc::tmem_st32(tc::tmem_addr(tbase + 256, warp * 32, c0), v);
        }
        tc::tmem_st_wait();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
    }
    if (a_tmem && warp == 0) {
        // A (M = 128) in TMEM columns 256.. (K / 2 columns): copied there by tcgen05.cp, one
        // 16-element K-step per copy, unless the threads wrote it above
        const uint32_t idesc = tc::idesc_bf16_f32(M, N, 0, b_mn);
        const uint32_t a0 = tc::smem_u32(sA), b0 = tc::smem_u32(sB);
        const uint32_t ta = tbase + 256;
        if (a_tmem == 1)
            for (int ks = 0; ks < K / 16; ++ks)
                tc::tmem_cp_128x256b_warp(ta + ks * 8, tc::smem_desc_sw128(a0 + (ks >> 2) * M * 128 + (ks & 3) * 32, 16, 1024));
        for (int ks = 0; ks < K / 16; ++ks) {
            uint64_t bd = b_mn ? tc::smem_desc_sw128(b0 + ks * 2048, K * 128, 1024)
                               : tc::smem_desc_sw128(b0 + (ks >> 2) * N * 128 + (ks & 3) * 32, 16, 1024);
            tc::mma_bf16_tmem_a_warp(tbase, ta + ks * 8, bd, idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit_warp(&bar);
    }
    tc::mbar_wait(&bar, 0, &abort_flag);
    tc::tc_fence_after();

    int row = -1;
    if (M == 128) row = warp * 32 + lane;
    else if (lane < 16) row = warp * 16 + lane;
    for (int col = 0; col < N; col += 16) {
        float v[16];
        tc::tmem_ld16_sync(tc::tmem_addr(tbase, warp * 32, col), v);
        if (row >= 0 && !abort_flag) {
#pragma unroll
            for (int i = 0; i < 16; ++i) D[(size_t)row * N + col + i] = v[i];
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, kSelftestTmemCols);
}

}  // namespace

cudaError_t launch_umma_selftest(const void* A, const void* B, float* D, int M, int N, int K,
                                 int mode, cudaStream_t stream) {
    const int b_mn_major = mode & 1, a_tmem = (mode & 2) ? 1 : (mode & 4) ? 2 : 0;
    // an MN-major B occupies whole 128-byte rows: ceil(N / 64) blocks of K rows
    const size_t b_bytes = b_mn_major ? (size_t)((N + 63) / 64) * K * 128 : (size_t)N * K * 2;
    size_t smem = (size_t)M * K * 2 + b_bytes + 1024;
    cudaError_t e = cudaFuncSetAttribute(umma_selftest_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    umma_selftest_kernel<<<1, 128, smem, stream>>>(static_cast<const __nv_bfloat16*>(A),
                                                   static_cast<const __nv_bfloat16*>(B), D, M, N,
                                                   K, b_mn_major, a_tmem);
    return cudaGetLastError();
}

}  // namespace ckda
