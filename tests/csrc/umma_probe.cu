// umma_probe.cu -- test-only kernel that checks the shared-memory layout and
// descriptor conventions of gdn_sm100.cuh against a plain matrix product:
// D[M x N] = (+/-) A[M x K] B[K x N], fp16 in, fp32 out, one tcgen05.mma chain.
#include <cuda_fp16.h>
#include "../../gated_delta_rule_fg_b200/csrc/gdn_sm100.cuh"

using namespace gdn::sm100;

// order = 0: the K-groups of one M/N 8-group are adjacent (LBO = 128 B);
// order = 1: the M/N 8-groups are adjacent (SBO = 128 B).
__device__ void strides(int mn_extent, int k_extent, int order, uint32_t& lbo, uint32_t& sbo) {
    if (order == 0) { lbo = 128; sbo = (k_extent / 8) * 128; }
    else            { sbo = 128; lbo = (mn_extent / 8) * 128; }
}

__global__ void probe_kernel(const __half* A, const __half* B, float* D, int M, int N, int K,
                             int a_mn, int b_mn, int a_order, int b_order, int a_neg, int* err) {
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    unsigned char* sA = sm;
    unsigned char* sB = sm + 128 * 128 * 2;
    uint32_t lbo_a, sbo_a, lbo_b, sbo_b;
    strides(M, K, a_order, lbo_a, sbo_a);
    strides(N, K, b_order, lbo_b, sbo_b);
    for (int idx = threadIdx.x; idx < M * K; idx += blockDim.x) {
        int m = idx / K, k = idx % K;
        uint32_t off = a_mn ? off_mnmajor(m, k, sbo_a, lbo_a) : off_kmajor(m, k, sbo_a, lbo_a);
        *reinterpret_cast<__half*>(sA + off) = A[idx];
    }
    for (int idx = threadIdx.x; idx < K * N; idx += blockDim.x) {
        int k = idx / N, n = idx % N;
        uint32_t off = b_mn ? off_mnmajor(n, k, sbo_b, lbo_b) : off_kmajor(n, k, sbo_b, lbo_b);
        *reinterpret_cast<__half*>(sB + off) = B[idx];
    }
    fence_async_smem();
    const int warp = threadIdx.x / 32;
    uint32_t ncols = N < 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));
    if (threadIdx.x == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
    if (warp == 0) { tmem_alloc(&tbase, ncols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = tbase;
    if (threadIdx.x == 0) {
        mma_f16_k(t0, smem_u32(sA), lbo_a, sbo_a, smem_u32(sB), lbo_b, sbo_b,
                  idesc_f16(M, N, a_mn, b_mn, a_neg), K, false);
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    if (!ok && (threadIdx.x & 31) == 0) atomicExch(err, 4);
    tc_fence_after();
    const int lane = threadIdx.x & 31;
    if (ok) {
        for (int c0 = 0; c0 < N; c0 += 32) {
            float v[32];
            tmem_ld32(t0 + ((uint32_t)(32 * warp) << 16) + c0, v);
            int row = -1;
            if (M == 128) row = 32 * warp + lane;
            else if (lane < 16) row = 16 * warp + lane;
            if (row >= 0)
                for (int j = 0; j < 32 && c0 + j < N; ++j) D[row * N + c0 + j] = v[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t0, ncols);
}

extern "C" int umma_probe(const void* A, const void* B, float* D, int M, int N, int K, int a_mn, int b_mn,
                          int a_order, int b_order, int a_neg, int* err) {
    if ((M != 64 && M != 128) || N % 32 || N > 256 || K % 16 || K > 128) return 1;
    // 200 KB: the operands use 96 KB; the rest keeps every address in bounds even if a
    // descriptor stride were read with the LBO/SBO roles exchanged.
    size_t smem = 200 * 1024;
    cudaFuncSetAttribute(probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    probe_kernel<<<1, 128, smem>>>(static_cast<const __half*>(A), static_cast<const __half*>(B), D, M, N, K,
                                   a_mn, b_mn, a_order, b_order, a_neg, err);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
