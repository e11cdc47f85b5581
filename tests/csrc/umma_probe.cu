// umma_probe.cu -- test-only kernels that check the shared-memory layout and
// descriptor conventions of gdn_sm100.cuh against a plain matrix product:
// D[M x N] = (+/-) A[M x K] B[K x N], fp16 in, fp32 out, one tcgen05.mma chain.
// umma_probe_ta takes A from tensor memory instead of shared memory.
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

// A operand in tensor memory: row m of A sits in TMEM lane lane_of(m), and its K values are
// packed two fp16 per 32-bit column (even k in the low half), K / 2 columns from column 256.
// row_map = 0: lane = m; row_map = 1 (M = 64): lane = (m % 16) + 32 * (m / 16).
__global__ void probe_ta_kernel(const __half* A, const __half* B, float* D, int M, int N, int K,
                                int b_mn, int b_order, int row_map, int* err) {
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    unsigned char* sB = sm;
    uint32_t lbo_b, sbo_b;
    strides(N, K, b_order, lbo_b, sbo_b);
    for (int idx = threadIdx.x; idx < K * N; idx += blockDim.x) {
        int k = idx / N, n = idx % N;
        uint32_t off = b_mn ? off_mnmajor(n, k, sbo_b, lbo_b) : off_kmajor(n, k, sbo_b, lbo_b);
        *reinterpret_cast<__half*>(sB + off) = B[idx];
    }
    fence_async_smem();
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
    if (warp == 0) { tmem_alloc(&tbase, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = tbase;
    const uint32_t tA = t0 + 256;
    const uint32_t lanebase = (uint32_t)(32 * warp) << 16;
    {   // this thread's TMEM lane holds row m of A (or zeros)
        int m = -1;
        if (row_map == 0) m = 32 * warp + lane < M ? 32 * warp + lane : -1;
        else if (lane < 16) m = 16 * warp + lane;
        for (int c0 = 0; c0 < 64; c0 += 32) {
            float v[32];
            for (int j = 0; j < 32; ++j) {
                const int c = c0 + j;
                uint32_t w = 0;
                if (m >= 0 && 2 * c + 1 < K + 1 && 2 * c < K) {
                    const __half lo = A[m * K + 2 * c];
                    const __half hi = A[m * K + 2 * c + 1];
                    w = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
                }
                v[j] = __uint_as_float(w);
            }
            tmem_st32(tA + lanebase + c0, v);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
        const uint32_t id = idesc_f16(M, N, false, b_mn, false);
        for (int kk = 0; kk < K / 16; ++kk) {
            const uint64_t b = sdesc(smem_u32(sB) + kk * 2 * lbo_b, lbo_b, sbo_b);
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(t0),
                "r"(tA + 8u * kk), "l"(b), "r"((uint32_t)(kk > 0)), "r"(id)
                : "memory");
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    if (!ok && lane == 0) atomicExch(err, 4);
    tc_fence_after();
    if (ok) {
        for (int c0 = 0; c0 < N; c0 += 32) {
            float v[32];
            tmem_ld32(t0 + lanebase + c0, v);
            int row = -1;
            if (M == 128) row = 32 * warp + lane;
            else if (lane < 16) row = 16 * warp + lane;
            if (row >= 0)
                for (int j = 0; j < 32 && c0 + j < N; ++j) D[row * N + c0 + j] = v[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t0, 512);
}

extern "C" int umma_probe_ta(const void* A, const void* B, float* D, int M, int N, int K, int b_mn,
                             int b_order, int row_map, int* err) {
    if ((M != 64 && M != 128) || N % 32 || N > 256 || K % 16 || K > 128) return 1;
    if (row_map == 1 && M != 64) return 1;
    size_t smem = 200 * 1024;
    cudaFuncSetAttribute(probe_ta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    probe_ta_kernel<<<1, 128, smem>>>(static_cast<const __half*>(A), static_cast<const __half*>(B), D, M,
                                      N, K, b_mn, b_order, row_map, err);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

// 128-byte-swizzled operands (the layout a TMA load with SWIZZLE_128B writes; sw128_off and
// sdesc_sw128 of gdn_sm100.cuh): boxes of 64-element rows, `rows * 128` bytes apart.
// a_mn = 0: A stored K-major as a [M][K] tile; a_mn = 1: A stored MN-major as a [K][M] tile.
// Same for B ([N][K] or [K][N]).  K-major steps: +32 bytes inside a box, the next box at
// k = 64.  MN-major steps: two 8-row groups (+2048 bytes) per K = 16; LBO = the box stride.
__global__ void probe_sw_kernel(const __half* A, const __half* B, float* D, int M, int N, int K, int a_mn,
                                int b_mn, int* err) {
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    // swizzled boxes must start on a 1024-byte boundary of the shared window
    unsigned char* sA = sm + ((1024u - (smem_u32(sm) & 1023u)) & 1023u);
    unsigned char* sB = sA + 32768;
    for (int idx = threadIdx.x; idx < M * K; idx += blockDim.x) {
        const int m = idx / K, k = idx % K;
        const uint32_t off = a_mn ? sw128_off(k, m, K * 128) : sw128_off(m, k, M * 128);
        *reinterpret_cast<__half*>(sA + off) = A[idx];
    }
    for (int idx = threadIdx.x; idx < K * N; idx += blockDim.x) {
        const int k = idx / N, n = idx % N;
        const uint32_t off = b_mn ? sw128_off(k, n, K * 128) : sw128_off(n, k, N * 128);
        *reinterpret_cast<__half*>(sB + off) = B[idx];
    }
    fence_async_smem();
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
    if (warp == 0) { tmem_alloc(&tbase, 256); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = tbase;
    if (threadIdx.x == 0) {
        const uint32_t id = idesc_f16(M, N, a_mn, b_mn, false);
        for (int kk = 0; kk < K / 16; ++kk) {
            const int k0 = 16 * kk;
            uint64_t a, b;
            if (a_mn) a = sdesc_sw128(smem_u32(sA) + (k0 / 8) * 1024, (uint32_t)(K * 128), 1024);
            else      a = sdesc_sw128(smem_u32(sA) + (k0 / 64) * M * 128 + (k0 % 64) * 2, 16, 1024);
            if (b_mn) b = sdesc_sw128(smem_u32(sB) + (k0 / 8) * 1024, (uint32_t)(K * 128), 1024);
            else      b = sdesc_sw128(smem_u32(sB) + (k0 / 64) * N * 128 + (k0 % 64) * 2, 16, 1024);
            mma_f16(t0, a, b, id, kk > 0);
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    if (!ok && lane == 0) atomicExch(err, 4);
    tc_fence_after();
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
    if (warp == 0) tmem_dealloc(t0, 256);
}

extern "C" int umma_probe_sw(const void* A, const void* B, float* D, int M, int N, int K, int a_mn,
                             int b_mn, int* err) {
    if ((M != 64 && M != 128) || N % 64 || N > 128 || K % 64 || K > 128) return 1;
    // 128 KB: the operands use 64 KB; the rest keeps every address in bounds even if a
    // descriptor stride were read with the LBO/SBO roles exchanged.
    size_t smem = 131072 + 1024;
    cudaFuncSetAttribute(probe_sw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    probe_sw_kernel<<<1, 128, smem>>>(static_cast<const __half*>(A), static_cast<const __half*>(B), D, M, N,
                                      K, a_mn, b_mn, err);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

// A operand copied from shared memory into tensor memory with tcgen05.cp (shape 128x256b: 128
// lanes x 8 columns, i.e. one K step of 16 fp16 for 128 rows), from the K-major canonical
// layout (8-row x 16-byte core matrices, LBO between K groups, SBO between row groups), then
// the product with A from tensor memory.  Rows m >= M of the copied tile are padding.
__global__ void probe_cp_kernel(const __half* A, const __half* B, float* D, int M, int N, int K, int b_mn,
                                int* err) {
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    unsigned char* sA = sm;                 // 128 rows x K, K-major, LBO 128, SBO (K / 8) * 128
    unsigned char* sB = sm + 128 * 128 * 2;
    const uint32_t lbo_a = 128, sbo_a = (uint32_t)(K / 8) * 128;
    uint32_t lbo_b, sbo_b;
    strides(N, K, 0, lbo_b, sbo_b);
    for (int idx = threadIdx.x; idx < 128 * K; idx += blockDim.x) {
        const int m = idx / K, k = idx % K;
        *reinterpret_cast<__half*>(sA + off_kmajor(m, k, sbo_a, lbo_a)) = m < M ? A[m * K + k] : __float2half(0.f);
    }
    for (int idx = threadIdx.x; idx < K * N; idx += blockDim.x) {
        const int k = idx / N, n = idx % N;
        uint32_t off = b_mn ? off_mnmajor(n, k, sbo_b, lbo_b) : off_kmajor(n, k, sbo_b, lbo_b);
        *reinterpret_cast<__half*>(sB + off) = B[idx];
    }
    fence_async_smem();
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
    if (warp == 0) { tmem_alloc(&tbase, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = tbase;
    const uint32_t tA = t0 + 256;
    if (threadIdx.x == 0) {
        for (int kk = 0; kk < K / 16; ++kk) {
            const uint64_t s = sdesc(smem_u32(sA) + kk * 2 * lbo_a, lbo_a, sbo_a);
            asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(tA + 8u * kk), "l"(s) : "memory");
        }
        const uint32_t id = idesc_f16(M == 64 ? 128 : M, N, false, b_mn, false);
        for (int kk = 0; kk < K / 16; ++kk) {
            const uint64_t b = sdesc(smem_u32(sB) + kk * 2 * lbo_b, lbo_b, sbo_b);
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(t0),
                "r"(tA + 8u * kk), "l"(b), "r"((uint32_t)(kk > 0)), "r"(id)
                : "memory");
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    if (!ok && lane == 0) atomicExch(err, 4);
    tc_fence_after();
    if (ok) {
        for (int c0 = 0; c0 < N; c0 += 32) {
            float v[32];
            tmem_ld32(t0 + ((uint32_t)(32 * warp) << 16) + c0, v);
            const int row = 32 * warp + lane;       // an M = 128 product: row m in lane m
            if (row < M)
                for (int j = 0; j < 32 && c0 + j < N; ++j) D[row * N + c0 + j] = v[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t0, 512);
}

extern "C" int umma_probe_cp(const void* A, const void* B, float* D, int M, int N, int K, int b_mn, int* err) {
    if ((M != 64 && M != 128) || N % 32 || N > 256 || K % 16 || K > 128) return 1;
    size_t smem = 200 * 1024;
    cudaFuncSetAttribute(probe_cp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    probe_cp_kernel<<<1, 128, smem>>>(static_cast<const __half*>(A), static_cast<const __half*>(B), D, M, N, K,
                                      b_mn, err);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
