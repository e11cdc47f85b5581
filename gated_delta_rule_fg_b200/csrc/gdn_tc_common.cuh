// gdn_tc_common.cuh -- constants and helpers shared by the tensor-core kernels (bf16, chunk 64,
// dk = dv = 128): the layout of the per-(head, chunk) block that the intra role writes and the
// scan role reads, and small conversion / store helpers.
#pragma once
#include "gdn_common.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace tc {
using namespace sm100;

constexpr int C = 64;          // chunk
constexpr int D = 128;         // dk = dv
constexpr int NT = 256;        // intra threads
constexpr int NS = 32;         // scan: columns per CTA
constexpr int J = D / NS;      // scan: slices per head
constexpr float kMaxHalfSpan = 6.0f;

// Per (head, chunk) block in the workspace (bytes), written by the intra kernel and read
// by the scan kernel.  "sw" rows: 32 fp16 per row, the four 16-byte groups of row x are
// stored in the order g ^ ((x >> 1) & 3), so eight consecutive rows read as 16-byte
// vectors hit eight different bank groups.
constexpr uint32_t kOffN = 0;            // N = -K'^T W, fp16 128x128, K-major (m=i, k=c): SBO 2048, LBO 128
constexpr uint32_t kOffQe = 32768;       // Qe fp16 64x128 (m=r, k=c), SBO 2048, LBO 128: MN-major from intra_tc_kernel, K-major from the TMA-fed intra kernel
constexpr uint32_t kOffB = 49152;        // b = K'^T U', fp16 [J][128][NS]: sw rows from intra_tc_kernel,
                                         //   [J][NS / 8][128][8] from the TMA-fed intra kernel
constexpr uint32_t kOffPU = 81920;       // PU', fp16 [J][64][NS]: sw rows / [J][NS / 8][64][8], the same way
constexpr uint32_t kOffGC = 98304;       // e^{g_last}, fp32 [128]
constexpr uint32_t kOffKp = 98816;       // K' fp16 (m=i, k=r), MN-major SBO 1024 LBO 128 (intra's own scratch)
constexpr uint32_t kBlockBytes = 115200;
// Fallback chunks (element-wise A and P) stage q^ (fp16) in the N area, k~ (fp16) in the
// PU' area and g (fp32) in the b area; those areas are written only afterwards.

__host__ __device__ __forceinline__ uint32_t sw_half(uint32_t row, uint32_t j) {
    return row * NS + 8u * (((j >> 3) ^ ((row >> 1) & 3u))) + (j & 7u);
}

// Group-major slice of `nrows` rows x 32 fp16: the 16-byte groups (8 columns) of consecutive rows
// are consecutive, so a warp whose lanes hold consecutive rows stores and loads 512 contiguous
// bytes per group (whole 32-byte sectors in L2, no bank conflicts in shared memory).
__host__ __device__ __forceinline__ uint32_t grp_half(uint32_t row, uint32_t j, uint32_t nrows) {
    return ((j >> 3) * nrows + row) * 8u + (j & 7u);
}

// swizzled fp32 64x64: element (r, i)
__device__ __forceinline__ int sw64(int r, int i) { return r * 64 + ((((i >> 2) ^ (r & 15))) << 2) + (i & 3); }

// sqrt(x) for x >= 0 as x * rsqrt(x): a few ulp in fp32, far below the fp16 rounding of the
// operands it scales, and shorter than the IEEE-rounded square root (x = 0 gives 0).
__device__ __forceinline__ float sqrt_op(float x) { return x > 0.f ? x * rsqrtf(x) : 0.f; }

__device__ __forceinline__ uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ float4 ldg16f(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }

__device__ __forceinline__ void bf8_to_f(const uint4 u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void h8_to_f(const uint4 u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ uint4 f_to_h8(const float* f) {
    uint4 u;
    __half2 h0 = __floats2half2_rn(f[0], f[1]);
    __half2 h1 = __floats2half2_rn(f[2], f[3]);
    __half2 h2 = __floats2half2_rn(f[4], f[5]);
    __half2 h3 = __floats2half2_rn(f[6], f[7]);
    u.x = *reinterpret_cast<uint32_t*>(&h0);
    u.y = *reinterpret_cast<uint32_t*>(&h1);
    u.z = *reinterpret_cast<uint32_t*>(&h2);
    u.w = *reinterpret_cast<uint32_t*>(&h3);
    return u;
}

__device__ __forceinline__ void st16(uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
}

__device__ __forceinline__ void record_timeout(int* status) {
    atomicCAS(status, kDevOk, kDevTimeout);
}

}  // namespace tc
}  // namespace gdn
