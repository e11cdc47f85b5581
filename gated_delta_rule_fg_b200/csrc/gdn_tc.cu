// gdn_tc.cu -- tensor-core (tcgen05, fp16 operands, fp32 TMEM accumulators)
// kernels for the bf16 path with chunk 64 and dk = dv = 128.
//
// intra_tc_kernel: one CTA per (chunk, head), 256 threads, ~110 KB shared
// memory (two CTAs per SM).  It computes the S-independent quantities of one
// chunk (see gdn_common.cuh) and writes them in the operand layouts the scan
// consumes directly.  The decay factors of A and P are split around a
// per-channel reference g_ref = g_last / 2 (the middle of the chunk's
// log-decay range), A = (K~ e^{g-g_ref}) (K~ e^{g_ref-g})^T and likewise P, so
// both operands stay within e^{+-span/2}; chunks whose half-span exceeds
// kMaxHalfSpan form A and P element by element in fp32 instead.  With the same
// reference, W~ = T (K~ e^{g-g_ref}) = W e^{-g_ref} and
// Qe e^{-g_ref} = Q^ e^{g-g_ref} - P W~, so the scaled operands double as the
// inputs of the later products; the per-channel factor e^{g_ref} is put back in
// the epilogue.
//
// scan_tc_kernel: one CTA per (head, 32-column slice of d_v), serial over the
// chunks.  Per chunk: D1 = [W; Qe] S (one M = 128 MMA), U = U' - D1[0:64],
// O = PU' + D1[64:128]; D2 = K'^T U; S <- Diag(gC) S + D2.  S stays in fp32
// registers (one d_k row per thread); its fp16 copy is the MMA operand.
// A producer warp streams the per-chunk blocks with bulk async copies into a
// two-stage buffer.
#include "gdn_common.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
using namespace sm100;

namespace tc {

constexpr int C = 64;          // chunk
constexpr int D = 128;         // dk = dv
constexpr int NT = 256;        // intra threads
constexpr int NS = 32;         // scan: columns per CTA
constexpr int J = D / NS;      // scan: slices per head
constexpr float kMaxHalfSpan = 6.0f;

// Per (head, chunk) block in the workspace (bytes).
constexpr uint32_t kOffAS1 = 0;          // [W; Qe] fp16 128x128, MN-major (mn=row, k=channel), SBO 2048, LBO 128
constexpr uint32_t kOffAS2 = 32768;      // K'^T fp16 (mn=channel, k=row), MN-major, SBO 1024, LBO 128
constexpr uint32_t kOffUp = 49152;       // U'  fp32 [J][C][NS]
constexpr uint32_t kOffPUp = 81920;      // PU' fp32 [J][C][NS]
constexpr uint32_t kOffGC = 114688;      // e^{g_last} fp32 [D]
constexpr uint32_t kBlockBytes = 115200;

// intra shared memory map (bytes)
constexpr uint32_t kR0 = 0;              // [KG; QG] fp16 K-major (row, ch): SBO 2048, LBO 128  -> later W~^T (K-major (ch, row): SBO 128, LBO 2048)
constexpr uint32_t kR1 = 32768;          // KIG fp16 (row, ch) K-major SBO 2048 LBO 128 -> later A fp32 64x64 (swizzled)
constexpr uint32_t kR2 = 49152;          // V~ fp16 (row, ch) -> later U'^T fp16 (ch, row) K-major SBO 128 LBO 2048
constexpr uint32_t kR3 = 65536;          // T fp16, B operand (n=r, k=i) K-major SBO 1024 LBO 128
constexpr uint32_t kR4 = 73728;          // P fp16, same layout
constexpr uint32_t kR5 = 81920;          // identity fp16, same layout
constexpr uint32_t kR6 = 90112;          // T fp32 64x64 (swizzled)
constexpr uint32_t kScr = 106496;        // 4 KB: per-warp log-decay totals, later solve scratch
constexpr uint32_t kGref = 110592;       // g_ref [128]
constexpr uint32_t kFK = 111104;         // e^{g_last - g_ref} [128]
constexpr uint32_t kGlast = 111616;      // g_last [128]
constexpr uint32_t kBar = 112128;        // mbarrier
constexpr uint32_t kTmem = 112136;       // TMEM base address
constexpr uint32_t kIntraSmem = 112192;

constexpr uint32_t kTmemCols = 256;
// TMEM columns: D0 / D3 at 0, D1 (W~^T) at 64, D2 (U'^T) at 128, D4 (PU'^T) at 192.

// swizzled fp32 64x64: element (r, i)
__device__ __forceinline__ int sw64(int r, int i) { return r * 64 + ((((i >> 2) ^ (r & 15))) << 2) + (i & 3); }

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

// ============================================================================ intra
__global__ void __launch_bounds__(NT, 2) intra_tc_kernel(Problem p) {
    extern __shared__ __align__(1024) uint8_t sm[];
    const int c = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int s0 = c * C;
    const int Cv = min(C, p.L - s0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* blk = static_cast<uint8_t*>(p.inter) + ((size_t)bh * p.NC + c) * kBlockBytes;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kTmem);
    float* scr = reinterpret_cast<float*>(sm + kScr);
    float* gref = reinterpret_cast<float*>(sm + kGref);
    float* fK = reinterpret_cast<float*>(sm + kFK);
    float* glast = reinterpret_cast<float*>(sm + kGlast);
    float* A32 = reinterpret_cast<float*>(sm + kR1);
    float* T32 = reinterpret_cast<float*>(sm + kR6);

    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    // identity operand (B layout: n = r, k = i)
    for (int idx = tid; idx < 512; idx += NT) {
        const int r = idx >> 3, j = idx & 7;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = (8 * j + e == r) ? 1.f : 0.f;
        st16(sm + kR5, off_kmajor(r, 8 * j, 1024, 128), f_to_h8(f));
    }

    // ---------------------------------------------------------------- prep
    const int r = 8 * warp + (lane & 7);     // row of the chunk handled by this lane
    const int o0 = lane >> 3;                // channel octets o0, o0+4, o0+8, o0+12
    const bool valid = r < Cv;
    RowRef rr{};
    size_t krow = 0;
    if (valid) {
        rr = row_ref(p, b, h, s0 + r);
        krow = p.dp ? rr.tok * p.nh + rr.m : rr.tok;
    }
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q);
    const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(p.k);
    const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(p.v);
    uint4 qp[4], kp[4];
    float ssq = 0.f, ssk = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = o0 + 4 * j;
        qp[j] = (valid && rr.has_q) ? ldg16(q + rr.tok * D + 8 * o) : make_uint4(0, 0, 0, 0);
        kp[j] = valid ? ldg16(k + krow * D + 8 * o) : make_uint4(0, 0, 0, 0);
        float fq[8], fk[8];
        bf8_to_f(qp[j], fq);
        bf8_to_f(kp[j], fk);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            ssq += fq[e] * fq[e];
            ssk += fk[e] * fk[e];
        }
    }
    ssq += __shfl_xor_sync(0xffffffffu, ssq, 8);
    ssq += __shfl_xor_sync(0xffffffffu, ssq, 16);
    ssk += __shfl_xor_sync(0xffffffffu, ssk, 8);
    ssk += __shfl_xor_sync(0xffffffffu, ssk, 16);
    const float iq = rsqrtf(ssq + kNormEps);
    const float ik = rsqrtf(ssk + kNormEps);

    const bool a_scalar = p.dp || p.alpha_scalar;
    const bool b_scalar = p.dp || p.beta_scalar;
    float la_s = 0.f, b_s = 0.f;
    if (valid) {
        if (p.dp) {
            la_s = rr.m == 0 ? __logf(p.alpha[rr.tok]) : 0.f;
            b_s = p.beta[rr.tok * p.nh + rr.m];
        } else {
            if (p.alpha_scalar) la_s = __logf(p.alpha[rr.tok]);
            if (p.beta_scalar) b_s = p.beta[rr.tok];
        }
    }
    // log alpha, inclusive scan over the 8 rows of this warp (lanes with equal o0)
    float la[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = o0 + 4 * j;
        if (a_scalar || !valid) {
#pragma unroll
            for (int e = 0; e < 8; ++e) la[j][e] = valid ? la_s : 0.f;
        } else {
            const float4 a0 = ldg16f(p.alpha + rr.tok * D + 8 * o);
            const float4 a1 = ldg16f(p.alpha + rr.tok * D + 8 * o + 4);
            la[j][0] = __logf(a0.x); la[j][1] = __logf(a0.y); la[j][2] = __logf(a0.z); la[j][3] = __logf(a0.w);
            la[j][4] = __logf(a1.x); la[j][5] = __logf(a1.y); la[j][6] = __logf(a1.z); la[j][7] = __logf(a1.w);
        }
#pragma unroll
        for (int d = 1; d < 8; d <<= 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float y = __shfl_up_sync(0xffffffffu, la[j][e], d, 8);
                if ((lane & 7) >= d) la[j][e] += y;
            }
        }
        if ((lane & 7) == 7) {
#pragma unroll
            for (int e = 0; e < 8; ++e) scr[warp * D + 8 * o + e] = la[j][e];
        }
    }
    __syncthreads();
    if (tid < D) {   // exclusive prefix over the warps' row blocks, and the chunk total
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const float t = scr[w * D + tid];
            scr[w * D + tid] = acc;
            acc += t;
        }
        glast[tid] = acc;
    }
    __syncthreads();
    const bool wide = tid < D && (-0.5f * glast[tid] > kMaxHalfSpan);
    const int fallback = __syncthreads_or(wide);
    if (tid < D) {
        const float gr = fallback ? 0.f : 0.5f * glast[tid];
        gref[tid] = gr;
        fK[tid] = __expf(glast[tid] - gr);
        reinterpret_cast<float*>(blk + kOffGC)[tid] = __expf(glast[tid]);
    }
    __syncthreads();

    // per octet: the fp16 operands
    float* fb_g = reinterpret_cast<float*>(blk + kOffUp);                 // fallback scratch: g fp32 [C][D]
    __half* fb_k = reinterpret_cast<__half*>(blk + kOffPUp);              // k~ fp16 [C][D]
    __half* fb_q = reinterpret_cast<__half*>(blk + kOffPUp + C * D * 2);  // q^ fp16 [C][D]
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = o0 + 4 * j;
        float g[8], sb[8], fq[8], fk[8], fv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = la[j][e] + scr[warp * D + 8 * o + e];
        if (b_scalar || !valid) {
            const float s = valid ? sqrtf(b_s) : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) sb[e] = s;
        } else {
            const float4 b0 = ldg16f(p.beta + rr.tok * D + 8 * o);
            const float4 b1 = ldg16f(p.beta + rr.tok * D + 8 * o + 4);
            sb[0] = sqrtf(b0.x); sb[1] = sqrtf(b0.y); sb[2] = sqrtf(b0.z); sb[3] = sqrtf(b0.w);
            sb[4] = sqrtf(b1.x); sb[5] = sqrtf(b1.y); sb[6] = sqrtf(b1.z); sb[7] = sqrtf(b1.w);
        }
        const uint4 vp = valid ? ldg16(v + krow * D + 8 * o) : make_uint4(0, 0, 0, 0);
        bf8_to_f(qp[j], fq);
        bf8_to_f(kp[j], fk);
        bf8_to_f(vp, fv);
        float KG[8], QG[8], KIG[8], VT[8], KP[8], KT[8], QH[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int ch = 8 * o + e;
            const float gr = gref[ch];
            const float ex = __expf(g[e] - gr);
            const float exi = __expf(gr - g[e]);
            const float kt = fk[e] * ik * sb[e];
            const float qh = fq[e] * iq;
            KT[e] = kt;
            QH[e] = qh;
            KG[e] = kt * ex;
            QG[e] = qh * ex;
            KIG[e] = kt * exi;
            VT[e] = fv[e] * sb[e];
            // fallback chunks: e^{-g} may overflow while e^{g_last} underflows, so take the
            // ratio in one exponent there (it is <= 1)
            KP[e] = fallback ? kt * __expf(glast[ch] - g[e]) : kt * exi * fK[ch];
        }
        const uint32_t off = off_kmajor(r, 8 * o, 2048, 128);
        st16(sm + kR0, off, f_to_h8(KG));
        st16(sm + kR0, off_kmajor(64 + r, 8 * o, 2048, 128), f_to_h8(QG));
        st16(sm + kR1, off, f_to_h8(KIG));
        st16(sm + kR2, off, f_to_h8(VT));
        *reinterpret_cast<uint4*>(blk + kOffAS2 + off_mnmajor(8 * o, r, 1024, 128)) = f_to_h8(KP);
        if (fallback) {
#pragma unroll
            for (int e = 0; e < 8; ++e) fb_g[r * D + 8 * o + e] = g[e];
            *reinterpret_cast<uint4*>(fb_k + r * D + 8 * o) = f_to_h8(KT);
            *reinterpret_cast<uint4*>(fb_q + r * D + 8 * o) = f_to_h8(QH);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = *tslot;
    bool ok = true;
    uint32_t phase = 0;      // parity of the next completion of `bar`

    // ---------------------------------------------------------------- A and P
    if (!fallback) {
        if (tid == 0) {
            mma_f16_k(t0, smem_u32(sm + kR0), 128, 2048, smem_u32(sm + kR1), 128, 2048,
                      idesc_f16(128, 64, false, false), D, false);
            mma_commit(bar);
        }
        ok = mbar_wait(bar, phase);
        phase ^= 1u;
    } else if (warp < 4) {
        // exact fp32 Gram products, element by element (decay formed per pair of rows)
        const int rho = 32 * warp + lane;
        const int rowr = rho & 63;
        const bool isP = rho >= 64;
        for (int cb = 0; cb < 64; cb += 32) {
            float acc[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = 0.f;
            for (int ch = 0; ch < D; ++ch) {
                const float gr = fb_g[rowr * D + ch];
                const float xr = __half2float(isP ? fb_q[rowr * D + ch] : fb_k[rowr * D + ch]);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int col = cb + i;
                    if (col < rowr || (isP && col == rowr)) {
                        acc[i] += xr * __half2float(fb_k[col * D + ch]) * __expf(gr - fb_g[col * D + ch]);
                    }
                }
            }
            tmem_st32(t0 + ((uint32_t)(32 * warp) << 16) + cb, acc);
        }
        tc_fence_before();
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) record_timeout(p.status);
    tc_fence_after();

    if (ok && warp < 4) {   // A rows -> fp32 (swizzled), P rows -> fp16 B operand
        float d0[32], d1[32];
        tmem_ld32(t0 + ((uint32_t)(32 * warp) << 16) + 0, d0);
        tmem_ld32(t0 + ((uint32_t)(32 * warp) << 16) + 32, d1);
        const int rho = 32 * warp + lane;
        if (rho < 64) {
            const int rw = rho;
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) {
                float4 x;
                const int i = 4 * i4;
                const float* src = i < 32 ? d0 : d1;
                const int ii = i & 31;
                x.x = (i + 0 < rw) ? src[ii + 0] : 0.f;
                x.y = (i + 1 < rw) ? src[ii + 1] : 0.f;
                x.z = (i + 2 < rw) ? src[ii + 2] : 0.f;
                x.w = (i + 3 < rw) ? src[ii + 3] : 0.f;
                *reinterpret_cast<float4*>(A32 + sw64(rw, i)) = x;
            }
        } else {
            const int rw = rho - 64;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float f[8];
                const float* src = j < 4 ? d0 : d1;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = 8 * j + e;
                    f[e] = (i <= rw) ? src[i & 31] : 0.f;
                }
                st16(sm + kR4, off_kmajor(rw, 8 * j, 1024, 128), f_to_h8(f));
            }
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- T = (I + A)^{-1}
    if (warp < 4 && lane < 16) {       // diagonal 16 x 16 blocks by forward substitution
        const int bb = 16 * warp, jc = lane;
        float t[16];
#pragma unroll
        for (int r2 = 0; r2 < 16; ++r2) {
            float acc = (r2 == jc) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (i >= jc && i < r2) acc -= A32[sw64(bb + r2, bb + i)] * t[i];
            t[r2] = (r2 < jc) ? 0.f : acc;
        }
#pragma unroll
        for (int r2 = 0; r2 < 16; ++r2) T32[sw64(bb + r2, bb + jc)] = t[r2];
    }
    __syncthreads();
    {   // 32 x 32 blocks: T10 = -T11 A10 T00 for the pairs (16..31 | 0..15) and (48..63 | 32..47)
        const int m = tid >> 7, qd = tid & 127;
        const int rw = qd >> 3, jc = (qd & 7) * 2;
        const int base = 32 * m;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int jj = jc + u;
            float acc = 0.f;
            for (int i = jj; i < 16; ++i) acc += A32[sw64(base + 16 + rw, base + i)] * T32[sw64(base + i, base + jj)];
            scr[m * 256 + rw * 16 + jj] = acc;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int jj = jc + u;
            float acc = 0.f;
            for (int mm = 0; mm <= rw; ++mm) acc += T32[sw64(base + 16 + rw, base + 16 + mm)] * scr[m * 256 + mm * 16 + jj];
            T32[sw64(base + 16 + rw, base + jj)] = -acc;
        }
    }
    __syncthreads();
    {   // 64 x 64: T_BL = -T_BR A_BL T_TL (blocks of 32)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int idx = tid + NT * u;
            const int rw = idx >> 5, jj = idx & 31;
            float acc = 0.f;
            for (int i = jj; i < 32; ++i) acc += A32[sw64(32 + rw, i)] * T32[sw64(i, jj)];
            scr[rw * 32 + jj] = acc;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int idx = tid + NT * u;
            const int rw = idx >> 5, jj = idx & 31;
            float acc = 0.f;
            for (int mm = 0; mm <= rw; ++mm) acc += T32[sw64(32 + rw, 32 + mm)] * scr[mm * 32 + jj];
            T32[sw64(32 + rw, jj)] = -acc;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < 512; idx += NT) {   // T -> fp16 B operand (n = r, k = i)
        const int rw = idx >> 3, j = idx & 7;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int i = 8 * j + e;
            f[e] = (i <= rw) ? T32[sw64(rw, i)] : 0.f;
        }
        st16(sm + kR3, off_kmajor(rw, 8 * j, 1024, 128), f_to_h8(f));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------------------------------------------------------- W~^T = KG^T T^T ; U'^T = V~^T T^T
    if (ok) {
        if (tid == 0) {
            const uint32_t id = idesc_f16(128, 64, true, false);
            mma_f16_k(t0 + 64, smem_u32(sm + kR0), 2048, 128, smem_u32(sm + kR3), 128, 1024, id, C, false);
            mma_f16_k(t0 + 128, smem_u32(sm + kR2), 2048, 128, smem_u32(sm + kR3), 128, 1024, id, C, false);
            mma_commit(bar);
        }
        ok = mbar_wait(bar, phase);
        phase ^= 1u;
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) record_timeout(p.status);
    tc_fence_after();
    if (ok && warp < 4) {
        const int ch = 32 * warp + lane;
        const float er = __expf(gref[ch]);
        const uint32_t lanebase = t0 + ((uint32_t)(32 * warp) << 16);
        float x0[32], x1[32];
        tmem_ld32(lanebase + 64, x0);
        tmem_ld32(lanebase + 96, x1);
#pragma unroll
        for (int i0 = 0; i0 < C; i0 += 8) {
            const float* src = (i0 < 32 ? x0 : x1) + (i0 & 31);
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = src[e] * er;
            *reinterpret_cast<uint4*>(blk + kOffAS1 + off_mnmajor(i0, ch, 2048, 128)) = f_to_h8(f);
            st16(sm + kR0, off_kmajor(ch, i0, 128, 2048), f_to_h8(src));
        }
        tmem_ld32(lanebase + 128, x0);
        tmem_ld32(lanebase + 160, x1);
        float* up = reinterpret_cast<float*>(blk + kOffUp) + (size_t)(ch / NS) * C * NS + (ch % NS);
#pragma unroll
        for (int i = 0; i < C; ++i) up[i * NS] = i < 32 ? x0[i] : x1[i - 32];
#pragma unroll
        for (int i0 = 0; i0 < C; i0 += 8) st16(sm + kR2, off_kmajor(ch, i0, 128, 2048), f_to_h8((i0 < 32 ? x0 : x1) + (i0 & 31)));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------------------------------------------------------- (Qe e^{-g_ref})^T and PU'^T
    if (ok) {
        if (tid == 0) {
            mma_f16_k(t0 + 0, smem_u32(sm + kR0), 2048, 128, smem_u32(sm + kR4), 128, 1024,
                      idesc_f16(128, 64, false, false, true), C, false);
            mma_f16_k(t0 + 0, smem_u32(sm + kR0 + 16384), 2048, 128, smem_u32(sm + kR5), 128, 1024,
                      idesc_f16(128, 64, true, false), C, true);
            mma_f16_k(t0 + 192, smem_u32(sm + kR2), 2048, 128, smem_u32(sm + kR4), 128, 1024,
                      idesc_f16(128, 64, false, false), C, false);
            mma_commit(bar);
        }
        ok = mbar_wait(bar, phase);
        phase ^= 1u;
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) record_timeout(p.status);
    tc_fence_after();
    if (ok && warp < 4) {
        const int ch = 32 * warp + lane;
        const float er = __expf(gref[ch]);
        const uint32_t lanebase = t0 + ((uint32_t)(32 * warp) << 16);
        float x0[32], x1[32];
        tmem_ld32(lanebase + 0, x0);
        tmem_ld32(lanebase + 32, x1);
#pragma unroll
        for (int r0 = 0; r0 < C; r0 += 8) {
            const float* src = (r0 < 32 ? x0 : x1) + (r0 & 31);
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = src[e] * er;
            *reinterpret_cast<uint4*>(blk + kOffAS1 + off_mnmajor(64 + r0, ch, 2048, 128)) = f_to_h8(f);
        }
        tmem_ld32(lanebase + 192, x0);
        tmem_ld32(lanebase + 224, x1);
        float* pu = reinterpret_cast<float*>(blk + kOffPUp) + (size_t)(ch / NS) * C * NS + (ch % NS);
#pragma unroll
        for (int i = 0; i < C; ++i) pu[i * NS] = i < 32 ? x0[i] : x1[i - 32];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t0, kTmemCols);
}

// ============================================================================ scan
constexpr int kScanThreads = 160;              // 4 epilogue warps + 1 producer warp
constexpr uint32_t kStageBytes = 32768 + 16384 + 8192 + 8192 + 512;   // AS1, AS2, U', PU', gC
constexpr uint32_t kSAS1 = 0, kSAS2 = 32768, kSUp = 49152, kSPUp = 57344, kSGC = 65536;
constexpr uint32_t kStage0 = 0;
constexpr uint32_t kStageStride = 66560;       // kStageBytes rounded up to 1 KB
constexpr uint32_t kSop = 2 * kStageStride;    // S fp16 B operand (k = ch, n = j): MN-major SBO 2048 LBO 128 (8 KB)
constexpr uint32_t kUop = kSop + 8192;         // U fp16 B operand (k = r, n = j): MN-major SBO 1024 LBO 128 (4 KB)
constexpr uint32_t kSBar = kUop + 4096;        // full[2], empty[2], s1, s2
constexpr uint32_t kSTmem = kSBar + 64;
constexpr uint32_t kScanSmem = kSTmem + 64;

__global__ void __launch_bounds__(kScanThreads, 1) scan_tc_kernel(Problem p) {
    extern __shared__ __align__(1024) uint8_t sm[];
    const int slice = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kSBar);
    uint64_t* empty = full + 2;
    uint64_t* s1 = full + 4;
    uint64_t* s2 = full + 5;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kSTmem);
    const uint8_t* blocks = static_cast<const uint8_t*>(p.inter) + (size_t)bh * p.NC * kBlockBytes;

    if (warp == 0) {
        tmem_alloc(tslot, 64);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&empty[0], 1);
        mbar_init(&empty[1], 1);
        mbar_init(s1, 1);
        mbar_init(s2, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = *tslot;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int ch = 0; ch < p.NC; ++ch) {
                const int st = ch & 1;
                if (ch >= 2 && !mbar_wait(&empty[st], ((ch >> 1) - 1) & 1)) {
                    record_timeout(p.status);
                    break;
                }
                uint8_t* dst = sm + kStage0 + st * kStageStride;
                const uint8_t* src = blocks + (size_t)ch * kBlockBytes;
                mbar_arrive_expect_tx(&full[st], kStageBytes);
                bulk_g2s(dst + kSAS1, src + kOffAS1, 32768, &full[st]);
                bulk_g2s(dst + kSAS2, src + kOffAS2, 16384, &full[st]);
                bulk_g2s(dst + kSUp, src + kOffUp + (size_t)slice * C * NS * 4, 8192, &full[st]);
                bulk_g2s(dst + kSPUp, src + kOffPUp + (size_t)slice * C * NS * 4, 8192, &full[st]);
                bulk_g2s(dst + kSGC, src + kOffGC, 512, &full[st]);
            }
        }
    } else {
        // ------------------------------------------------------------ state chain (128 threads)
        const int row = tid;                           // TMEM lane: d_k row of S / chunk row of D1
        const int j0 = slice * NS;
        const uint32_t lanebase = t0 + ((uint32_t)(32 * warp) << 16);
        float S[NS];
#pragma unroll
        for (int j = 0; j < NS; ++j) S[j] = p.S0 ? p.S0[((size_t)bh * D + row) * D + j0 + j] : 0.f;
#pragma unroll
        for (int j = 0; j < NS; j += 8) st16(sm + kSop, off_mnmajor(j, row, 2048, 128), f_to_h8(S + j));
        fence_async_smem();
        named_barrier(1, 128);
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
        const uint32_t id1 = idesc_f16(128, NS, true, true);
        const uint32_t id2 = idesc_f16(128, NS, true, true);
        bool ok = true;
        for (int ch = 0; ch < p.NC; ++ch) {
            const int st = ch & 1;
            uint8_t* stg = sm + kStage0 + st * kStageStride;
            bool mine = mbar_wait(&full[st], (ch >> 1) & 1);
            if (tid == 0 && mine) {
                tc_fence_after();
                mma_f16_k(t0 + 0, smem_u32(stg + kSAS1), 128, 2048, smem_u32(sm + kSop), 128, 2048, id1, D, false);
                mma_commit(s1);
            }
            mine = mine && mbar_wait(s1, ch & 1);
            tc_fence_after();
            float d[NS];
            if (mine) {
                tmem_ld32(lanebase + 0, d);
                const float* up = reinterpret_cast<const float*>(stg + kSUp);
                const float* pu = reinterpret_cast<const float*>(stg + kSPUp);
                if (row < C) {
#pragma unroll
                    for (int j = 0; j < NS; ++j) d[j] = up[row * NS + j] - d[j];
#pragma unroll
                    for (int j = 0; j < NS; j += 8) st16(sm + kUop, off_mnmajor(j, row, 1024, 128), f_to_h8(d + j));
                    fence_async_smem();
                } else {
                    const int rw = row - C;
                    const int s = ch * C + rw;
                    if (s < p.L) {
                        const RowRef ro = row_ref(p, b, h, s);
                        if (ro.has_q) {
                            uint4* dst = reinterpret_cast<uint4*>(out + ro.tok * D + j0);
#pragma unroll
                            for (int j = 0; j < NS; j += 8) {
                                __nv_bfloat162 o2[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    o2[e] = __floats2bfloat162_rn(pu[rw * NS + j + 2 * e] + d[j + 2 * e],
                                                                  pu[rw * NS + j + 2 * e + 1] + d[j + 2 * e + 1]);
                                dst[j / 8] = *reinterpret_cast<uint4*>(o2);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            ok = named_barrier_and(1, 128, mine);
            if (!ok) break;
            if (tid == 0) {
                tc_fence_after();
                mma_f16_k(t0 + 32, smem_u32(stg + kSAS2), 128, 1024, smem_u32(sm + kUop), 128, 1024, id2, C, false);
                mma_commit(s2);
            }
            mine = mbar_wait(s2, ch & 1);
            tc_fence_after();
            if (mine) {
                tmem_ld32(lanebase + 32, d);
                const float gc = reinterpret_cast<const float*>(stg + kSGC)[row];
#pragma unroll
                for (int j = 0; j < NS; ++j) S[j] = gc * S[j] + d[j];
#pragma unroll
                for (int j = 0; j < NS; j += 8) st16(sm + kSop, off_mnmajor(j, row, 2048, 128), f_to_h8(S + j));
                fence_async_smem();
            }
            tc_fence_before();
            ok = named_barrier_and(1, 128, mine);
            if (!ok) break;
            if (tid == 0) mbar_arrive(&empty[st]);
        }
        if (!ok) {
            if (lane == 0) record_timeout(p.status);
        } else if (p.S_final) {
            float4* dst = reinterpret_cast<float4*>(p.S_final + ((size_t)bh * D + row) * D + j0);
#pragma unroll
            for (int j = 0; j < NS; j += 4) dst[j / 4] = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t0, 64);
}

}  // namespace tc

bool tc_supported(const Problem& p, bool bf16) {
    return bf16 && p.C == tc::C && p.dk == tc::D && p.dv == tc::D && p.T > 0;
}

size_t tc_inter_bytes(const Problem& p) { return (size_t)p.B * p.H * p.NC * tc::kBlockBytes; }

int tc_launches(const Problem& p) { return p.NC > 0 ? 2 : 1; }

cudaError_t launch_tc(const Problem& p, cudaStream_t stream) {
    cudaFuncSetAttribute(tc::intra_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kIntraSmem);
    cudaFuncSetAttribute(tc::scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kScanSmem);
    dim3 g1(p.NC, p.B * p.H);
    tc::intra_tc_kernel<<<g1, tc::NT, tc::kIntraSmem, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2(tc::J, p.B * p.H);
    tc::scan_tc_kernel<<<g2, tc::kScanThreads, tc::kScanSmem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
