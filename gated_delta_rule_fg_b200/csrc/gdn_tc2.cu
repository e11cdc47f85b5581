// gdn_tc2.cu -- the intra role of the tensor-core path, fed by TMA: one CTA per (chunk, head),
// 256 threads, two CTAs per SM.  It writes the same per-(head, chunk) block as
// tc::intra_tc_kernel (gdn_tc_common.cuh), so the scan role is shared.
//
// Loads.  One thread issues six TMA boxes (64 tokens x 64 channels of q, k, v, 128-byte
// swizzle) through 4-D tensor maps over this GPU's own input buffers; rows past the end of
// the sequence arrive as zeros.  alpha and beta are read with vector loads while the boxes land.
//
// Decay.  With P_r = prod_{s <= r} alpha_s (per channel, inside the chunk), gamma = P_{C-1} and
// the reference ref = sqrt(gamma) (the middle of the chunk's log-decay range),
//   KG = k~ P / ref,  QG = q^ P / ref,  KI = k~ ref / P     (all within e^{+-span/2})
// so that A = strictly-lower(KG KI^T) and P = lower(QG KI^T).  The fp16 operands are written
// in place over the raw boxes (KG over k, QG over q, V over v; KI into its own box), in the
// swizzled layout the tensor cores read, each thread rewriting the 16-byte pieces it read.
// Chunks with gamma < e^{-2 kMaxHalfSpan} take the element-wise fp32 path for A and P (as
// tc::intra_tc_kernel does), with ref = 1 and K' = k~ e^{g_C - g} in the KI box.
//
// Products.  With T = (I + A)^{-1}, Y = KI^T T (128 x 64) and Z = P T (64 x 64):
//   N  = -diag(ref) (Y KG) diag(ref)      (= -K'^T W)
//   b  =  diag(ref) (Y V)                 (=  K'^T U')
//   Qe = (QG - Z KG) diag(ref)            (=  Q^ e^g - P W)
//   PU' = Z V
// because K' = KI diag(ref) and W = T KG diag(ref).  Four rounds of tensor-core products:
// [A; P]; Y and Z; N~ = Y KG and -Z KG (the Qe epilogue adds QG from shared memory); b~ and
// PU'.  Each round is issued by two threads (see bar_mma2).  Qe is stored K-major (rows of 128
// channels), the layout the scan copies into tensor memory as an A operand.
#include <cuda.h>

#include "gdn_tc_common.cuh"

namespace gdn {
namespace tc2 {
using namespace sm100;
using tc::C;
using tc::D;
using tc::NS;

constexpr int NT = 256;
constexpr float kMinGamma = 6.14421235e-06f;   // e^{-2 kMaxHalfSpan}: below it, the element-wise path
constexpr float kFp16Max = 65504.f;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t kKQ = 0;          // 128-byte-swizzled boxes: KG ch 0-63 @0, QG ch 0-63 @8192,
                                     //   KG ch 64-127 @16384, QG ch 64-127 @24576 (rows = tokens)
constexpr uint32_t kV = 32768;       // V boxes @32768, @40960
constexpr uint32_t kKI = 49152;      // KI boxes @49152, @57344
constexpr uint32_t kA32 = 65536;     // A, then T in place: fp32 64x64 (tc::sw64); later Y fp16
                                     //   (K-major (m = channel, k = row): SBO 1024, LBO 128)
constexpr uint32_t kT16 = 81920;     // T fp16 (k = row, n = column): MN-major SBO 128, LBO 1024;
                                     //   later Z fp16 (n = row r, k = r'): K-major SBO 1024, LBO 128
constexpr uint32_t kP16 = 90112;     // P fp16 (m = row, k = column): K-major SBO 1024, LBO 128
constexpr uint32_t kScr = 98304;     // 8 KB: row-group decay totals [16][128]; solve temporaries
constexpr uint32_t kTab = 106496;    // fp32 [5][128]: gamma, ref, 1/ref, row scale, column scale
constexpr uint32_t kBarOff = 109056; // mbarriers (TMA, MMA), TMEM base
constexpr uint32_t kSmem = kBarOff + 64 + 1024;   // + slack to align the base to 1024 bytes
static_assert(2 * (kSmem + 1024) <= 233472, "two CTAs per SM");

// fp32 -> tf32 (round to nearest, ties away) for the warp-level tensor-core products
__device__ __forceinline__ uint32_t f_to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// x = hi + lo to about 2^-22 relative, both tf32
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = f_to_tf32(x);
    lo = f_to_tf32(x - __uint_as_float(hi));
}
// d += a b: one m16n8k8 tf32 product with fp32 accumulation (warp-wide)
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// in-box offset of the 16-byte piece holding channels 8j .. 8j+7 (j < 8) of row r
__device__ __forceinline__ uint32_t box16(int r, int j) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

// kPlus: FG^2-GDN+ (value rate beta^v).  kDP: DeltaProduct with n_h dividing the chunk: row s of
// the chunk is sub-step s0 + s (token (s0 + s) / n_h, step (s0 + s) % n_h); k and v arrive through
// 5-D maps (channel, step, head, token, batch) whose boxes are whole tokens, and q (one row per
// token, on its last step) is read with vector loads.
template <bool kPlus, bool kDP>
__global__ void __launch_bounds__(NT, 2) intra_tma_kernel(Problem p, int cb, int head_fastest,
                                                          const __grid_constant__ CUtensorMap tmq,
                                                          const __grid_constant__ CUtensorMap tmk,
                                                          const __grid_constant__ CUtensorMap tmv) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    // head_fastest: blockIdx.x is the head, so CTAs launched together read the same token rows
    // (adjacent in memory) for different heads.  Chunks are taken last to first: the blocks the
    // scan reads first are then the ones written last, still in L2 when it starts.
    const int c = cb + (head_fastest ? gridDim.y - 1 - blockIdx.y : gridDim.x - 1 - blockIdx.x);
    const int bh = head_fastest ? blockIdx.x : blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int s0 = c * C;
    const int Cv = min(C, p.L - s0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (!GDN_IN_BOUNDS(c < p.NC && bh < p.B * p.H, p.status)) return;   // the whole CTA, before any barrier
    uint8_t* blk = static_cast<uint8_t*>(p.inter) + ((size_t)bh * p.NC + c) * tc::kBlockBytes;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + kBarOff);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kBarOff + 16);
    // Every round of products is issued by two threads in different warps (thread 0 and thread 32),
    // each committing to its own barrier: a thread issuing tcgen05.mma is held for about the time
    // the tensor pipe takes to accept each instruction, and two issuers proceed side by side.
    uint64_t* bar_mma2 = reinterpret_cast<uint64_t*>(sm + kBarOff + 24);
    float* scr = reinterpret_cast<float*>(sm + kScr);
    float* tgam = reinterpret_cast<float*>(sm + kTab);
    float* tref = tgam + 128;
    float* tinv = tgam + 256;
    float* trow = tgam + 384;
    float* tcol = tgam + 512;
    float* A32 = reinterpret_cast<float*>(sm + kA32);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_mma2, 1);
        fence_mbar_init();
        if (kDP) {
            const int t0 = s0 / p.nh;
            mbar_arrive_expect_tx(bar_tma, 4 * 8192);
            tma_load_5d(sm + kKQ + 0, &tmk, 0, 0, h, t0, b, bar_tma);
            tma_load_5d(sm + kKQ + 16384, &tmk, 64, 0, h, t0, b, bar_tma);
            tma_load_5d(sm + kV, &tmv, 0, 0, h, t0, b, bar_tma);
            tma_load_5d(sm + kV + 8192, &tmv, 64, 0, h, t0, b, bar_tma);
        } else {
            mbar_arrive_expect_tx(bar_tma, 6 * 8192);
            tma_load_4d(sm + kKQ + 0, &tmk, 0, h, s0, b, bar_tma);
            tma_load_4d(sm + kKQ + 16384, &tmk, 64, h, s0, b, bar_tma);
            tma_load_4d(sm + kKQ + 8192, &tmq, 0, h, s0, b, bar_tma);
            tma_load_4d(sm + kKQ + 24576, &tmq, 64, h, s0, b, bar_tma);
            tma_load_4d(sm + kV, &tmv, 0, h, s0, b, bar_tma);
            tma_load_4d(sm + kV + 8192, &tmv, 64, h, s0, b, bar_tma);
        }
    }

    // ---------------------------------------------------------------- prep
    // thread: channel octet o (channels 8o .. 8o+7) of rows 4 rg .. 4 rg + 3
    const int o = tid & 15, rg = tid >> 4, hf = o >> 3, j8 = o & 7;
    const int ch0 = 8 * o;
    // largest |value| this thread converts to fp16 among the operands that scale with v
    // (V, b, PU'); above the fp16 range the chunk's results are not valid (reported as RANGE)
    float vmax = 0.f;
    const bool a_scalar = p.alpha_scalar != 0, b_scalar = p.beta_scalar != 0;
    float lp[4][8];     // alpha, then the cumulative product inside this thread's rows
    float be[4][8];     // beta (key rate)
    uint4 qdp[4];       // DeltaProduct: raw q of the row (zero unless the row is its token's last step)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = 4 * rg + i;
        const bool valid = r < Cv;
        size_t tok;
        if (kDP) {
            const int sub = s0 + r, t = sub / p.nh, m = sub - t * p.nh;
            tok = ((size_t)b * p.T + t) * p.H + h;
            const float a = (valid && m == 0) ? __ldg(p.alpha + tok) : 1.f;
            const float bb = valid ? __ldg(p.beta + tok * p.nh + m) : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                lp[i][e] = a;
                be[i][e] = bb;
            }
            qdp[i] = (valid && m == p.nh - 1)
                         ? tc::ldg16(static_cast<const __nv_bfloat16*>(p.q) + tok * D + ch0)
                         : make_uint4(0, 0, 0, 0);
            continue;
        }
        tok = ((size_t)b * p.T + s0 + r) * p.H + h;
        const bool vr = valid && GDN_IN_BOUNDS(tok < (size_t)p.B * p.T * p.H, p.status);
        if (vr && !a_scalar) {
            const float4 x0 = tc::ldg16f(p.alpha + tok * D + ch0), x1 = tc::ldg16f(p.alpha + tok * D + ch0 + 4);
            lp[i][0] = x0.x; lp[i][1] = x0.y; lp[i][2] = x0.z; lp[i][3] = x0.w;
            lp[i][4] = x1.x; lp[i][5] = x1.y; lp[i][6] = x1.z; lp[i][7] = x1.w;
        } else {
            const float a = vr ? __ldg(p.alpha + tok) : 1.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) lp[i][e] = a;
        }
        if (vr && !b_scalar) {
            const float4 x0 = tc::ldg16f(p.beta + tok * D + ch0), x1 = tc::ldg16f(p.beta + tok * D + ch0 + 4);
            be[i][0] = x0.x; be[i][1] = x0.y; be[i][2] = x0.z; be[i][3] = x0.w;
            be[i][4] = x1.x; be[i][5] = x1.y; be[i][6] = x1.z; be[i][7] = x1.w;
        } else {
            const float bb = vr ? __ldg(p.beta + tok) : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) be[i][e] = bb;
        }
    }
    // the tensor memory is taken once the q, k, v boxes and this warp's alpha / beta loads are in
    // flight (its latency then overlaps theirs)
    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    // cumulative product over this thread's four rows; the row-group total goes to scr
#pragma unroll
    for (int i = 1; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) lp[i][e] *= lp[i - 1][e];
    *reinterpret_cast<float4*>(scr + rg * D + ch0) = make_float4(lp[3][0], lp[3][1], lp[3][2], lp[3][3]);
    *reinterpret_cast<float4*>(scr + rg * D + ch0 + 4) = make_float4(lp[3][4], lp[3][5], lp[3][6], lp[3][7]);

    // row norms of q and k (the 16 octets of a row are the 16 lanes of a half-warp)
    tc_fence_before();
    __syncthreads();                      // mbarrier init and TMEM slot visible; scr totals written
    tc_fence_after();
    bool ok = mbar_wait(bar_tma, 0);
    uint8_t* kbox = sm + kKQ + hf * 16384;
    uint8_t* qbox = kbox + 8192;
    uint8_t* vbox = sm + kV + hf * 8192;
    uint8_t* ibox = sm + kKI + hf * 8192;
    float ik[4], iq[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t off = box16(4 * rg + i, j8);
        float fk[8], fq[8];
        tc::bf8_to_f(*reinterpret_cast<const uint4*>(kbox + off), fk);
        tc::bf8_to_f(kDP ? qdp[i] : *reinterpret_cast<const uint4*>(qbox + off), fq);
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sk = fmaf(fk[e], fk[e], sk);
            sq = fmaf(fq[e], fq[e], sq);
        }
#pragma unroll
        for (int m = 1; m < 16; m <<= 1) {
            sk += __shfl_xor_sync(0xffffffffu, sk, m);
            sq += __shfl_xor_sync(0xffffffffu, sq, m);
        }
        ik[i] = rsqrtf(sk + kNormEps);
        iq[i] = rsqrtf(sq + kNormEps);
    }
    // exclusive prefix of the row-group totals per channel, and gamma
    bool wide = false;
    if (tid < D) {
        float v[16];                      // all sixteen loads first, then the dependent products
#pragma unroll
        for (int g = 0; g < 16; ++g) v[g] = scr[g * D + tid];
        float acc = 1.f;
#pragma unroll
        for (int g = 0; g < 16; ++g) {
            scr[g * D + tid] = acc;
            acc *= v[g];
        }
        tgam[tid] = acc;
        wide = !(acc >= kMinGamma);
    }
    const int fallback = __syncthreads_or(wide);
    if (tid < D) {
        const float gm = tgam[tid];
        const float rf = fallback ? 1.f : sqrtf(gm);
        tref[tid] = rf;
        tinv[tid] = fallback ? 1.f : rsqrtf(gm);
        trow[tid] = rf;
        tcol[tid] = rf;
    }
    __syncthreads();

    float* fb_g = reinterpret_cast<float*>(blk + tc::kOffB);                  // fallback scratch: g fp32 [C][D]
    __half* fb_k = reinterpret_cast<__half*>(blk + tc::kOffPU);               // k~ fp16 [C][D]
    __half* fb_q = reinterpret_cast<__half*>(blk + tc::kOffN);                // q^ fp16 [C][D]
    if (!fallback) {
        float pre[8];       // the row group's prefix, over ref: P = pre * lp * ref
        {
            const float4 a0 = *reinterpret_cast<const float4*>(scr + rg * D + ch0);
            const float4 a1 = *reinterpret_cast<const float4*>(scr + rg * D + ch0 + 4);
            pre[0] = a0.x; pre[1] = a0.y; pre[2] = a0.z; pre[3] = a0.w;
            pre[4] = a1.x; pre[5] = a1.y; pre[6] = a1.z; pre[7] = a1.w;
#pragma unroll
            for (int e = 0; e < 8; ++e) pre[e] *= tinv[ch0 + e];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * rg + i;
            const uint32_t off = box16(r, j8);
            float fk[8], fq[8], fv[8], sv[8];
            tc::bf8_to_f(*reinterpret_cast<const uint4*>(kbox + off), fk);
            tc::bf8_to_f(kDP ? qdp[i] : *reinterpret_cast<const uint4*>(qbox + off), fq);
            tc::bf8_to_f(*reinterpret_cast<const uint4*>(vbox + off), fv);
            if (kPlus) {
                const bool valid = r < Cv;
                const size_t tok = ((size_t)b * p.T + s0 + r) * p.H + h;
                if (valid && !b_scalar) {
                    const float4 x0 = tc::ldg16f(p.beta_v + tok * D + ch0), x1 = tc::ldg16f(p.beta_v + tok * D + ch0 + 4);
                    sv[0] = tc::sqrt_op(x0.x); sv[1] = tc::sqrt_op(x0.y); sv[2] = tc::sqrt_op(x0.z); sv[3] = tc::sqrt_op(x0.w);
                    sv[4] = tc::sqrt_op(x1.x); sv[5] = tc::sqrt_op(x1.y); sv[6] = tc::sqrt_op(x1.z); sv[7] = tc::sqrt_op(x1.w);
                } else {
                    const float s = valid ? tc::sqrt_op(__ldg(p.beta_v + tok)) : 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) sv[e] = s;
                }
            }
            float KG[8], QG[8], KI[8], VT[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float Pv = pre[e] * lp[i][e];      // P / ref, in [e^{-6}, e^{6}]
                const float rpv = __fdividef(1.f, Pv);   // ref / P
                const float sb = tc::sqrt_op(be[i][e]);
                const float kt = fk[e] * ik[i] * sb;
                KG[e] = kt * Pv;
                KI[e] = kt * rpv;
                QG[e] = fq[e] * iq[i] * Pv;
                VT[e] = fv[e] * (kPlus ? sv[e] : sb);
                vmax = fmax_nan(vmax, fabsf(VT[e]));
            }
            *reinterpret_cast<uint4*>(kbox + off) = tc::f_to_h8(KG);
            *reinterpret_cast<uint4*>(qbox + off) = tc::f_to_h8(QG);
            *reinterpret_cast<uint4*>(vbox + off) = tc::f_to_h8(VT);
            *reinterpret_cast<uint4*>(ibox + off) = tc::f_to_h8(KI);
        }
    } else {
        // Element-wise path: log-domain cumulative decay (the products above may have
        // underflowed), ref = 1, K' = k~ e^{g_C - g} in the KI box; g, k~ and q^ are staged
        // in this chunk's block for the element-wise A and P.
        float lg[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * rg + i;
            const bool valid = r < Cv;
            const size_t tok = ((size_t)b * p.T + s0 + r) * p.H + h;
            float a_dp = 1.f;
            if (kDP) {
                const int sub = s0 + r, t = sub / p.nh, m = sub - t * p.nh;
                a_dp = (valid && m == 0) ? __ldg(p.alpha + ((size_t)b * p.T + t) * p.H + h) : 1.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float a = kDP ? a_dp
                                    : (!valid ? 1.f : (a_scalar ? __ldg(p.alpha + tok) : __ldg(p.alpha + tok * D + ch0 + e)));
                lg[i][e] = __logf(a) + (i ? lg[i - 1][e] : 0.f);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) scr[rg * D + ch0 + e] = lg[3][e];
        __syncthreads();
        if (tid < D) {
            float acc = 0.f;
#pragma unroll
            for (int g = 0; g < 16; ++g) {
                const float v = scr[g * D + tid];
                scr[g * D + tid] = acc;
                acc += v;
            }
            tgam[tid] = acc;          // g_C (log) for now
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * rg + i;
            const uint32_t off = box16(r, j8);
            float fk[8], fq[8], fv[8], sv[8];
            tc::bf8_to_f(*reinterpret_cast<const uint4*>(kbox + off), fk);
            tc::bf8_to_f(kDP ? qdp[i] : *reinterpret_cast<const uint4*>(qbox + off), fq);
            tc::bf8_to_f(*reinterpret_cast<const uint4*>(vbox + off), fv);
            if (kPlus) {
                const bool valid = r < Cv;
                const size_t tok = ((size_t)b * p.T + s0 + r) * p.H + h;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    sv[e] = !valid ? 0.f : tc::sqrt_op(b_scalar ? __ldg(p.beta_v + tok) : __ldg(p.beta_v + tok * D + ch0 + e));
            }
            float KG[8], QG[8], KP[8], VT[8], KT[8], QH[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float g = lg[i][e] + scr[rg * D + ch0 + e];
                const float sb = tc::sqrt_op(be[i][e]);
                const float kt = fk[e] * ik[i] * sb;
                const float qh = fq[e] * iq[i];
                const float eg = __expf(g);
                KG[e] = kt * eg;
                QG[e] = qh * eg;
                KP[e] = kt * __expf(tgam[ch0 + e] - g);
                VT[e] = fv[e] * (kPlus ? sv[e] : sb);
                vmax = fmax_nan(vmax, fabsf(VT[e]));
                KT[e] = kt;
                QH[e] = qh;
                fb_g[r * D + ch0 + e] = g;
            }
            *reinterpret_cast<uint4*>(kbox + off) = tc::f_to_h8(KG);
            *reinterpret_cast<uint4*>(qbox + off) = tc::f_to_h8(QG);
            *reinterpret_cast<uint4*>(vbox + off) = tc::f_to_h8(VT);
            *reinterpret_cast<uint4*>(ibox + off) = tc::f_to_h8(KP);
            *reinterpret_cast<uint4*>(fb_k + r * D + ch0) = tc::f_to_h8(KT);
            *reinterpret_cast<uint4*>(fb_q + r * D + ch0) = tc::f_to_h8(QH);
        }
        __syncthreads();
        if (tid < D) tgam[tid] = __expf(tgam[tid]);     // gamma = e^{g_C}
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = *tslot;
    const uint32_t base = smem_u32(sm);
    uint32_t phase = 0;

    // ---------------------------------------------------------------- [A; P] = [KG; QG] KI^T
    if (!fallback) {
        // channels 0-63 (thread 0) into columns 0-63, channels 64-127 (thread 32) into 64-127;
        // the epilogue adds the two
        if ((tid == 0 || tid == 32) && ok) {
            const uint32_t id = idesc_f16(128, 64, false, false);
            const int hk = tid >> 5;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const uint32_t koff = (uint32_t)(hk * 16384 + k4 * 32);
                const uint32_t kioff = (uint32_t)(hk * 8192 + k4 * 32);
                mma_f16(t0 + 64u * hk, sdesc_sw128(base + kKQ + koff, 16, 1024), sdesc_sw128(base + kKI + kioff, 16, 1024),
                        id, k4 > 0);
            }
            mma_commit(hk ? bar_mma2 : bar_mma);
        }
        ok = ok && mbar_wait(bar_mma, phase) && mbar_wait(bar_mma2, phase);
        phase ^= 1u;
    } else if (warp < 4) {
        // exact fp32 Gram products, element by element (decay formed per pair of rows)
        const int rho = 32 * warp + lane;
        const int rowr = rho & 63;
        const bool isP = rho >= 64;
        for (int cb2 = 0; cb2 < 64; cb2 += 32) {
            float acc[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = 0.f;
            for (int ch = 0; ch < D; ++ch) {
                const float gr = fb_g[rowr * D + ch];
                const float xr = __half2float(isP ? fb_q[rowr * D + ch] : fb_k[rowr * D + ch]);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int col = cb2 + i;
                    if (col < rowr || (isP && col == rowr))
                        acc[i] += xr * __half2float(fb_k[col * D + ch]) * __expf(gr - fb_g[col * D + ch]);
                }
            }
            tmem_st32(t0 + ((uint32_t)(32 * warp) << 16) + cb2, acc);
        }
        tc_fence_before();
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) tc::record_timeout(p.status);
    tc_fence_after();
    if (ok) {   // A rows -> fp32 (strictly lower), P rows -> fp16 (lower); warps w, w+4 share a lane quarter
        const int q = warp & 3, chh = warp >> 2;
        float d[32];
        if (!fallback) {
            float d2[32];
            tmem_ld32_async(t0 + ((uint32_t)(32 * q) << 16) + 32 * chh, d);
            tmem_ld32_async(t0 + ((uint32_t)(32 * q) << 16) + 64 + 32 * chh, d2);
            tmem_ld_wait2(d, d2);
#pragma unroll
            for (int i = 0; i < 32; ++i) d[i] += d2[i];
        } else {
            tmem_ld32(t0 + ((uint32_t)(32 * q) << 16) + 32 * chh, d);
        }
        const int rho = 32 * q + lane;
        if (rho < 64) {
            const int rw = rho;
#pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {
                const int i = 32 * chh + 4 * i4;
                float4 x;
                x.x = (i + 0 < rw) ? d[4 * i4 + 0] : 0.f;
                x.y = (i + 1 < rw) ? d[4 * i4 + 1] : 0.f;
                x.z = (i + 2 < rw) ? d[4 * i4 + 2] : 0.f;
                x.w = (i + 3 < rw) ? d[4 * i4 + 3] : 0.f;
                *reinterpret_cast<float4*>(A32 + tc::sw64(rw, i)) = x;
            }
        } else {
            const int rw = rho - 64;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = 32 * chh + 8 * j + e;
                    f[e] = (i <= rw) ? d[8 * j + e] : 0.f;
                }
                tc::st16(sm + kP16, off_kmajor(rw, 32 * chh + 8 * j, 1024, 128), tc::f_to_h8(f));
            }
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- T = (I + A)^{-1}, in place
    // Four 16x16 diagonal blocks by forward substitution in registers (lane j carries column j,
    // rows of A are broadcast shared-memory reads), then T10 = -T11 (A10 T00) on 16x16 and
    // 32x32 blocks; each merge overwrites the A block it consumed.
    if (warp < 4) {
        // rows of A read as broadcast float4 (four consecutive entries share one swizzled 16-byte
        // piece); four partial sums keep the dependent chain of each row short
        const int bb = 16 * warp, jc = lane & 15;
        float t[16];
#pragma unroll
        for (int r2 = 0; r2 < 16; ++r2) {
            float acc[4] = {(r2 == jc) ? 1.f : 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i4 = 0; i4 < r2; i4 += 4) {
                const float4 a = *reinterpret_cast<const float4*>(A32 + tc::sw64(bb + r2, bb + i4));
                const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (i4 + e < r2) acc[e] = fmaf(-av[e], t[i4 + e], acc[e]);
            }
            t[r2] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        }
        __syncwarp();
        if (lane < 16) {
#pragma unroll
            for (int r2 = 0; r2 < 16; ++r2) A32[tc::sw64(bb + r2, bb + jc)] = t[r2];
        }
    }
    __syncthreads();
    // Block merges T10 = -T11 (A10 T00) as warp-level tensor-core products (m16n8k8) in split
    // tf32: every fp32 operand x = hi + lo with hi = tf32(x), lo = tf32(x - hi), and the product
    // a b ~ a_hi b_hi + a_hi b_lo + a_lo b_hi accumulated in fp32 (the error of the dropped
    // a_lo b_lo term and of the splits is near fp32 rounding).  Operands are read from the fp32
    // A / T array.  gid = lane / 4, tig = lane % 4.
    {
        const int gid = lane >> 2, tig = lane & 3;
        auto Af = [&](int m0, int k0, uint32_t (&ah)[4], uint32_t (&al)[4]) {   // rows m0.., columns k0..
            split_tf32(A32[tc::sw64(m0 + gid, k0 + tig)], ah[0], al[0]);
            split_tf32(A32[tc::sw64(m0 + gid + 8, k0 + tig)], ah[1], al[1]);
            split_tf32(A32[tc::sw64(m0 + gid, k0 + tig + 4)], ah[2], al[2]);
            split_tf32(A32[tc::sw64(m0 + gid + 8, k0 + tig + 4)], ah[3], al[3]);
        };
        auto Bf = [&](const float* M, int ld, int k0, int n0, uint32_t (&bh)[2], uint32_t (&bl)[2], bool swz) {
            split_tf32(swz ? M[tc::sw64(k0 + tig, n0 + gid)] : M[(k0 + tig) * ld + n0 + gid], bh[0], bl[0]);
            split_tf32(swz ? M[tc::sw64(k0 + tig + 4, n0 + gid)] : M[(k0 + tig + 4) * ld + n0 + gid], bh[1], bl[1]);
        };
        // the three terms go to three accumulators (three short dependency chains), summed at the end
        auto mma3 = [&](float (&d)[12], const uint32_t (&ah)[4], const uint32_t (&al)[4], const uint32_t (&bh)[2],
                        const uint32_t (&bl)[2]) {
            mma_tf32(*reinterpret_cast<float(*)[4]>(d + 8), al, bh);
            mma_tf32(*reinterpret_cast<float(*)[4]>(d + 4), ah, bl);
            mma_tf32(*reinterpret_cast<float(*)[4]>(d + 0), ah, bh);
        };
        auto sum3 = [](const float (&d)[12], int i) { return d[i] + (d[4 + i] + d[8 + i]); };
        // 16-row merges, block pairs (16..31 | 0..15) and (48..63 | 32..47): warp w < 4 takes pair
        // w / 2 and the 8 columns 8 (w % 2) of its 16; X = A10 T00 stays in this warp
        if (warp < 4) {
            const int bs = 32 * (warp >> 1), n0 = bs + 8 * (warp & 1);
            float x[12] = {};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8) {
                uint32_t ah[4], al[4], bh[2], bl[2];
                Af(bs + 16, bs + k0, ah, al);
                Bf(A32, 0, bs + k0, n0, bh, bl, true);
                mma3(x, ah, al, bh, bl);
            }
            float* xs = scr + warp * 128;                       // X columns n0 .. n0+7: [16][8]
            xs[gid * 8 + 2 * tig] = sum3(x, 0);
            xs[gid * 8 + 2 * tig + 1] = sum3(x, 1);
            xs[(gid + 8) * 8 + 2 * tig] = sum3(x, 2);
            xs[(gid + 8) * 8 + 2 * tig + 1] = sum3(x, 3);
            __syncwarp();
            float y[12] = {};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8) {
                uint32_t ah[4], al[4], bh[2], bl[2];
                Af(bs + 16, bs + 16 + k0, ah, al);
                Bf(xs, 8, k0, 0, bh, bl, false);
                mma3(y, ah, al, bh, bl);
            }
            A32[tc::sw64(bs + 16 + gid, n0 + 2 * tig)] = -sum3(y, 0);
            A32[tc::sw64(bs + 16 + gid, n0 + 2 * tig + 1)] = -sum3(y, 1);
            A32[tc::sw64(bs + 24 + gid, n0 + 2 * tig)] = -sum3(y, 2);
            A32[tc::sw64(bs + 24 + gid, n0 + 2 * tig + 1)] = -sum3(y, 3);
        }
        __syncthreads();
        // 32-row merge: T_BL = -T_BR (A_BL T_TL); warp w takes rows 32 + 16 (w / 4) and columns
        // 8 (w % 4) of the 32 x 32 products
        const int m0 = 16 * (warp >> 2), n0 = 8 * (warp & 3);
        float x[12] = {};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8) {
            uint32_t ah[4], al[4], bh[2], bl[2];
            Af(32 + m0, k0, ah, al);
            Bf(A32, 0, k0, n0, bh, bl, true);
            mma3(x, ah, al, bh, bl);
        }
        float* xs = scr + 512;                                 // X: [32][32]
        xs[(m0 + gid) * 32 + n0 + 2 * tig] = sum3(x, 0);
        xs[(m0 + gid) * 32 + n0 + 2 * tig + 1] = sum3(x, 1);
        xs[(m0 + gid + 8) * 32 + n0 + 2 * tig] = sum3(x, 2);
        xs[(m0 + gid + 8) * 32 + n0 + 2 * tig + 1] = sum3(x, 3);
        __syncthreads();
        float y[12] = {};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8) {
            uint32_t ah[4], al[4], bh[2], bl[2];
            Af(32 + m0, 32 + k0, ah, al);
            Bf(xs, 32, k0, n0, bh, bl, false);
            mma3(y, ah, al, bh, bl);
        }
        A32[tc::sw64(32 + m0 + gid, n0 + 2 * tig)] = -sum3(y, 0);
        A32[tc::sw64(32 + m0 + gid, n0 + 2 * tig + 1)] = -sum3(y, 1);
        A32[tc::sw64(40 + m0 + gid, n0 + 2 * tig)] = -sum3(y, 2);
        A32[tc::sw64(40 + m0 + gid, n0 + 2 * tig + 1)] = -sum3(y, 3);
    }
    __syncthreads();
    for (int idx = tid; idx < 512; idx += NT) {   // T -> fp16 (rows contiguous in 16-byte pieces)
        const int rw = idx & 63, j = idx >> 6;
        const float4 ta = *reinterpret_cast<const float4*>(A32 + tc::sw64(rw, 8 * j));
        const float4 tb = *reinterpret_cast<const float4*>(A32 + tc::sw64(rw, 8 * j + 4));
        float f[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (8 * j + e > rw) f[e] = 0.f;
        tc::st16(sm + kT16, off_kmajor(rw, 8 * j, 1024, 128), tc::f_to_h8(f));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------------------------------------------------------- Y = KI^T T, Z = P T
    if (ok) {
        if (tid == 0) {               // Y
            const uint32_t idY = idesc_f16(128, 64, true, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(t0 + 64, sdesc_sw128(base + kKI + kk * 2048, 8192, 1024), sdesc(base + kT16 + kk * 2048, 1024, 128),
                        idY, kk > 0);
            mma_commit(bar_mma);
        } else if (tid == 32) {       // Z
            const uint32_t idZ = idesc_f16(64, 64, false, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(t0 + 128, sdesc(base + kP16 + kk * 256, 128, 1024), sdesc(base + kT16 + kk * 2048, 1024, 128),
                        idZ, kk > 0);
            mma_commit(bar_mma2);
        }
        ok = mbar_wait(bar_mma, phase) && mbar_wait(bar_mma2, phase);
        phase ^= 1u;
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) tc::record_timeout(p.status);
    tc_fence_after();
    if (ok) {
        const int q = warp & 3, chh = warp >> 2;
        const uint32_t lb = (uint32_t)(32 * q) << 16;
        float d[32], dz[32];
        tmem_ld32_async(t0 + lb + 64 + 32 * chh, d);
        tmem_ld32_async(t0 + lb + 128 + 32 * chh, dz);
        tmem_ld_wait2(d, dz);
        {   // Y (M = 128): row = channel, 32 columns per warp -> A operand (K-major) over A32
            const int cc = 32 * q + lane;
#pragma unroll
            for (int j = 0; j < 4; ++j) tc::st16(sm + kA32, off_kmajor(cc, 32 * chh + 8 * j, 1024, 128), tc::f_to_h8(d + 8 * j));
        }
        {   // Z (M = 64: row r in lane (r % 16) + 32 (r / 16)) -> A operand (K-major (m = r, k = r'),
            // SBO 1024, LBO 128) over T16, and again over P16 (free once Z = P T is done): the
            // products with Z then run at M = 128 with rows 64-127 repeating rows 0-63, so that their
            // epilogues use every lane
            if (lane < 16) {
                const int r = 16 * q + lane;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 h = tc::f_to_h8(dz + 8 * j);
                    tc::st16(sm + kT16, off_kmajor(r, 32 * chh + 8 * j, 1024, 128), h);
                    tc::st16(sm + kP16, off_kmajor(r, 32 * chh + 8 * j, 1024, 128), h);
                }
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------------------------------------------------------- N~ = Y KG, Qe~ = QG - Z KG
    if (ok) {
        if (tid == 0) {               // N~ = Y KG
            const uint32_t idN = idesc_f16(128, 128, false, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(t0 + 0, sdesc(base + kA32 + kk * 256, 128, 1024), sdesc_sw128(base + kKQ + kk * 2048, 16384, 1024),
                        idN, kk > 0);
            mma_commit(bar_mma);
        } else if (tid == 32) {       // -Z KG (M = 64; the epilogue adds QG)
            const uint32_t idQn = idesc_f16(128, 128, false, true, true);   // [Z; Z]
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(t0 + 128, sdesc(base + kT16 + kk * 256, 128, 1024), sdesc_sw128(base + kKQ + kk * 2048, 16384, 1024),
                        idQn, kk > 0);
            mma_commit(bar_mma2);
        }
        ok = mbar_wait(bar_mma, phase) && mbar_wait(bar_mma2, phase);
        phase ^= 1u;
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) tc::record_timeout(p.status);
    tc_fence_after();
    if (ok) {
        const int q = warp & 3, chh = warp >> 2;
        const uint32_t lb = (uint32_t)(32 * q) << 16;
        {   // N = -diag(row) N~ diag(col) -> block (K-major (m = i, k = c): SBO 2048, LBO 128)
            const int cc = 32 * q + lane;
            const float rs = -trow[cc];
            auto emit = [&](float (&x)[32], int c0) {
#pragma unroll
                for (int e4 = 0; e4 < 32; e4 += 4) {
                    const float4 cs = *reinterpret_cast<const float4*>(tcol + c0 + e4);
                    x[e4] *= rs * cs.x; x[e4 + 1] *= rs * cs.y; x[e4 + 2] *= rs * cs.z; x[e4 + 3] *= rs * cs.w;
                }
#pragma unroll
                for (int g8 = 0; g8 < 32; g8 += 8)
                    *reinterpret_cast<uint4*>(blk + tc::kOffN + off_kmajor(cc, c0 + g8, 2048, 128)) = tc::f_to_h8(x + g8);
            };
            float xa[32], xb[32];
            tmem_ld32_async(t0 + lb + 64 * chh, xa);
            tmem_ld32_async(t0 + lb + 64 * chh + 32, xb);
            tmem_ld_wait2(xa, xb);
            emit(xa, 64 * chh);
            emit(xb, 64 * chh + 32);
        }
        // Qe = (QG - Z KG) diag(col) -> block (K-major (m = r, k = c): SBO 2048, LBO 128).  The
        // product ran at M = 128 with rows repeated, so row r sits in lanes r and 64 + r: warp
        // (q, chh) takes rows 32 (q % 2) .. +31 and the 32 columns of quarter q / 2 + 2 chh.
        {
            auto emit = [&](float (&x)[32], int c0) {
                const int r = 32 * (q & 1) + lane;
#pragma unroll
                for (int g8 = 0; g8 < 32; g8 += 8) {
                    float qg[8];
                    tc::h8_to_f(*reinterpret_cast<const uint4*>(sm + kKQ + 8192 + sw128_off(r, c0 + g8, 16384)), qg);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[g8 + e] += qg[e];
                }
#pragma unroll
                for (int e4 = 0; e4 < 32; e4 += 4) {
                    const float4 cs = *reinterpret_cast<const float4*>(tcol + c0 + e4);
                    x[e4] *= cs.x; x[e4 + 1] *= cs.y; x[e4 + 2] *= cs.z; x[e4 + 3] *= cs.w;
                }
#pragma unroll
                for (int g8 = 0; g8 < 32; g8 += 8)
                    *reinterpret_cast<uint4*>(blk + tc::kOffQe + off_kmajor(r, c0 + g8, 2048, 128)) = tc::f_to_h8(x + g8);
            };
            const int c0 = 32 * ((q >> 1) + 2 * chh);
            float x[32];
            tmem_ld32(t0 + lb + 128 + c0, x);
            emit(x, c0);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---------------------------------------------------------------- b~ = Y V, PU' = Z V
    if (ok) {
        if (tid == 0) {               // b~ = Y V
            const uint32_t idN = idesc_f16(128, 128, false, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(t0 + 0, sdesc(base + kA32 + kk * 256, 128, 1024), sdesc_sw128(base + kV + kk * 2048, 8192, 1024),
                        idN, kk > 0);
            mma_commit(bar_mma);
        } else if (tid == 32) {       // PU' = Z V
            const uint32_t idP = idesc_f16(128, 128, false, true);           // [Z; Z]
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(t0 + 128, sdesc(base + kT16 + kk * 256, 128, 1024), sdesc_sw128(base + kV + kk * 2048, 8192, 1024),
                        idP, kk > 0);
            mma_commit(bar_mma2);
        }
        ok = mbar_wait(bar_mma, phase) && mbar_wait(bar_mma2, phase);
        phase ^= 1u;
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) tc::record_timeout(p.status);
    tc_fence_after();
    if (ok) {                    // b = diag(row) b~ -> block (fp16 group-major slices, one per load)
        const int q = warp & 3, chh = warp >> 2;
        const int cc = 32 * q + lane;
        const float rs = trow[cc];
        const uint32_t lb = (uint32_t)(32 * q) << 16;
        auto emit = [&](float (&x)[32], int c0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                x[e] *= rs;
                vmax = fmax_nan(vmax, fabsf(x[e]));
            }
            __half* bb = reinterpret_cast<__half*>(blk + tc::kOffB) + (size_t)(c0 / NS) * D * NS;
#pragma unroll
            for (int g8 = 0; g8 < 32; g8 += 8) *reinterpret_cast<uint4*>(bb + tc::grp_half(cc, g8, D)) = tc::f_to_h8(x + g8);
        };
        float xa[32], xb[32];
        tmem_ld32_async(t0 + lb + 64 * chh, xa);
        tmem_ld32_async(t0 + lb + 64 * chh + 32, xb);
        tmem_ld_wait2(xa, xb);
        emit(xa, 64 * chh);
        emit(xb, 64 * chh + 32);
    }
    if (ok) {   // PU' (M = 128, rows repeated; the Qe epilogue's warp split) -> block (fp16 group-major slices)
        const int q = warp & 3, chh = warp >> 2;
        const uint32_t lb = (uint32_t)(32 * q) << 16;
        auto emit = [&](float (&x)[32], int c0) {
            const int r = 32 * (q & 1) + lane;
            __half* pu = reinterpret_cast<__half*>(blk + tc::kOffPU) + (size_t)(c0 / NS) * C * NS;
#pragma unroll
            for (int e = 0; e < 32; ++e) vmax = fmax_nan(vmax, fabsf(x[e]));
#pragma unroll
            for (int g8 = 0; g8 < 32; g8 += 8) *reinterpret_cast<uint4*>(pu + tc::grp_half(r, g8, C)) = tc::f_to_h8(x + g8);
        };
        const int c0 = 32 * ((q >> 1) + 2 * chh);
        float x[32];
        tmem_ld32(t0 + lb + 128 + c0, x);
        emit(x, c0);
    }
    if (tid < D) reinterpret_cast<float*>(blk + tc::kOffGC)[tid] = tgam[tid];
    tc_fence_before();
    // NaN compares false: a NaN input is reported too
    if (__syncthreads_or(!(vmax <= kFp16Max)) && tid == 0) atomicCAS(p.status, kDevOk, kDevRange);
    if (warp == 0) tmem_dealloc(t0, 256);
}

// ---------------------------------------------------------------- host side: tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, nullptr) == cudaSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// [B, T, H, 128] bf16 viewed as the 4-D tensor (channel, head, token, batch); boxes of 64 channels
// x 1 head x 64 tokens, 128-byte swizzle, zeros past the end.
bool make_map(CUtensorMap* m, const void* ptr, const Problem& p) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)p.H, (cuuint64_t)p.T, (cuuint64_t)p.B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)p.H * D * 2, (cuuint64_t)p.T * p.H * D * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// DeltaProduct k or v, [B, T, H, n_h, 128] bf16, as the 5-D tensor (channel, step, head, token,
// batch); boxes of 64 channels x n_h steps x 1 head x 64 / n_h tokens: one chunk of sub-steps.
bool make_map_dp(CUtensorMap* m, const void* ptr, const Problem& p) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t nh = (cuuint64_t)p.nh;
    const cuuint64_t dims[5] = {(cuuint64_t)D, nh, (cuuint64_t)p.H, (cuuint64_t)p.T, (cuuint64_t)p.B};
    const cuuint64_t strides[4] = {(cuuint64_t)D * 2, nh * D * 2, (cuuint64_t)p.H * nh * D * 2,
                                   (cuuint64_t)p.T * p.H * nh * D * 2};
    const cuuint32_t box[5] = {64, (cuuint32_t)p.nh, 1, (cuuint32_t)(C / p.nh), 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc2

// Usable for this problem: bf16 FG^2-GDN / FG^2-GDN+ / KDA / GDN / DeltaNet, and DeltaProduct
// with n_h dividing the chunk, with chunk 64, dk = dv = 128 (not GDN2).
bool tc2_usable(const Problem& p) {
    return !p.gdn2_eta && (!p.dp || tc::C % p.nh == 0) && tc2::encode_fn() != nullptr;
}

// Intra role over chunks [cb, cb + n) of every head.
cudaError_t launch_intra_tma(const Problem& p, int cb, int n, cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    if (p.dp) {
        mq = CUtensorMap{};
        if (!tc2::make_map_dp(&mk, p.k, p) || !tc2::make_map_dp(&mv, p.v, p)) return cudaErrorInvalidValue;
    } else if (!tc2::make_map(&mq, p.q, p) || !tc2::make_map(&mk, p.k, p) || !tc2::make_map(&mv, p.v, p)) {
        return cudaErrorInvalidValue;
    }
    auto kern = p.dp ? tc2::intra_tma_kernel<false, true>
              : (p.beta_v ? tc2::intra_tma_kernel<true, false> : tc2::intra_tma_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc2::kSmem);
    if (e != cudaSuccess) return e;
    const int hf = n <= 65535 ? 1 : 0;                 // grid y is at most 65535
    kern<<<hf ? dim3(p.B * p.H, n) : dim3(n, p.B * p.H), tc2::NT, tc2::kSmem, stream>>>(p, cb, hf, mq, mk, mv);
    return cudaGetLastError();
}

}  // namespace gdn
