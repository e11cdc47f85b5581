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
// The intra kernel also forms N = -K'^T W and b = K'^T U', so the chunk update
// S <- Diag(gC) S + K'^T (U' - W S) becomes S <- Diag(gC) S + N S + b: one
// tensor-core product per chunk on the serial path.
//
// scan_tc_kernel<W>: one CTA per (head, W 32-column slices of d_v; W = 1, or 2 when
// one slice per CTA would need more than one wave of SMs), serial over the chunks of
// its range.  Per chunk: D_S = N S (M = 128, the chain), then
// S <- Diag(gC) S + D_S + b in fp32 registers (one d_k row per thread; the fp16
// copy is the next B operand); off the chain, D_O = Qe S (M = 64) and
// O = D_O + PU'.  A producer warp streams the per-chunk blocks with bulk async
// copies into two rings, one thread issues every MMA, and all hand-offs are
// bounded mbarrier waits.
//
// launch_tc cuts long sequences into chunk ranges: intra of range s+1 runs on
// the caller's stream while the scan of range s runs on the side stream.
#include <cstdlib>
#include <mutex>

#include "gdn_tc_common.cuh"

namespace gdn {
using namespace sm100;

namespace tc {

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
constexpr uint32_t kBar = 112128;        // mbarrier (MMA completion)
constexpr uint32_t kBarK = 112144;       // mbarrier (K' reload)
constexpr uint32_t kTmem = 112136;       // TMEM base address
constexpr uint32_t kEgr = 112192;        // e^{g_ref} [128]
constexpr uint32_t kIntraSmem = 112704;
static_assert(2 * (kIntraSmem + 1024) <= 228 * 1024, "two intra CTAs per SM (1 KB reserved each)");

constexpr uint32_t kTmemCols = 256;
// TMEM columns: D0 / D3 at 0, D1 (W~^T) at 64, D2 (U'^T) at 128, D4 (PU'^T) at 192.

// ============================================================================ intra
// kPlus: FG^2-GDN+ (separate value rate beta^v, eq. (13)).
// kG2: GDN2 (Su Jianlin's GDN2 stability note): the A rows and the state read use the erase
// vector j' = eta k^ (.) b after the token-wise transform, the write vector is k^, and v is
// scaled by eta; everything after the prep is the tied computation.
template <bool kPlus, bool kG2 = false>
__global__ void __launch_bounds__(NT, 2) intra_tc_kernel(Problem p, int cb) {
    extern __shared__ __align__(1024) uint8_t sm[];
    const int c = cb + blockIdx.x;             // this launch covers chunks cb .. cb + gridDim.x - 1
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int s0 = c * C;
    const int Cv = min(C, p.L - s0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (!GDN_IN_BOUNDS(c < p.NC && bh < p.B * p.H, p.status)) return;   // the whole CTA, before any barrier
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
    uint64_t* bark = reinterpret_cast<uint64_t*>(sm + kBarK);
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bark, 1);
        fence_mbar_init();
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
    const bool a_scalar = p.dp || p.alpha_scalar;
    const bool b_scalar = p.dp || p.beta_scalar;
    // beta (channel-wise) and v go to shared memory with register-free async copies: beta
    // into a staging area over R3..R6 (free until the solve), v straight into its final
    // place in R2 (converted in place later).  Everything is issued before any arithmetic.
    float* bstage = reinterpret_cast<float*>(sm + kR3);
    // half h of octet o of row rr in the staging area: 16-byte units XOR-swizzled by the row,
    // so eight consecutive rows reading the same unit hit eight different bank groups
    auto bst = [bstage](int rr_, int o_, int h_) { return bstage + (rr_ * 32 + ((2 * o_ + h_) ^ (rr_ & 7))) * 4; };
    // Without beta^v, raw q and k also go to shared memory, into the R0 slots this thread
    // later overwrites with its own QG and KG octets; they are the first commit group, so
    // the norms wait for them alone.  (Holding them in registers through the norm and
    // prefix phases costs 32 registers and forces spills.)
    // With beta^v (which takes the R0 slots), raw k goes to this thread's R1 slots (later
    // its KIG octets) and only q stays in registers.
    {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int o = o0 + 4 * j;
            uint8_t* kdst = kPlus ? sm + kR1 + off_kmajor(r, 8 * o, 2048, 128)
                                  : sm + kR0 + off_kmajor(r, 8 * o, 2048, 128);
            if (valid) cp_async16(kdst, k + krow * D + 8 * o);
            else *reinterpret_cast<uint4*>(kdst) = make_uint4(0, 0, 0, 0);
            if (!kPlus) {
                uint8_t* qdst = sm + kR0 + off_kmajor(64 + r, 8 * o, 2048, 128);
                if (valid && rr.has_q) cp_async16(qdst, q + rr.tok * D + 8 * o);
                else *reinterpret_cast<uint4*>(qdst) = make_uint4(0, 0, 0, 0);
            }
        }
        cp_async_commit();
    }
    if (valid) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int o = o0 + 4 * j;
            if (!b_scalar) {      // beta, or GDN2's gate b (always channel-wise)
                const float* bsrc = kG2 ? p.gdn2_b : p.beta;
                cp_async16(bst(r, o, 0), bsrc + rr.tok * D + 8 * o);
                cp_async16(bst(r, o, 1), bsrc + rr.tok * D + 8 * o + 4);
            }
            cp_async16(sm + kR2 + off_kmajor(r, 8 * o, 2048, 128), v + krow * D + 8 * o);
            if (kPlus && !b_scalar) {
                // beta^v of (r, o) goes to the two R0 slots this thread later overwrites
                // with its own KG and QG octets (read first, in the same thread)
                cp_async16(sm + kR0 + off_kmajor(r, 8 * o, 2048, 128), p.beta_v + rr.tok * D + 8 * o);
                cp_async16(sm + kR0 + off_kmajor(64 + r, 8 * o, 2048, 128), p.beta_v + rr.tok * D + 8 * o + 4);
            }
        }
    }
    cp_async_commit();
    uint4 qp[4], kp[4];
    float4 al0[4], al1[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = o0 + 4 * j;
        if (kPlus) qp[j] = (valid && rr.has_q) ? ldg16(q + rr.tok * D + 8 * o) : make_uint4(0, 0, 0, 0);
        if (valid && !a_scalar) {
            al0[j] = ldg16f(p.alpha + rr.tok * D + 8 * o);
            al1[j] = ldg16f(p.alpha + rr.tok * D + 8 * o + 4);
        } else {
            al0[j] = make_float4(1.f, 1.f, 1.f, 1.f);
            al1[j] = al0[j];
        }
    }
    cp_async_wait_group<1>();      // raw k (and q without beta^v), the older group, has landed
    float ssq = 0.f, ssk = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = o0 + 4 * j;
        float fq[8], fk[8];
        if (!kPlus) qp[j] = *reinterpret_cast<const uint4*>(sm + kR0 + off_kmajor(64 + r, 8 * o, 2048, 128));
        kp[j] = *reinterpret_cast<const uint4*>(sm + (kPlus ? kR1 : kR0) + off_kmajor(r, 8 * o, 2048, 128));
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

    float la_s = 0.f, b_s = 0.f, bv_s = 0.f;
    if (valid) {
        if (p.dp) {
            la_s = rr.m == 0 ? __logf(p.alpha[rr.tok]) : 0.f;
            b_s = p.beta[rr.tok * p.nh + rr.m];
        } else {
            if (p.alpha_scalar) la_s = __logf(p.alpha[rr.tok]);
            if (p.beta_scalar) b_s = p.beta[rr.tok];
            if (kPlus && p.beta_scalar) bv_s = p.beta_v[rr.tok];
        }
    }
    // GDN2 row quantities: c = j'^T k^, ||j'||^2 and max alpha over the row's 4 lanes, then
    // the transform: the clip bound on log alpha (mode 1) or the shrink factor (mode 2).
    float g2_eta = 0.f, g2_c = 0.f, g2_lam = 1.f, g2_lr = 0.f;
    if constexpr (kG2) {
        cp_async_wait_all();       // the gate b has landed (this thread's own slots)
        float cd = 0.f, nj = 0.f, am = 0.f;
        if (valid) {
            g2_eta = p.gdn2_eta[rr.tok];
            const float as_ = a_scalar ? p.alpha[rr.tok] : 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int o = o0 + 4 * j;
                const float* blo = bst(r, o, 0);
                const float* bhi = bst(r, o, 1);
                float fk[8];
                bf8_to_f(kp[j], fk);
                const float a8[8] = {al0[j].x, al0[j].y, al0[j].z, al0[j].w, al1[j].x, al1[j].y, al1[j].z, al1[j].w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float kh = fk[e] * ik;
                    const float jp = g2_eta * kh * (e < 4 ? blo[e] : bhi[e - 4]);
                    cd += jp * kh;
                    nj += jp * jp;
                    am = fmaxf(am, a_scalar ? as_ : a8[e]);
                }
            }
        }
        cd += __shfl_xor_sync(0xffffffffu, cd, 8);
        cd += __shfl_xor_sync(0xffffffffu, cd, 16);
        nj += __shfl_xor_sync(0xffffffffu, nj, 8);
        nj += __shfl_xor_sync(0xffffffffu, nj, 16);
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 8));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 16));
        g2_c = cd;
        if (valid && p.gdn2_mode == 1) {          // D -> min(D, 1/rho)
            const float rho = 0.5f * (sqrtf(nj) + sqrtf(fmaxf(nj - 4.f * cd + 4.f, 0.f)));
            g2_lr = -__logf(rho);
        }
        if (valid && p.gdn2_mode == 2) {          // j* = c k + lambda* (j' - c k)
            const float tau = (cd - 1.f) * am + 1.f / am;
            const float den = nj - cd * cd;
            g2_lam = den > 0.f ? fminf(1.f, sqrtf(fmaxf(tau * tau - cd * cd, 0.f) / den)) : 1.f;
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
            const float4 a0 = al0[j], a1 = al1[j];
            la[j][0] = __logf(a0.x); la[j][1] = __logf(a0.y); la[j][2] = __logf(a0.z); la[j][3] = __logf(a0.w);
            la[j][4] = __logf(a1.x); la[j][5] = __logf(a1.y); la[j][6] = __logf(a1.z); la[j][7] = __logf(a1.w);
        }
        if (kG2 && valid && p.gdn2_mode == 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) la[j][e] = fminf(la[j][e], g2_lr);
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
        reinterpret_cast<float*>(sm + kEgr)[tid] = __expf(gr);
        reinterpret_cast<float*>(blk + kOffGC)[tid] = __expf(glast[tid]);
    }
    __syncthreads();

    // per octet: the fp16 operands
    float* fb_g = reinterpret_cast<float*>(blk + kOffB);                  // fallback scratch: g fp32 [C][D]
    __half* fb_k = reinterpret_cast<__half*>(blk + kOffPU);               // k~ fp16 [C][D]
    __half* fb_q = reinterpret_cast<__half*>(blk + kOffN);                // q^ fp16 [C][D]
    __half* fb_e = fb_q + C * D;                                          // GDN2 erase fp16 [C][D]
    cp_async_wait_all();     // this thread's own staged beta and v
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = o0 + 4 * j;
        float g[8], sb[8], sv[8], fq[8], fk[8], fv[8], gb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = la[j][e] + scr[warp * D + 8 * o + e];
        if (kG2) {                // no beta: k~ = k^; the gate b feeds the erase vector
            const float* blo = bst(r, o, 0);
            const float* bhi = bst(r, o, 1);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                sb[e] = valid ? 1.f : 0.f;
                gb[e] = valid ? (e < 4 ? blo[e] : bhi[e - 4]) : 0.f;
            }
        } else if (b_scalar || !valid) {
            const float s = valid ? sqrtf(b_s) : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) sb[e] = s;
        } else {
            const float4 b0 = *reinterpret_cast<const float4*>(bst(r, o, 0));
            const float4 b1 = *reinterpret_cast<const float4*>(bst(r, o, 1));
            sb[0] = sqrt_op(b0.x); sb[1] = sqrt_op(b0.y); sb[2] = sqrt_op(b0.z); sb[3] = sqrt_op(b0.w);
            sb[4] = sqrt_op(b1.x); sb[5] = sqrt_op(b1.y); sb[6] = sqrt_op(b1.z); sb[7] = sqrt_op(b1.w);
        }
        if (kG2) {
#pragma unroll
            for (int e = 0; e < 8; ++e) sv[e] = g2_eta;
        } else if (!kPlus) {
#pragma unroll
            for (int e = 0; e < 8; ++e) sv[e] = sb[e];
        } else if (b_scalar || !valid) {
            const float s = valid ? sqrtf(bv_s) : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) sv[e] = s;
        } else {
            const float4 b0 = *reinterpret_cast<const float4*>(sm + kR0 + off_kmajor(r, 8 * o, 2048, 128));
            const float4 b1 = *reinterpret_cast<const float4*>(sm + kR0 + off_kmajor(64 + r, 8 * o, 2048, 128));
            sv[0] = sqrt_op(b0.x); sv[1] = sqrt_op(b0.y); sv[2] = sqrt_op(b0.z); sv[3] = sqrt_op(b0.w);
            sv[4] = sqrt_op(b1.x); sv[5] = sqrt_op(b1.y); sv[6] = sqrt_op(b1.z); sv[7] = sqrt_op(b1.w);
        }
        const uint4 vp = valid ? *reinterpret_cast<const uint4*>(sm + kR2 + off_kmajor(r, 8 * o, 2048, 128))
                               : make_uint4(0, 0, 0, 0);
        // reread from shared memory: not held in registers across the phases
        if (!kPlus) qp[j] = *reinterpret_cast<const uint4*>(sm + kR0 + off_kmajor(64 + r, 8 * o, 2048, 128));
        kp[j] = *reinterpret_cast<const uint4*>(sm + (kPlus ? kR1 : kR0) + off_kmajor(r, 8 * o, 2048, 128));
        bf8_to_f(qp[j], fq);
        bf8_to_f(kp[j], fk);
        bf8_to_f(vp, fv);
        float KG[8], QG[8], KIG[8], VT[8], KP[8], KT[8], QH[8], EJ[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int ch = 8 * o + e;
            const float gr = gref[ch];
            const float ex = __expf(g[e] - gr);
            const float exi = __expf(gr - g[e]);
            const float kt = fk[e] * ik * sb[e];
            const float qh = fq[e] * iq;
            // the erase (A-row, state-read) vector: k~ itself, or GDN2's j' (shrunk in mode 2)
            float er = kt;
            if (kG2) {
                const float jp = g2_eta * kt * gb[e];
                er = g2_lam * jp + (1.f - g2_lam) * g2_c * kt;
            }
            EJ[e] = er;
            KT[e] = kt;
            QH[e] = qh;
            KG[e] = er * ex;
            QG[e] = qh * ex;
            KIG[e] = kt * exi;
            VT[e] = fv[e] * sv[e];
            KP[e] = KIG[e] * fK[ch];
        }
        if (fallback) {          // CTA-uniform: keeps the extra exponent off the common path
            // e^{-g} may overflow while e^{g_last} underflows there, so take the ratio in one
            // exponent (it is <= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) KP[e] = KT[e] * __expf(glast[8 * o + e] - g[e]);
        }
        const uint32_t off = off_kmajor(r, 8 * o, 2048, 128);
        st16(sm + kR0, off, f_to_h8(KG));
        st16(sm + kR0, off_kmajor(64 + r, 8 * o, 2048, 128), f_to_h8(QG));
        st16(sm + kR1, off, f_to_h8(KIG));
        st16(sm + kR2, off, f_to_h8(VT));
        *reinterpret_cast<uint4*>(blk + kOffKp + off_mnmajor(8 * o, r, 1024, 128)) = f_to_h8(KP);
        if (fallback) {
#pragma unroll
            for (int e = 0; e < 8; ++e) fb_g[r * D + 8 * o + e] = g[e];
            *reinterpret_cast<uint4*>(fb_k + r * D + 8 * o) = f_to_h8(KT);
            *reinterpret_cast<uint4*>(fb_q + r * D + 8 * o) = f_to_h8(QH);
            if (kG2) *reinterpret_cast<uint4*>(fb_e + r * D + 8 * o) = f_to_h8(EJ);
        }
    }
    fence_async_smem();
    asm volatile("fence.proxy.async.global;" ::: "memory");   // K' is read back by a bulk copy
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = *tslot;
    bool ok = true;
    uint32_t phase = 0;      // parity of the next completion of `bar`
    // identity operand (B layout: n = r, k = i); its area held staged beta until now.
    // Eight consecutive lanes take eight consecutive rows: one 128-byte line per store phase.
    for (int idx = tid; idx < 512; idx += NT) {
        const int ri = idx & 63, j = idx >> 6;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = (8 * j + e == ri) ? 1.f : 0.f;
        st16(sm + kR5, off_kmajor(ri, 8 * j, 1024, 128), f_to_h8(f));
    }

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
                const float xr = __half2float(isP ? fb_q[rowr * D + ch]
                                                  : (kG2 ? fb_e[rowr * D + ch] : fb_k[rowr * D + ch]));
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
    // Blocked forward substitution in fp32: four 16x16 diagonal blocks in registers
    // (lane j carries column j; row r of A is a broadcast shared-memory read, which
    // does not depend on the running solution and so issues ahead of it; fetching it
    // from other lanes by shuffles ran as fast here but depended on how the compiler
    // ordered the exchanges -- one instrumented build ran that loop ~15x slower), then
    // T10 = -T11 A10 T00 on 16x16 and 32x32 blocks.
    if (warp < 4) {
        const int bb = 16 * warp, jc = lane & 15;
        float t[16];
#pragma unroll
        for (int r2 = 0; r2 < 16; ++r2) {
            float acc = (r2 == jc) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < r2; ++i) acc -= A32[sw64(bb + r2, bb + i)] * t[i];
            t[r2] = acc;
        }
        if (lane < 16) {
#pragma unroll
            for (int r2 = 0; r2 < 16; ++r2) T32[sw64(bb + r2, bb + jc)] = t[r2];
        }
    } else {
        // zero the upper off-diagonal blocks the merges read: (0..15, 16..31), (32..47, 48..63)
        const int u = tid - 128;
        const int blk2 = u >> 6, e = (u & 63) * 4;
        const int r0 = blk2 ? 32 : 0, c0 = blk2 ? 48 : 16;
        *reinterpret_cast<float4*>(T32 + sw64(r0 + (e >> 4), c0 + (e & 15))) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    {   // 16x16 merges for the block pairs (16..31 | 0..15) and (48..63 | 32..47)
        const int m = tid >> 7, qd = tid & 127;
        const int rw = qd >> 3, j2 = (qd & 7) * 2;
        const int base = 32 * m;
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = A32[sw64(base + 16 + rw, base + i)];
            x0 = fmaf(a, T32[sw64(base + i, base + j2)], x0);
            x1 = fmaf(a, T32[sw64(base + i, base + j2 + 1)], x1);
        }
        scr[m * 256 + rw * 16 + j2] = x0;
        scr[m * 256 + rw * 16 + j2 + 1] = x1;
        __syncthreads();
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int mm = 0; mm < 16; ++mm) {
            const float tt = T32[sw64(base + 16 + rw, base + 16 + mm)];
            y0 = fmaf(tt, scr[m * 256 + mm * 16 + j2], y0);
            y1 = fmaf(tt, scr[m * 256 + mm * 16 + j2 + 1], y1);
        }
        T32[sw64(base + 16 + rw, base + j2)] = -y0;
        T32[sw64(base + 16 + rw, base + j2 + 1)] = -y1;
    }
    __syncthreads();
    {   // 32x32 merge: T_BL = -T_BR (A_BL T_TL)
        const int rw = tid >> 3, j4 = (tid & 7) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            const float a = A32[sw64(32 + rw, i)];
            const float4 tv = *reinterpret_cast<const float4*>(T32 + sw64(i, j4));
            x.x = fmaf(a, tv.x, x.x); x.y = fmaf(a, tv.y, x.y); x.z = fmaf(a, tv.z, x.z); x.w = fmaf(a, tv.w, x.w);
        }
        *reinterpret_cast<float4*>(scr + rw * 32 + j4) = x;
        __syncthreads();
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int mm = 0; mm < 32; ++mm) {
            const float tt = T32[sw64(32 + rw, 32 + mm)];
            const float4 xv = *reinterpret_cast<const float4*>(scr + mm * 32 + j4);
            y.x = fmaf(tt, xv.x, y.x); y.y = fmaf(tt, xv.y, y.y); y.z = fmaf(tt, xv.z, y.z); y.w = fmaf(tt, xv.w, y.w);
        }
        *reinterpret_cast<float4*>(T32 + sw64(32 + rw, j4)) = make_float4(-y.x, -y.y, -y.z, -y.w);
    }
    __syncthreads();
    for (int idx = tid; idx < 512; idx += NT) {   // T -> fp16 B operand (n = r, k = i)
        // eight consecutive lanes take eight consecutive rows: the swizzled float4 reads and
        // the 16-byte stores both fall in distinct bank groups
        const int rw = idx & 63, j = idx >> 6;
        const float4 ta = *reinterpret_cast<const float4*>(T32 + sw64(rw, 8 * j));
        const float4 tb = *reinterpret_cast<const float4*>(T32 + sw64(rw, 8 * j + 4));
        float f[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (8 * j + e > rw) f[e] = 0.f;
        st16(sm + kR3, off_kmajor(rw, 8 * j, 1024, 128), f_to_h8(f));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // reload K' (written by the prep) into R1 as the A operand of the N and b products
    if (ok && tid == 0) {
        mbar_arrive_expect_tx(bark, 16384);
        bulk_g2s(sm + kR1, blk + kOffKp, 16384, bark);
    }

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
    if (ok) {   // warps 0-3: W~^T -> R0 (K-major (c, r)); warps 4-7: U'^T -> R2 (K-major (j, r))
        const int ch = 32 * (warp & 3) + lane;
        const uint32_t lanebase = t0 + ((uint32_t)(32 * (warp & 3)) << 16);
        const uint32_t col = warp < 4 ? 64 : 128;
        uint8_t* dst = sm + (warp < 4 ? kR0 : kR2);
        float x0[32], x1[32];
        tmem_ld32(lanebase + col, x0);
        tmem_ld32(lanebase + col + 32, x1);
#pragma unroll
        for (int i0 = 0; i0 < C; i0 += 8) st16(dst, off_kmajor(ch, i0, 128, 2048), f_to_h8((i0 < 32 ? x0 : x1) + (i0 & 31)));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------------------------------------------------------- (Qe e^{-g_ref})^T, PU'^T, N~ = -K'^T W~
    if (ok) {
        const bool kok = mbar_wait(bark, 0);
        if (tid == 0) {
            if (kok) {
                tc_fence_after();
                mma_f16_k(t0 + 0, smem_u32(sm + kR0), 2048, 128, smem_u32(sm + kR4), 128, 1024,
                          idesc_f16(128, 64, false, false, true), C, false);
                mma_f16_k(t0 + 0, smem_u32(sm + kR0 + 16384), 2048, 128, smem_u32(sm + kR5), 128, 1024,
                          idesc_f16(128, 64, true, false), C, true);
                mma_f16_k(t0 + 192, smem_u32(sm + kR2), 2048, 128, smem_u32(sm + kR4), 128, 1024,
                          idesc_f16(128, 64, false, false), C, false);
                mma_f16_k(t0 + 64, smem_u32(sm + kR1), 128, 1024, smem_u32(sm + kR0), 2048, 128,
                          idesc_f16(128, 128, true, false, true), C, false);
                mma_commit(bar);
            }
        }
        ok = kok && mbar_wait(bar, phase);
        phase ^= 1u;
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) record_timeout(p.status);
    tc_fence_after();
    if (ok && warp < 4) {        // Qe -> block (MN-major (r, c)); PU' -> block (fp16, sw rows)
        const int ch = 32 * warp + lane;
        const float er = reinterpret_cast<const float*>(sm + kEgr)[ch];
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
            *reinterpret_cast<uint4*>(blk + kOffQe + off_mnmajor(r0, ch, 2048, 128)) = f_to_h8(f);
        }
        tmem_ld32(lanebase + 192, x0);
        tmem_ld32(lanebase + 224, x1);
        // Warp w holds PU' slice w (its 32 channels, all rows): build the slice's block image
        // in the dead T32 area (R6), then copy it out as 16-byte vectors.
        __half* st = reinterpret_cast<__half*>(sm + kR6 + warp * (C * NS * 2));
#pragma unroll
        for (int r2 = 0; r2 < C; ++r2) st[sw_half(r2, lane)] = __float2half_rn(r2 < 32 ? x0[r2] : x1[r2 - 32]);
        __syncwarp();
        const uint4* srcv = reinterpret_cast<const uint4*>(st);
        uint4* dstv = reinterpret_cast<uint4*>(blk + kOffPU + warp * (C * NS * 2));
#pragma unroll
        for (int i = 0; i < C * NS * 2 / 16 / 32; ++i) dstv[lane + 32 * i] = srcv[lane + 32 * i];
    } else if (ok) {             // N = N~ * e^{g_ref[c]} (column scale) -> block (K-major (i, c))
        const int row = 32 * (warp & 3) + lane;
        const uint32_t lanebase = t0 + ((uint32_t)(32 * (warp & 3)) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
            float x[32];
            tmem_ld32(lanebase + 64 + c0, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] *= reinterpret_cast<const float*>(sm + kEgr)[c0 + e];
#pragma unroll
            for (int g8 = 0; g8 < 32; g8 += 8)
                *reinterpret_cast<uint4*>(blk + kOffN + off_kmajor(row, c0 + g8, 2048, 128)) = f_to_h8(x + g8);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------------------------------------------------------- b = K'^T U'
    if (ok) {
        if (tid == 0) {
            mma_f16_k(t0 + 0, smem_u32(sm + kR1), 128, 1024, smem_u32(sm + kR2), 2048, 128,
                      idesc_f16(128, 128, true, false), C, false);
            mma_commit(bar);
        }
        ok = mbar_wait(bar, phase);
        phase ^= 1u;
    }
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) record_timeout(p.status);
    tc_fence_after();
    if (ok) {                    // warps 0-3: columns 0-63, warps 4-7: columns 64-127
        const int row = 32 * (warp & 3) + lane;
        const uint32_t lanebase = t0 + ((uint32_t)(32 * (warp & 3)) << 16);
        const int cbase = warp < 4 ? 0 : 64;
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
            float x[32];
            tmem_ld32(lanebase + cbase + c0, x);
            const int j0 = cbase + c0;                  // one full 32-column slice
            __half* bb = reinterpret_cast<__half*>(blk + kOffB) + (size_t)(j0 / NS) * D * NS;
#pragma unroll
            for (int g8 = 0; g8 < 32; g8 += 8)
                *reinterpret_cast<uint4*>(bb + sw_half(row, g8)) = f_to_h8(x + g8);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t0, kTmemCols);
}

// ============================================================================ scan
// One CTA per (head, W consecutive 32-column slices).  Per chunk c, with S_c in fp32
// registers (row i per thread, 32 columns per warp) and its fp16 copy in Sop[c % 3]:
//   MMA_S: D_S = N_c S_c          -> S_{c+1} = Diag(gC) S_c + D_S + b_c   (the serial chain)
//   MMA_O: D_O[c & 1] = Qe_c S_c  -> O_c = D_O + PU'_c                     (off the chain)
// MMA_O(c) is issued right after MMA_S(c+1), so it runs in the tensor pipe while the state
// epilogue of chunk c+1 works instead of sitting in front of the next chain MMA; the fp16
// state therefore keeps three buffers.
// Roles: warps 0 .. 4W-1 carry the state (warp w: TMEM lane quarter w % 4, slice w / 4),
// warps 4W .. 4W+3 form the outputs of all W slices in turn (the M = 64 accumulator puts
// row r in lane (r%16) + 32*(r/16)), warp 4W+4 streams the per-chunk blocks with bulk copies
// into two rings ({N, b slices, gC} and {Qe, PU' slices}), and one thread of warp 4W+5
// issues every MMA.  All hand-offs are mbarriers with bounded waits.  (Four output warps
// rather than 4W keep at most four warps on each scheduler, so each thread may keep
// up to 128 registers.  One producer warp per ring, an L2 prefetch of the blocks a few
// chunks ahead, and reading every slice's D_O before freeing it were each measured slower.)
// The chain MMA costs about the same for N = 32 and N = 64 (its latency is the tensor pipe's,
// not the columns'), so W = 2 carries a head's state on half as many SMs.  Its step is slower
// (twice the state warps per scheduler, a shallower ring), so launch_tc takes W = 2 only when
// the W = 1 grid would need more than one wave of SMs.
template <int W>
struct ScanCfg {
    static constexpr int kThreads = 32 * (4 * W + 6);
    static constexpr int kNB = W == 1 ? 3 : 2;             // ring depths (shared memory bound)
    static constexpr int kQP = W == 1 ? 4 : 3;
    static constexpr uint32_t kNBBytes = 32768 + 8192 * W + 512;
    static constexpr uint32_t kNBStride = kNBBytes;        // a 128-byte multiple
    static constexpr uint32_t kSN = 0, kSB = 32768, kSG = 32768 + 8192 * W;   // within an NB stage
    static constexpr uint32_t kQPBytes = 16384 + 4096 * W;
    static constexpr uint32_t kQPStride = kQPBytes;
    static constexpr uint32_t kSQe = 0, kSPU = 16384;                        // within a QP stage
    static constexpr uint32_t kRingNB = 0;
    static constexpr uint32_t kRingQP = kRingNB + kNB * kNBStride;
    static constexpr uint32_t kSopBytes = 8192 * W;        // S fp16 (k = i, n = j) MN-major SBO 2048 LBO 128
    static constexpr uint32_t kSop = kRingQP + kQP * kQPStride;
    static constexpr uint32_t kSBar = kSop + 3 * kSopBytes;
    static constexpr uint32_t kSTmem = kSBar + 256;
    static constexpr uint32_t kSmem = kSTmem + 64;
    static constexpr uint32_t kTmemCols = W == 1 ? 128 : 256;   // D_S (32W) + 2 x D_O (32W)
};
static_assert(ScanCfg<1>::kSmem == 231232 && ScanCfg<2>::kSmem <= 232448 - 1024, "scan shared memory");
static_assert(ScanCfg<1>::kNBBytes % 128 == 0 && ScanCfg<2>::kNBBytes % 128 == 0 &&
              ScanCfg<2>::kSop % 1024 == 0, "stage alignment");
static_assert(2 * ScanCfg<1>::kNB + 2 * ScanCfg<1>::kQP + 6 <= 32 &&
              2 * ScanCfg<2>::kNB + 2 * ScanCfg<2>::kQP + 6 <= 32, "mbarrier area");

// This launch covers chunks cb .. ce-1, starting from S_in (null: zero) and leaving the
// state in S_out (may be null); ring stages and barrier phases count from cb.
template <int W>
__global__ void __launch_bounds__(ScanCfg<W>::kThreads, 1) scan_tc_kernel(Problem p, int cb, int ce,
                                                                         const float* S_in, float* S_out) {
    using Cfg = ScanCfg<W>;
    constexpr int kNB = Cfg::kNB, kQP = Cfg::kQP;
    constexpr int NSW = NS * W;                            // columns of this CTA
    extern __shared__ __align__(1024) uint8_t sm[];
    const int slice0 = blockIdx.x * W;                     // first 32-column slice of this CTA
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (!GDN_IN_BOUNDS(cb >= 0 && ce <= p.NC && bh < p.B * p.H && slice0 + W <= J, p.status)) return;
    uint64_t* fullNB = reinterpret_cast<uint64_t*>(sm + Cfg::kSBar);
    uint64_t* emptyNB = fullNB + kNB;
    uint64_t* fullQP = emptyNB + kNB;
    uint64_t* emptyQP = fullQP + kQP;
    uint64_t* bar_s = emptyQP + kQP;       // MMA_S done
    uint64_t* bar_o = bar_s + 1;           // [2] MMA_O done, per D_O buffer
    uint64_t* s_ready = bar_o + 2;         // S_c written to Sop (4W warp arrivals)
    uint64_t* o_free = s_ready + 1;        // [2] D_O buffer read (4 warp arrivals)
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Cfg::kSTmem);
    const uint8_t* blocks = static_cast<const uint8_t*>(p.inter) + (size_t)bh * p.NC * kBlockBytes;
    const int nloc = ce - cb;              // chunks of this launch; loop indices below are local

    if (warp == 0) {
        tmem_alloc(tslot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < kNB; ++i) { mbar_init(&fullNB[i], 1); mbar_init(&emptyNB[i], 4 * W); }
        for (int i = 0; i < kQP; ++i) { mbar_init(&fullQP[i], 1); mbar_init(&emptyQP[i], 4); }
        mbar_init(bar_s, 1);
        mbar_init(&bar_o[0], 1);
        mbar_init(&bar_o[1], 1);
        mbar_init(s_ready, 4 * W);
        mbar_init(&o_free[0], 4);
        mbar_init(&o_free[1], 4);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = *tslot;
    const uint32_t tS = t0, tO = t0 + NSW;                 // D_S (NSW columns); D_O[0], D_O[1]
    bool ok = true;

    if (warp == 4 * W + 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int ch = 0; ch < nloc && ok; ++ch) {
                const uint8_t* src = blocks + (size_t)(cb + ch) * kBlockBytes;
                const int s3 = ch % kNB, s4 = ch % kQP;
                if (ch >= kNB && !mbar_wait(&emptyNB[s3], ((ch / kNB) - 1) & 1)) { ok = false; break; }
                uint8_t* d3 = sm + Cfg::kRingNB + s3 * Cfg::kNBStride;
                mbar_arrive_expect_tx(&fullNB[s3], Cfg::kNBBytes);
                bulk_g2s(d3 + Cfg::kSN, src + kOffN, 32768, &fullNB[s3]);
                bulk_g2s(d3 + Cfg::kSB, src + kOffB + (size_t)slice0 * D * NS * 2, 8192 * W, &fullNB[s3]);
                bulk_g2s(d3 + Cfg::kSG, src + kOffGC, 512, &fullNB[s3]);
                if (ch >= kQP && !mbar_wait(&emptyQP[s4], ((ch / kQP) - 1) & 1)) { ok = false; break; }
                uint8_t* d4 = sm + Cfg::kRingQP + s4 * Cfg::kQPStride;
                mbar_arrive_expect_tx(&fullQP[s4], Cfg::kQPBytes);
                bulk_g2s(d4 + Cfg::kSQe, src + kOffQe, 16384, &fullQP[s4]);
                bulk_g2s(d4 + Cfg::kSPU, src + kOffPU + (size_t)slice0 * C * NS * 2, 4096 * W, &fullQP[s4]);
            }
            if (!ok) record_timeout(p.status);
        }
    } else if (warp == 4 * W + 5) {
        // ------------------------------------------------------------ MMA issuer (one thread)
        if (lane == 0) {
            const uint32_t idS = idesc_f16(128, NSW, false, true);
            const uint32_t idO = idesc_f16(64, NSW, true, true);
            // MMA_O of chunk cc (reads Sop[cc % 3] and the QP stage of cc)
            auto issue_o = [&](int cc) -> bool {
                const int s4 = cc % kQP;
                if (cc >= 2 && !mbar_wait(&o_free[cc & 1], ((cc >> 1) - 1) & 1)) return false;
                if (!mbar_wait(&fullQP[s4], (cc / kQP) & 1)) return false;
                tc_fence_after();
                const uint64_t a0 = sdesc(smem_u32(sm + Cfg::kRingQP + s4 * Cfg::kQPStride + Cfg::kSQe), 128, 2048);
                const uint64_t b0 = sdesc(smem_u32(sm + Cfg::kSop + (cc % 3) * Cfg::kSopBytes), 128, 2048);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) mma_f16(tO + NSW * (cc & 1), a0 + 16 * kk, b0 + 16 * kk, idO, kk > 0);
                mma_commit(&bar_o[cc & 1]);
                return true;
            };
            for (int ch = 0; ch < nloc && ok; ++ch) {
                const int s3 = ch % kNB;
                if (!mbar_wait(s_ready, ch & 1) || !mbar_wait(&fullNB[s3], (ch / kNB) & 1)) { ok = false; break; }
                tc_fence_after();
                {
                    const uint64_t a0 = sdesc(smem_u32(sm + Cfg::kRingNB + s3 * Cfg::kNBStride + Cfg::kSN), 128, 2048);
                    const uint64_t b0 = sdesc(smem_u32(sm + Cfg::kSop + (ch % 3) * Cfg::kSopBytes), 128, 2048);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) mma_f16(tS, a0 + 16 * kk, b0 + 16 * kk, idS, kk > 0);
                    mma_commit(bar_s);
                }
                if (ch > 0 && !issue_o(ch - 1)) { ok = false; break; }
            }
            if (ok && nloc > 0) ok = issue_o(nloc - 1);
            if (!ok) record_timeout(p.status);
        }
    } else if (warp < 4 * W) {
        // ------------------------------------------------------------ state chain
        const int q = warp & 3, sl = warp >> 2;                // TMEM lane quarter, slice within the CTA
        const int row = 32 * q + lane;                         // d_k row of S (TMEM lane)
        const int j0 = (slice0 + sl) * NS;                     // first state column of this warp
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        float S[NS];
        float smax = 0.f;
#pragma unroll
        for (int j = 0; j < NS; ++j) S[j] = S_in ? S_in[((size_t)bh * D + row) * D + j0 + j] : 0.f;
#pragma unroll
        for (int j = 0; j < NS; ++j) smax = fmax_nan(smax, fabsf(S[j]));
#pragma unroll
        for (int j = 0; j < NS; j += 8) st16(sm + Cfg::kSop, off_mnmajor(NS * sl + j, row, 2048, 128), f_to_h8(S + j));
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_ready);
        for (int ch = 0; ch < nloc && ok; ++ch) {
            const int s3 = ch % kNB;
            const uint8_t* nb = sm + Cfg::kRingNB + s3 * Cfg::kNBStride;
            if (!__all_sync(0xffffffffu, mbar_wait(&fullNB[s3], (ch / kNB) & 1))) { ok = false; break; }
            const __half* bsm = reinterpret_cast<const __half*>(nb + Cfg::kSB) + sl * (D * NS);
            float bv[NS];
#pragma unroll
            for (int g8 = 0; g8 < NS; g8 += 8) {
                const uint4 v = *reinterpret_cast<const uint4*>(bsm + sw_half(row, g8));
                const __half2* hh = reinterpret_cast<const __half2*>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __half22float2(hh[e]);
                    bv[g8 + 2 * e] = f.x;
                    bv[g8 + 2 * e + 1] = f.y;
                }
            }
            const float gc = reinterpret_cast<const float*>(nb + Cfg::kSG)[row];
            if (!__all_sync(0xffffffffu, mbar_wait(bar_s, ch & 1))) { ok = false; break; }
            tc_fence_after();
            float d[NS];
            tmem_ld32(tS + lanebase + NS * sl, d);
#pragma unroll
            for (int j = 0; j < NS; ++j) S[j] = fmaf(gc, S[j], d[j] + bv[j]);
            uint8_t* snext = sm + Cfg::kSop + ((ch + 1) % 3) * Cfg::kSopBytes;
#pragma unroll
            for (int j = 0; j < NS; j += 8) st16(snext, off_mnmajor(NS * sl + j, row, 2048, 128), f_to_h8(S + j));
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(s_ready);                          // this warp's part of S_{ch+1} is in Sop
                mbar_arrive(&emptyNB[s3]);
            }
            // largest |S| entry so far (off the chain: nothing waits for it); above the fp16
            // range the fp16 copy, and so the result, is not valid
#pragma unroll
            for (int j = 0; j < NS; ++j) smax = fmax_nan(smax, fabsf(S[j]));
        }
        // NaN compares false: a NaN state is reported too
        if (ok && __any_sync(0xffffffffu, !(smax <= 65504.f)) && lane == 0)
            atomicCAS(p.status, kDevOk, kDevRange);
        if (!ok) {
            if (lane == 0) record_timeout(p.status);
        } else if (S_out) {
            float4* dst = reinterpret_cast<float4*>(S_out + ((size_t)bh * D + row) * D + j0);
#pragma unroll
            for (int j = 0; j < NS; j += 4) dst[j / 4] = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    } else {
        // ------------------------------------------------------------ outputs (warps 4W .. 4W+3)
        const int q = warp - 4 * W;                            // TMEM lane quarter
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        const int rw = 16 * q + lane;                          // output row (valid for lane < 16)
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
        for (int ch = 0; ch < nloc && ok; ++ch) {
            const int s4 = ch % kQP;
            const bool got = mbar_wait(&fullQP[s4], (ch / kQP) & 1) && mbar_wait(&bar_o[ch & 1], (ch >> 1) & 1);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int s = (cb + ch) * C + rw;
            RowRef ro{};
            const bool write = lane < 16 && s < p.L && (ro = row_ref(p, b, h, s)).has_q;
#pragma unroll 1
            for (int sl = 0; sl < W; ++sl) {
                float d[NS];
                tmem_ld32(tO + lanebase + NSW * (ch & 1) + NS * sl, d);
                if (sl == W - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&o_free[ch & 1]);
                }
                if (write) {
                    const __half* pu = reinterpret_cast<const __half*>(sm + Cfg::kRingQP + s4 * Cfg::kQPStride + Cfg::kSPU) +
                                       sl * (C * NS);
                    uint4* dst = reinterpret_cast<uint4*>(out + ro.tok * D + (slice0 + sl) * NS);
#pragma unroll
                    for (int g8 = 0; g8 < NS; g8 += 8) {
                        const uint4 pv = *reinterpret_cast<const uint4*>(pu + sw_half(rw, g8));
                        const __half2* ph = reinterpret_cast<const __half2*>(&pv);
                        __nv_bfloat162 o2[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 pf = __half22float2(ph[e]);
                            o2[e] = __floats2bfloat162_rn(pf.x + d[g8 + 2 * e], pf.y + d[g8 + 2 * e + 1]);
                        }
                        dst[g8 / 8] = *reinterpret_cast<uint4*>(o2);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&emptyQP[s4]);
        }
        if (!ok && lane == 0) record_timeout(p.status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t0, Cfg::kTmemCols);
}

}  // namespace tc

bool tc_supported(const Problem& p, bool bf16) {
    return bf16 && p.C == tc::C && p.dk == tc::D && p.dv == tc::D && p.T > 0;
}

// Segments of one call: the sequence's chunks are cut into P consecutive ranges.  Intra of
// range s+1 runs on the caller's stream while the scan of range s runs on a high-priority
// side stream, so the scan's chain no longer waits for the whole intra role and the SMs
// the scan leaves idle keep working.  Each range keeps at least kMinSegChunks chunks.
constexpr int kMaxSegments = 4;
static_assert(kMaxSegments <= kSideEvents, "one ready event per range");
constexpr int kMinSegChunks = 32;

int tc_segments(const Problem& p) {
    const int s = p.NC / kMinSegChunks;
    return s < 1 ? 1 : (s > kMaxSegments ? kMaxSegments : s);
}

// Chunk range [cb, ce) of segment sg of P.  Only the last range's scan runs with no intra
// work beside it, and a chunk's intra role costs several times its scan step, so the last
// range is short (NC/8, at least kMinSegChunks) and the others share the rest evenly.
void seg_range(int NC, int P, int sg, int& cb, int& ce) {
    int last = NC / 8 > kMinSegChunks ? NC / 8 : kMinSegChunks;
    if (last > NC / P) last = NC / P;
    const int head = NC - last;
    if (sg == P - 1) {
        cb = head;
        ce = NC;
    } else {
        cb = (int)((long)head * sg / (P - 1));
        ce = (int)((long)head * (sg + 1) / (P - 1));
    }
}

size_t tc_inter_bytes(const Problem& p) {
    const size_t blocks = (size_t)p.B * p.H * p.NC * tc::kBlockBytes;   // 256-byte multiple
    const size_t handoff = tc_segments(p) > 1 ? (size_t)p.B * p.H * tc::D * tc::D * sizeof(float) : 0;
    return blocks + handoff;
}

int tc_launches(const Problem& p) { return p.NC > 0 ? 2 * tc_segments(p) : 1; }


// gdn_tc2.cu: the TMA-fed intra role, for the problems it covers; gdn_scan2.cu: the scan role
// for its blocks
bool tc2_usable(const Problem& p);
cudaError_t launch_intra_tma(const Problem& p, int cb, int n, cudaStream_t stream);
cudaError_t launch_scan2(const Problem& p, int cb, int ce, const float* S_in, float* S_out, cudaStream_t stream);

cudaError_t launch_tc(const Problem& p, cudaStream_t stream) {
#ifdef GDN_DEBUG_BOUNDS
    // Test knob of the bounds-checking build only (environment GDN_TEST_BOUNDS_NC_OFF=1): the
    // kernels are told one chunk fewer than their grids cover, so the checks on the last chunk's
    // CTAs fire (and skip their accesses); the block stride shrinks with it, so every address
    // formed stays inside the workspace.
    Problem pk_ = p;
    if (const char* e = std::getenv("GDN_TEST_BOUNDS_NC_OFF"))
        if (e[0] == '1' && pk_.NC > 1) pk_.NC -= 1;
    const Problem& pk = pk_;
#else
    const Problem& pk = p;
#endif
    auto intra = p.gdn2_eta ? tc::intra_tc_kernel<false, true>
               : (p.beta_v ? tc::intra_tc_kernel<true> : tc::intra_tc_kernel<false>);
    const bool tma = tc2_usable(p);
    cudaError_t ae = cudaSuccess;
    if (!tma) {
        ae = cudaFuncSetAttribute(intra, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kIntraSmem);
        if (ae != cudaSuccess) return ae;
    }
    // intra role over chunks [cb, cb + n) of every head
    auto launch_intra = [&](int cb, int n, cudaStream_t st) -> cudaError_t {
        if (tma) return launch_intra_tma(pk, cb, n, st);
        intra<<<dim3(n, p.B * p.H), tc::NT, tc::kIntraSmem, st>>>(pk, cb);
        return cudaGetLastError();
    };
    // scan width: two slices per CTA when one slice per CTA would take more than one wave
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 0;
    const bool w2 = (long)p.B * p.H * tc::J > (long)sms;
    auto scan = w2 ? tc::scan_tc_kernel<2> : tc::scan_tc_kernel<1>;
    const uint32_t scan_smem = w2 ? tc::ScanCfg<2>::kSmem : tc::ScanCfg<1>::kSmem;
    const int scan_threads = w2 ? tc::ScanCfg<2>::kThreads : tc::ScanCfg<1>::kThreads;
    if (!tma) {
        ae = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan_smem);
        if (ae != cudaSuccess) return ae;
    }
    const dim3 g2(tc::J / (w2 ? 2 : 1), p.B * p.H);
    const int P = tc_segments(p);
    // scan role over chunks [cb, ce)
    auto launch_scan = [&](int cb, int ce, const float* S_in, float* S_out, cudaStream_t st) -> cudaError_t {
        if (tma) return launch_scan2(pk, cb, ce, S_in, S_out, st);
        scan<<<g2, scan_threads, scan_smem, st>>>(pk, cb, ce, S_in, S_out);
        return cudaGetLastError();
    };
    auto one_stream = [&]() {               // both roles over all chunks, on the caller's stream
        cudaError_t e = launch_intra(0, p.NC, stream);
        if (e != cudaSuccess) return e;
        return launch_scan(0, p.NC, p.S0, p.S_final, stream);
    };
    if (P == 1 || p.single_stream) return one_stream();
    std::unique_lock<std::mutex> lock;
    SideStream* side = side_stream_lock(lock);
    if (!side) return one_stream();
    SideStream& ss = *side;
    float* handoff = reinterpret_cast<float*>(static_cast<char*>(p.inter) +
                                              (size_t)p.B * p.H * p.NC * tc::kBlockBytes);
    cudaError_t e = cudaEventRecord(ss.fork, stream);             // the side stream starts after
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.stream, ss.fork, 0);   // the caller's prior work
    for (int sg = 0; sg < P && e == cudaSuccess; ++sg) {
        int cb, ce;
        seg_range(p.NC, P, sg, cb, ce);
        e = launch_intra(cb, ce - cb, stream);
        if (e == cudaSuccess) e = cudaEventRecord(ss.ready[sg], stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.stream, ss.ready[sg], 0);
        if (e != cudaSuccess) break;
        e = launch_scan(cb, ce, sg == 0 ? p.S0 : handoff, sg == P - 1 ? p.S_final : handoff, ss.stream);
    }
    // join: whatever happened above, the caller's stream waits for the side stream's work
    cudaError_t j = cudaEventRecord(ss.join, ss.stream);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(stream, ss.join, 0);
    return e != cudaSuccess ? e : j;
}

}  // namespace gdn
