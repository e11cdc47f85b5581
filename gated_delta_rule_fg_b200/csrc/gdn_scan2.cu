// gdn_scan2.cu -- the scan role of the tensor-core path for the blocks of the TMA-fed intra
// kernel (gdn_tc2.cu): one CTA per (head, W consecutive 32-column slices of d_v), serial over
// the chunks of its range, one CTA per SM.  W = 2 carries a head on two SMs: the chain product
// costs about the same for 64 columns as for 32, and the SMs it does not hold run intra CTAs.
//
// Per chunk c, with S_c in fp32 registers (row i per thread) and its fp16 copy in Sop[c % kSl]:
//   MMA_S: D_S = N_c S_c            -> S_{c+1} = Diag(gC) S_c + D_S + b_c   (the serial chain)
//   MMA_O: D_O = [Qe_c; *] S_c      -> O_c = D_O + PU'_c                      (off the chain)
// Both products take their A operand from tensor memory: four feeder warps copy N_c (128 rows)
// out of the shared-memory ring into tensor-memory buffers (row m in lane m, two fp16 per
// column), and two more warps copy Qe_c (64 rows) into lanes 64 .. 127 of another buffer.  The
// tensor pipe then reads only the fp16 state from shared memory per instruction, so the chain
// product is short and the output product (an M = 128 product whose rows 0 .. 63 are not used)
// costs little beside it.  N feeding waits only for the chain, never for the outputs.
//
// Warps: 0 .. 4W-1 state (lane quarter w % 4, slice w / 4), 4W .. 4W+3 N feeders (lane quarter
// w - 4W), 4W+4 producer (bulk copies into three rings: {N, Qe}, {b slices, gC}, {PU' slices}),
// 4W+5 chain MMA issuer, 4W+6 and 4W+7 Qe feeders (lane quarters 2 and 3: Qe
// rows 0 .. 63 into lanes 64 .. 127), 4W+8 output MMA issuer, 4W+10 and 4W+11 output writers
// (D_O lanes 64 .. 127; warp 4W+9 only fills the lane-quarter pattern).  Every hand-off is an
// mbarrier with a bounded wait; a wait that runs out records GDN_ERR_TIMEOUT and the role unwinds.
#include "gdn_tc_common.cuh"

namespace gdn {
namespace sc2 {
using namespace sm100;
using tc::C;
using tc::D;
using tc::NS;

template <int W>
struct Cfg {
    static constexpr int NSW = NS * W;                       // columns of this CTA
    // Warp roles.  A warp reads and writes the tensor-memory lanes of quarter warp % 4, which
    // fixes where the Qe feeders and output writers sit.  One slice: Qe rows 0 .. 63 go to lanes
    // 64 .. 127 only (quarters 2, 3); two slices: to both lane halves (quarters 0 .. 3), and the
    // outputs of slice 0 are read from lanes 64 .. 127, those of slice 1 from lanes 0 .. 63.
    static constexpr int kNFeed0 = 4 * W;                    // 4 N feeders
    static constexpr int kQe0 = W == 1 ? 10 : 12, kNQe = W == 1 ? 2 : 4;
    static constexpr int kOut0 = W == 1 ? 14 : 16, kNOut = W == 1 ? 2 : 4;
    static constexpr int kProducer = W == 1 ? 8 : 20, kMmaS = W == 1 ? 9 : 21, kMmaO = W == 1 ? 12 : 22;
    static constexpr int kWarps = W == 1 ? 16 : 23;
    static constexpr int kThreads = 32 * kWarps;
    // Three rings, each released by the role that reads it last: {N, Qe} by the feeders once
    // copied into tensor memory, {b slices, gC} by the state warps, {PU' slices} by the output
    // warps (which run two chunks behind the chain, so their data must not hold back the state
    // warps' ring).
    static constexpr int kNQ = 2;                            // {N, Qe} ring depth
    static constexpr int kBG = W == 1 ? 4 : 3;               // {b, gC} ring depth
    static constexpr int kPU = W == 1 ? 4 : 3;               // {PU'} ring depth
    static constexpr uint32_t kNQBytes = 32768 + 16384;      // N, then Qe (K-major, SBO 2048, LBO 128)
    static constexpr uint32_t kBGBytes = 8192 * W + 512;     // b slices (fp16 group-major), gC
    static constexpr uint32_t kPUBytes = 4096 * W;           // PU' slices (fp16 group-major)
    static constexpr uint32_t kSopBytes = 8192 * W;          // S fp16 (k = i, n = j) MN-major SBO 2048 LBO 128
    // Sop slots: S_c lives in slot c % kSl until MMA_S(c) and MMA_O(c) have read it; the output
    // product may lag the chain by kSl - 2 chunks before the state warps wait for it
    static constexpr int kSl = W == 1 ? 4 : 3;
    static constexpr uint32_t kRingNQ = 0;
    static constexpr uint32_t kRingBG = kRingNQ + kNQ * kNQBytes;
    static constexpr uint32_t kRingPU = kRingBG + kBG * kBGBytes;
    static constexpr uint32_t kSop = kRingPU + kPU * kPUBytes;
    static constexpr uint32_t kBar = kSop + kSl * kSopBytes;
    static constexpr uint32_t kTslot = kBar + 512;
    static constexpr uint32_t kSmem = kTslot + 64;
    // tensor memory columns (512 allocated): D_S, D_O[2], Qe[2] (64 each), N[2] (64 each)
    // Qe and D_O buffers: three with one slice, so that the output product of a chunk is never
    // held back by the outputs of the chunk before (it then runs beside the state epilogue
    // instead of in front of the next chain product)
    static constexpr int kNO = W == 1 ? 3 : 2;
    static constexpr uint32_t kTS = 0, kTO = NSW, kTQ = kTO + kNO * NSW, kTN = kTQ + kNO * 64;
};
static_assert(Cfg<1>::kRingBG % 128 == 0 && Cfg<1>::kRingPU % 128 == 0 && Cfg<1>::kSop % 128 == 0, "alignment");
static_assert(Cfg<2>::kRingBG % 128 == 0 && Cfg<2>::kRingPU % 128 == 0 && Cfg<2>::kSop % 128 == 0, "alignment");
static_assert(Cfg<1>::kSmem <= 227 * 1024 && Cfg<2>::kSmem <= 227 * 1024, "shared memory");
static_assert(Cfg<1>::kTN + 128 <= 512 && Cfg<2>::kTN + 128 <= 512, "tensor memory");
static_assert(Cfg<1>::kQe0 % 4 == 2 && Cfg<1>::kOut0 % 4 == 2 && Cfg<2>::kQe0 % 4 == 0 && Cfg<2>::kOut0 % 4 == 0,
              "Qe feeders and output writers on the lane quarters they use");

// Copies rows of a K-major (SBO 2048, LBO 128) fp16 tile from shared memory into tensor memory
// as an A operand: this thread's row `row`, 128 fp16 = 64 columns, lane = row.
__device__ __forceinline__ void rows_to_tmem(const uint8_t* tile, int row, uint32_t taddr_lane) {
    float v[32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            const uint4 u = *reinterpret_cast<const uint4*>(tile + off_kmajor(row, 64 * half + 8 * g, 2048, 128));
            v[4 * g + 0] = __uint_as_float(u.x);
            v[4 * g + 1] = __uint_as_float(u.y);
            v[4 * g + 2] = __uint_as_float(u.z);
            v[4 * g + 3] = __uint_as_float(u.w);
        }
        tmem_st32(taddr_lane + 32 * half, v);
    }
}

__device__ __forceinline__ void mma_ta(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(bdesc), "r"((uint32_t)acc), "r"(idesc)
        : "memory");
}

// This launch covers chunks cb .. ce-1, starting from S_in (null: zero) and leaving the state in
// S_out (may be null); ring stages and barrier phases count from cb.
template <int W>
__global__ void __launch_bounds__(Cfg<W>::kThreads, 1) scan2_kernel(Problem p, int cb, int ce, const float* S_in,
                                                                   float* S_out) {
    using K = Cfg<W>;
    constexpr int NSW = K::NSW, kNQ = K::kNQ, kBG = K::kBG, kPU = K::kPU;
    constexpr uint32_t kNQBytes = K::kNQBytes, kBGBytes = K::kBGBytes, kPUBytes = K::kPUBytes;
    constexpr uint32_t kRingNQ = K::kRingNQ, kRingBG = K::kRingBG, kRingPU = K::kRingPU, kSop = K::kSop;
    constexpr uint32_t kSopBytes = K::kSopBytes, kBar = K::kBar, kTslot = K::kTslot;
    constexpr uint32_t kTS = K::kTS, kTO = K::kTO, kTQ = K::kTQ, kTN = K::kTN;
    constexpr int kNO = K::kNO, kSl = K::kSl;
    extern __shared__ __align__(1024) uint8_t sm[];
    const int slice0 = blockIdx.x * W;                     // first 32-column slice of this CTA
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (!GDN_IN_BOUNDS(cb >= 0 && ce <= p.NC && bh < p.B * p.H && slice0 + W <= tc::J, p.status)) return;
    uint64_t* fullNQ = reinterpret_cast<uint64_t*>(sm + kBar);
    uint64_t* emptyNQ = fullNQ + kNQ;
    uint64_t* fullBG = emptyNQ + kNQ;
    uint64_t* emptyBG = fullBG + kBG;
    uint64_t* fullPU = emptyBG + kBG;
    uint64_t* emptyPU = fullPU + kPU;
    uint64_t* bar_s = emptyPU + kPU;       // MMA_S done
    uint64_t* s_ready = bar_s + 1;         // S_c in Sop (4 state warps)
    uint64_t* n_ready = s_ready + 1;       // [2] N_c in tensor memory (4 feeders)
    uint64_t* n_free = n_ready + 2;        // [2] MMA_S that read N buffer done
    uint64_t* q_ready = n_free + 2;        // [kNO] Qe_c in tensor memory (2 Qe feeders)
    uint64_t* q_free = q_ready + kNO;      // [kNO] MMA_O that read Qe buffer done
    uint64_t* bar_o = q_free + kNO;        // [kNO] MMA_O done, per D_O buffer
    uint64_t* o_free = bar_o + kNO;        // [kNO] D_O buffer read (the 2 output warps)
    uint64_t* s_slot = o_free + kNO;       // [kSl] S_c written into Sop slot c % kSl (4W state warps)
    uint64_t* o_done = s_slot + kSl;       // [kSl] MMA_O that read Sop slot c % kSl done
    uint64_t* bar_d = o_done + kSl;        // drain: both MMA threads' last products done
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kTslot);
    const uint8_t* blocks = static_cast<const uint8_t*>(p.inter) + (size_t)bh * p.NC * tc::kBlockBytes;
    const int nloc = ce - cb;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < kNQ; ++i) { mbar_init(&fullNQ[i], 1); mbar_init(&emptyNQ[i], 4 + K::kNQe); }
        for (int i = 0; i < kBG; ++i) { mbar_init(&fullBG[i], 1); mbar_init(&emptyBG[i], 4 * W); }
        for (int i = 0; i < kPU; ++i) { mbar_init(&fullPU[i], 1); mbar_init(&emptyPU[i], K::kNOut); }
        mbar_init(bar_s, 1);
        mbar_init(s_ready, 4 * W);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&n_ready[i], 4);
            mbar_init(&n_free[i], 1);
        }
        for (int i = 0; i < kNO; ++i) {
            mbar_init(&q_ready[i], K::kNQe);
            mbar_init(&q_free[i], 1);
            mbar_init(&bar_o[i], 1);
            mbar_init(&o_free[i], K::kNOut);
        }
        for (int i = 0; i < kSl; ++i) {
            mbar_init(&s_slot[i], 4 * W);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(bar_d, 2);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t0 = *tslot;
    const uint64_t lim = p.test_wait_ns ? p.test_wait_ns : kWaitLimitNs;
    bool ok = true;

    if (warp == K::kProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // The rings are only a few chunks deep, less than a DRAM round trip at the chain's
            // pace, so the blocks kPrefetch chunks ahead are first pulled into L2.
            constexpr int kPrefetch = 4;
            auto prefetch = [&](int ch) {
                const uint8_t* src = blocks + (size_t)(cb + ch) * tc::kBlockBytes;
                bulk_prefetch_l2(src + tc::kOffN, 32768 + 16384);                       // N, Qe
                bulk_prefetch_l2(src + tc::kOffB + (size_t)slice0 * D * NS * 2, 8192 * W);
                bulk_prefetch_l2(src + tc::kOffPU + (size_t)slice0 * C * NS * 2, 4096 * W);
                bulk_prefetch_l2(src + tc::kOffGC, 512);
            };
            for (int ch = 0; ch < kPrefetch && ch < nloc; ++ch) prefetch(ch);
            int ld_bg[kBG], ld_nq[kNQ], ld_pu[kPU];           // last chunk loaded into each stage
            for (int i = 0; i < kBG; ++i) ld_bg[i] = -1;
            for (int i = 0; i < kNQ; ++i) ld_nq[i] = -1;
            for (int i = 0; i < kPU; ++i) ld_pu[i] = -1;
            for (int ch = 0; ch < nloc && ok; ++ch) {
                if (ch + kPrefetch < nloc) prefetch(ch + kPrefetch);
                const uint8_t* src = blocks + (size_t)(cb + ch) * tc::kBlockBytes;
                const int s2 = ch % kNQ, sb = ch % kBG, sp = ch % kPU;
                if (ch >= kBG && !mbar_wait(&emptyBG[sb], ((ch / kBG) - 1) & 1, lim)) { ok = false; break; }
                uint8_t* db = sm + kRingBG + sb * kBGBytes;
                mbar_arrive_expect_tx(&fullBG[sb], kBGBytes);
                bulk_g2s(db, src + tc::kOffB + (size_t)slice0 * D * NS * 2, 8192 * W, &fullBG[sb]);
                bulk_g2s(db + 8192 * W, src + tc::kOffGC, 512, &fullBG[sb]);
                ld_bg[sb] = ch;
                if (ch >= kNQ && !mbar_wait(&emptyNQ[s2], ((ch / kNQ) - 1) & 1, lim)) { ok = false; break; }
                if (cb + ch != p.test_skip_chunk) {            // (failure-detection test knob)
                    uint8_t* d2 = sm + kRingNQ + s2 * kNQBytes;
                    mbar_arrive_expect_tx(&fullNQ[s2], kNQBytes);
                    bulk_g2s(d2, src + tc::kOffN, 32768, &fullNQ[s2]);
                    bulk_g2s(d2 + 32768, src + tc::kOffQe, 16384, &fullNQ[s2]);
                    ld_nq[s2] = ch;
                }
                if (ch >= kPU && !mbar_wait(&emptyPU[sp], ((ch / kPU) - 1) & 1, lim)) { ok = false; break; }
                uint8_t* dp = sm + kRingPU + sp * kPUBytes;
                mbar_arrive_expect_tx(&fullPU[sp], kPUBytes);
                bulk_g2s(dp, src + tc::kOffPU + (size_t)slice0 * C * NS * 2, 4096 * W, &fullPU[sp]);
                ld_pu[sp] = ch;
            }
            if (!ok) tc::record_timeout(p.status);
            // Every copy issued lands before the CTA leaves, also when a role unwound early: the
            // last load into each stage of each ring (an earlier load into a stage completed
            // before its consumers released the stage for this one).  Already complete on the
            // normal path.
            for (int i = 0; i < kBG; ++i)
                if (ld_bg[i] >= 0) mbar_wait(&fullBG[i], (ld_bg[i] / kBG) & 1, lim);
            for (int i = 0; i < kNQ; ++i)
                if (ld_nq[i] >= 0) mbar_wait(&fullNQ[i], (ld_nq[i] / kNQ) & 1, lim);
            for (int i = 0; i < kPU; ++i)
                if (ld_pu[i] >= 0) mbar_wait(&fullPU[i], (ld_pu[i] / kPU) & 1, lim);
        }
    } else if (warp == K::kMmaS) {
        // ------------------------------------------------------------ chain MMA issuer (one thread)
        // A thread that issues tcgen05.mma is held for about the time the tensor pipe takes to
        // accept each instruction, while two issuing threads proceed side by side; so the chain
        // product has a thread of its own, and the output products another (warp 4W+8).
        if (lane == 0) {
            const uint32_t idS = idesc_f16(128, NSW, false, true);
            for (int ch = 0; ch < nloc && ok; ++ch) {
                if (!mbar_wait(s_ready, ch & 1, lim) || !mbar_wait(&n_ready[ch & 1], (ch >> 1) & 1, lim)) { ok = false; break; }
                tc_fence_after();
                const uint64_t b0 = sdesc(smem_u32(sm + kSop + (ch % kSl) * kSopBytes), 128, 2048);
                const uint32_t an = t0 + kTN + 64u * (ch & 1);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) mma_ta(t0 + kTS, an + 8u * kk, b0 + 16 * kk, idS, kk > 0);
                mma_commit(bar_s);
                mma_commit(&n_free[ch & 1]);
            }
            if (!ok) tc::record_timeout(p.status);
            // drain: every product this thread issued has completed before the tensor memory goes
            mma_commit(bar_d);
            if (!mbar_wait(bar_d, 0, lim)) tc::record_timeout(p.status);
        }
    } else if (warp == K::kMmaO) {
        // ------------------------------------------------------------ output MMA issuer (one thread)
        // MMA_O(c) reads S_c from Sop slot c % kSl once the state warps have written it; its
        // completion (o_done) lets them write S_{c+kSl} there.
        if (lane == 0) {
            const uint32_t idO = idesc_f16(128, NSW, false, true);
            for (int cc = 0; cc < nloc && ok; ++cc) {
                const int bo = cc % kNO, uo = cc / kNO;        // buffer, and its use count
                if (!mbar_wait(&s_slot[cc % kSl], (cc / kSl) & 1, lim) || !mbar_wait(&q_ready[bo], uo & 1, lim) ||
                    (uo >= 1 && !mbar_wait(&o_free[bo], (uo - 1) & 1, lim))) { ok = false; break; }
                tc_fence_after();
                const uint64_t b0 = sdesc(smem_u32(sm + kSop + (cc % kSl) * kSopBytes), 128, 2048);
                const uint32_t aq = t0 + kTQ + 64u * bo;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) mma_ta(t0 + kTO + NSW * bo, aq + 8u * kk, b0 + 16 * kk, idO, kk > 0);
                mma_commit(&bar_o[bo]);
                mma_commit(&q_free[bo]);
                mma_commit(&o_done[cc % kSl]);
            }
            if (!ok) tc::record_timeout(p.status);
            mma_commit(bar_d);
            if (!mbar_wait(bar_d, 0, lim)) tc::record_timeout(p.status);
        }
    } else if (warp < 4 * W) {
        // ------------------------------------------------------------ state chain
        const int q = warp & 3, sl = warp >> 2;                // TMEM lane quarter, slice within the CTA
        const int row = 32 * q + lane;                         // d_k row of S (TMEM lane)
        const int j0 = (slice0 + sl) * NS;
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        float S[NS];
        float smax = 0.f;
#pragma unroll
        for (int j = 0; j < NS; ++j) S[j] = S_in ? S_in[((size_t)bh * D + row) * D + j0 + j] : 0.f;
#pragma unroll
        for (int j = 0; j < NS; ++j) smax = fmax_nan(smax, fabsf(S[j]));
#pragma unroll
        for (int j = 0; j < NS; j += 8) tc::st16(sm + kSop, off_mnmajor(NS * sl + j, row, 2048, 128), tc::f_to_h8(S + j));
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(s_ready);
            mbar_arrive(&s_slot[0]);
        }
        for (int ch = 0; ch < nloc && ok; ++ch) {
            const int sb = ch % kBG;
            const uint8_t* bp = sm + kRingBG + sb * kBGBytes;
            if (!__all_sync(0xffffffffu, mbar_wait(&fullBG[sb], (ch / kBG) & 1, lim))) { ok = false; break; }
            const __half* bsm = reinterpret_cast<const __half*>(bp) + sl * (D * NS);
            uint4 bq[NS / 8];                                  // b, kept as fp16 pairs until used
#pragma unroll
            for (int g8 = 0; g8 < NS; g8 += 8) bq[g8 / 8] = *reinterpret_cast<const uint4*>(bsm + tc::grp_half(row, g8, D));
            const float gc = reinterpret_cast<const float*>(bp + 8192 * W)[row];
            // Sop slot (ch + 1) % kSl last held S_{ch+1-kSl}: its output product must be done before
            // S_{ch+1} goes there (its chain product is: MMA_S(ch) completes after it).  Checked
            // before the chain product's wait, off the chain's path.
            if (ch + 1 >= kSl &&
                !__all_sync(0xffffffffu, mbar_wait(&o_done[(ch + 1) % kSl], ((ch + 1 - kSl) / kSl) & 1, lim))) {
                ok = false;
                break;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(bar_s, ch & 1, lim))) { ok = false; break; }
            tc_fence_after();
            float d[NS];
            tmem_ld32(t0 + kTS + lanebase + NS * sl, d);
#pragma unroll
            for (int g8 = 0; g8 < NS; g8 += 8) {
                const __half2* hh = reinterpret_cast<const __half2*>(&bq[g8 / 8]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __half22float2(hh[e]);
                    S[g8 + 2 * e] = fmaf(gc, S[g8 + 2 * e], d[g8 + 2 * e] + f.x);
                    S[g8 + 2 * e + 1] = fmaf(gc, S[g8 + 2 * e + 1], d[g8 + 2 * e + 1] + f.y);
                }
            }
            uint8_t* snext = sm + kSop + ((ch + 1) % kSl) * kSopBytes;
#pragma unroll
            for (int j = 0; j < NS; j += 8) tc::st16(snext, off_mnmajor(NS * sl + j, row, 2048, 128), tc::f_to_h8(S + j));
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(s_ready);                          // this warp's part of S_{ch+1} is in Sop
                mbar_arrive(&s_slot[(ch + 1) % kSl]);
                mbar_arrive(&emptyBG[sb]);
            }
#pragma unroll
            for (int j = 0; j < NS; ++j) smax = fmax_nan(smax, fabsf(S[j]));
        }
        if (ok && __any_sync(0xffffffffu, !(smax <= 65504.f)) && lane == 0) atomicCAS(p.status, kDevOk, kDevRange);
        if (!ok) {
            if (lane == 0) tc::record_timeout(p.status);
        } else if (S_out) {
            float4* dst = reinterpret_cast<float4*>(S_out + ((size_t)bh * D + row) * D + j0);
#pragma unroll
            for (int j = 0; j < NS; j += 4) dst[j / 4] = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    } else if (warp >= K::kNFeed0 && warp < K::kNFeed0 + 4) {
        // ------------------------------------------------------------ N feeders
        const int q = warp - K::kNFeed0;                       // TMEM lane quarter
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        const int row = 32 * q + lane;
        // N_c into buffer c & 1 once MMA_S(c - 2) has read it
        for (int it = 0; it < nloc && ok; ++it) {
            const int s2 = it % kNQ;
            bool got = mbar_wait(&fullNQ[s2], (it / kNQ) & 1, lim);
            if (it >= 2) got = got && mbar_wait(&n_free[it & 1], ((it >> 1) - 1) & 1, lim);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            rows_to_tmem(sm + kRingNQ + s2 * kNQBytes, row, t0 + kTN + 64u * (it & 1) + lanebase);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&n_ready[it & 1]);
                mbar_arrive(&emptyNQ[s2]);
            }
        }
        if (!ok && lane == 0) tc::record_timeout(p.status);
    } else if (warp >= K::kQe0 && warp < K::kQe0 + K::kNQe) {
        // ------------------------------------------------------------ Qe feeders
        const int q = warp & 3;                                // TMEM lane quarter
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        const int row = 32 * (q & 1) + lane;                   // Qe row of the chunk
        // Qe_it into buffer it % kNO (lanes 64 .. 127) once MMA_O(it - kNO) has read it
        for (int it = 0; it < nloc && ok; ++it) {
            const int s2 = it % kNQ;
            bool got = mbar_wait(&fullNQ[s2], (it / kNQ) & 1, lim);
            const int bq = it % kNO, uq = it / kNO;
            if (uq >= 1) got = got && mbar_wait(&q_free[bq], (uq - 1) & 1, lim);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            rows_to_tmem(sm + kRingNQ + s2 * kNQBytes + 32768, row, t0 + kTQ + 64u * bq + lanebase);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&q_ready[bq]);
                mbar_arrive(&emptyNQ[s2]);
            }
        }
        if (!ok && lane == 0) tc::record_timeout(p.status);
    } else if (warp >= K::kOut0 && warp < K::kOut0 + K::kNOut) {
        // ------------------------------------------------------------ output writers
        const int q = warp & 3;                                // TMEM lane quarter
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        const int row = 32 * (q & 1) + lane;                   // output row of the chunk
        const int sl = W == 1 ? 0 : 1 - (q >> 1);              // slice: lanes 64-127 slice 0, 0-63 slice 1
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
        for (int oc = 0; oc < nloc && ok; ++oc) {
            const int sp = oc % kPU;
            const int bo = oc % kNO;
            const bool got = mbar_wait(&fullPU[sp], (oc / kPU) & 1, lim) && mbar_wait(&bar_o[bo], (oc / kNO) & 1, lim);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            const int s = (cb + oc) * C + row;
            RowRef ro{};
            const bool write = s < p.L && (ro = row_ref(p, b, h, s)).has_q &&
                               GDN_IN_BOUNDS(ro.tok < (size_t)p.B * p.T * p.H, p.status);
            {
                float d[NS];
                tmem_ld32(t0 + kTO + NSW * bo + NS * sl + lanebase, d);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_free[bo]);
                if (write) {
                    const __half* pu = reinterpret_cast<const __half*>(sm + kRingPU + sp * kPUBytes) + sl * (C * NS);
                    uint4* dst = reinterpret_cast<uint4*>(out + ro.tok * D + (slice0 + sl) * NS);
#pragma unroll
                    for (int g8 = 0; g8 < NS; g8 += 8) {
                        const uint4 pv = *reinterpret_cast<const uint4*>(pu + tc::grp_half(row, g8, C));
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
            if (lane == 0) mbar_arrive(&emptyPU[sp]);
        }
        if (!ok && lane == 0) tc::record_timeout(p.status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t0, 512);
}

}  // namespace sc2

// Scan role over chunks [cb, ce): one slice per CTA.
cudaError_t launch_scan2(const Problem& p, int cb, int ce, const float* S_in, float* S_out, cudaStream_t stream) {
    constexpr int W = 1;
    const cudaError_t e = cudaFuncSetAttribute(sc2::scan2_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)sc2::Cfg<W>::kSmem);
    if (e != cudaSuccess) return e;
    sc2::scan2_kernel<W><<<dim3(tc::J / W, p.B * p.H), sc2::Cfg<W>::kThreads, sc2::Cfg<W>::kSmem, stream>>>(
        p, cb, ce, S_in, S_out);
    return cudaGetLastError();
}

}  // namespace gdn
