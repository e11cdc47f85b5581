// gdn_bwd.cu -- chunkwise backward of the FG^2-GDN forward (float32, CUDA cores).
//
// Gradients of a loss L(o, S_final) given dO = dL/do and dS_final = dL/dS_final,
// for the recurrence of eq. (11) of the FG^2-GDN reading notes (sec. 2.2; the
// split rates of eq. (13), sec. 2.3, when beta_v is given), computed chunkwise as
// the training half of the chunkwise algorithm (sec. 2.4).
//
// Per chunk, with S the state at the chunk start, S' the state at its end and
// (forward, see gdn_common.cuh)
//     R = V~ - K_G S,  U = (I + A)^{-1} R,  O = Q_G S + P U,  S' = Diag(e^{g_C}) S + K_E^T U
// where K_G = K~ (.) e^g, Q_G = Q^ (.) e^g, K_E = K~ (.) e^{g_C - g}, the adjoints are
//     dU = K_E dS' + P^T dO,   dR = (I + A)^{-T} dU,   dV~ = dR,
//     dP = lower(dO U^T),      dA = strictly-lower(-dR U^T),
//     dS = Diag(e^{g_C}) dS' + Q_G^T dO - K_G^T dR  =  M^T dS' + Qe^T dO,
// with M = Diag(e^{g_C}) - K'^T W the forward's chunk transition and Qe = Q_G - P W.
// So the state gradient runs backwards over chunks with the forward's own chunk
// quantities (W, Qe, K', e^{g_C}), column by column like the forward scan, and
// every chunk's remaining gradients follow in parallel from (S, dS', dO):
//     dq^_r = e^{g_r} (.) (dO S^T)_r + sum_{i<=r} dP_ri k~_i (.) e^{g_r - g_i}
//     dk~_r = -e^{g_r} (.) (dR S^T)_r + sum_{i<r} dA_ri k~_i (.) e^{g_r - g_i}        ("+" part)
//           + sum_{r'>r} dA_r'r k~_r' (.) e^{g_r' - g_r} + sum_{r'>=r} dP_r'r q^_r' (.) e^{g_r' - g_r}
//           + e^{g_C - g_r} (.) (U dS'^T)_r                                           ("-" part)
//     dg_r  = q^_r (.) dq^_r + k~_r (.) (dk~+_r - dk~-_r),
//     dg_C += e^{g_C} (.) rowsum(S (.) dS') + sum_r k~_r (.) e^{g_C - g_r} (.) (U dS'^T)_r
// and d log alpha_s = sum_{r >= s} dg_r (with dg_C added at the chunk's last row).
// Last, the chain through v~ = sqrt(beta^v) v, k~ = sqrt(beta^k) k^ and the L2
// normalisations: dx = (dx^ - x^ (x^ . dx^)) / ||x||.
//
// Kernels: the forward's intra role (chunk quantities) and scan role (storing the
// state at every chunk start), then rev_scan_kernel (dS' at every chunk end, and
// dS0), then grad_chunk_kernel (one CTA per chunk and head).
#include "gdn.h"
#include "gdn_common.cuh"

namespace gdn {

cudaError_t launch_simt_intra(const Problem& p, bool bf16, cudaStream_t stream);
cudaError_t launch_simt_scan(const Problem& p, bool bf16, cudaStream_t stream);

namespace bwd {

constexpr int NT = 256;
constexpr int kNS = 32;          // d_v columns per reverse-scan CTA and per S tile
constexpr int kLd = kNS + 1;     // padded tile row
constexpr int kMaxRPT = 16;      // rows per thread in the per-element phase: C * dk / NT
constexpr int kGroups = NT / kNS;              // 8 threads per column in the reverse scan
// Kernels are instantiated per rows-per-thread (NR = C / 8, NI = dk / 8 in the reverse
// scan; RPT = C * dk / 256 in the gradient kernel) so unrolled loops have no idle steps.

struct Grads {
    const void* dO;              // [B,T,H,dv], dtype storage
    const float* dS_final;       // [B,H,dk,dv] or null
    float* dq;                   // [B,T,H,dk]
    float* dk;
    float* dv;                   // [B,T,H,dv]
    float* dalpha;               // [B,T,H,dk] or [B,T,H]
    float* dbeta;                // [B,T,H,dk] or [B,T,H]
    float* dbeta_v;              // [B,T,H,dv] or [B,T,H]; only with beta_v
    float* dS0;                  // [B,H,dk,dv]
    float* dS_chunks;            // workspace: dL/dS at every chunk end [B,H,NC,dk,dv]
};

__host__ __device__ inline size_t rev_smem(int C, int dk, int ns = kNS) {
    return sizeof(float) * ((size_t)dk * ns + (size_t)2 * C * ns + (size_t)3 * C * dk + dk);
}

__device__ __forceinline__ void cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((unsigned)__cvta_generic_to_shared(dst)),
                 "l"(src) : "memory");
}
__device__ __forceinline__ void cp_floats(float* dst, const float* src, int n, int tid) {
    for (int i = 4 * tid; i < n; i += 4 * NT) cp16(dst + i, src + i);
}
__device__ __forceinline__ void commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// L2 prefetch of `bytes` (a multiple of 16) from a 16-byte aligned global address
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void wait_all_but_newest() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// One CTA per (d_v slice of NSC columns, head); serial over chunks from last to first.  Per chunk:
// Y = K' dS' (phase A), then dS = Diag(e^{g_C}) dS' - W^T Y + Qe^T dO (phase B).  The
// chunk quantities are fetched one phase ahead with asynchronous copies: K' of chunk c-1
// while phase B of c runs, and W, Qe, e^{g_C}, dO of c-1 while phase A of c-1 runs.
template <typename Tin, int NR, int NI, int NSC = kNS>
__global__ void __launch_bounds__(NT) rev_scan_kernel(Problem p, Grads gr) {
    constexpr int kW = NSC;                  // columns of this CTA
    constexpr int kG = NT / NSC;             // threads per column
    const int j0 = blockIdx.x * kW;
    const int bh = blockIdx.y;
    // the launcher picks NR = C / kG and NI = dk / kG, so both are compile-time here (the loops
    // over rows and channels unroll with constant offsets)
    constexpr int C = kG * NR, dk = kG * NI;
    if (!GDN_IN_BOUNDS(j0 + kW <= p.dv && bh < p.B * p.H && p.C == C && p.dk == dk, p.status)) return;
    const int b = bh / p.H, h = bh % p.H;
    const int dv = p.dv;
    const int tid = threadIdx.x;
    extern __shared__ __align__(16) float sm[];
    float* dS = sm;                          // dk x kW
    float* Y = dS + (size_t)dk * kW;         // C x kW: K' dS'
    float* dOc = Y + (size_t)C * kW;         // C x kW slots: raw dO rows (Tin)
    float* Wc = dOc + (size_t)C * kW;        // C x dk
    float* Qc = Wc + (size_t)C * dk;
    float* Kc = Qc + (size_t)C * dk;
    float* gc = Kc + (size_t)C * dk;         // dk
    const Tin* dO = static_cast<const Tin*>(gr.dO);
    Tin* dOs = reinterpret_cast<Tin*>(dOc);
    constexpr int kRowChunks = kW * (int)sizeof(Tin) / 16;   // 16-byte pieces of one row slice

    InterF32 L{C, dk, dv};
    const float* inter = static_cast<const float*>(p.inter);
    auto block = [&](int c) { return inter + ((size_t)bh * p.NC + c) * L.floats(); };
    auto fetch_a = [&](int c) {
        if (c >= 0) cp_floats(Kc, block(c) + L.Kp(), C * dk, tid);
        commit_group();
    };
    auto fetch_b = [&](int c) {
        if (c >= 0) {
            const float* in = block(c);
            cp_floats(Wc, in + L.W(), C * dk, tid);
            cp_floats(Qc, in + L.Qe(), C * dk, tid);
            cp_floats(gc, in + L.gC(), dk, tid);
            for (int i = tid; i < C * kRowChunks; i += NT) {
                const int r = i / kRowChunks, q16 = i % kRowChunks;
                const int s = c * C + r;
                Tin* dst = dOs + (size_t)r * kW;
                bool ok = false;
                if (s < p.L) {
                    const RowRef rr = row_ref(p, b, h, s);
                    if (rr.has_q) {
                        cp16(reinterpret_cast<char*>(dst) + 16 * q16,
                             reinterpret_cast<const char*>(dO + rr.tok * dv + j0) + 16 * q16);
                        ok = true;
                    }
                }
                if (!ok) *reinterpret_cast<uint4*>(reinterpret_cast<char*>(dst) + 16 * q16) = make_uint4(0, 0, 0, 0);
            }
        }
        commit_group();
    };

    for (int idx = tid; idx < dk * kW; idx += NT) {
        const int i = idx / kW, j = idx % kW;
        dS[idx] = gr.dS_final ? gr.dS_final[((size_t)bh * dk + i) * dv + j0 + j] : 0.f;
    }
    fetch_a(p.NC - 1);
    fetch_b(p.NC - 1);
    for (int c = p.NC - 1; c >= 0; --c) {
        wait_all_but_newest();               // K' of chunk c
        __syncthreads();                     // ... for all; dS' of chunk c is complete
        float* dst = gr.dS_chunks + ((size_t)bh * p.NC + c) * dk * dv;
        for (int idx = tid; idx < dk * kW; idx += NT) {
            const int i = idx / kW, j = idx % kW;
            dst[(size_t)i * dv + j0 + j] = dS[idx];
        }
        {   // thread: column j, rows rg, rg + 8, ...; each dS'[i][j] read once for all its rows
            const int j = tid % kW, rg = tid / kW;
            float acc[NR];
#pragma unroll
            for (int m = 0; m < NR; ++m) acc[m] = 0.f;
            for (int i = 0; i < dk; i += 4) {    // K' rows as float4 along i
                const float x0 = dS[(size_t)i * kW + j], x1 = dS[(size_t)(i + 1) * kW + j];
                const float x2 = dS[(size_t)(i + 2) * kW + j], x3 = dS[(size_t)(i + 3) * kW + j];
#pragma unroll
                for (int m = 0; m < NR; ++m) {
                    const float4 kk = *reinterpret_cast<const float4*>(Kc + (size_t)(rg + kG * m) * dk + i);
                    acc[m] = fmaf(kk.w, x3, fmaf(kk.z, x2, fmaf(kk.y, x1, fmaf(kk.x, x0, acc[m]))));
                }
            }
#pragma unroll
            for (int m = 0; m < NR; ++m) Y[(size_t)(rg + kG * m) * kW + j] = acc[m];
        }
        __syncthreads();                     // K' buffer free; Y complete
        fetch_a(c - 1);
        wait_all_but_newest();               // W, Qe, e^{g_C}, dO of chunk c
        __syncthreads();
        // dS <- Diag(gC) dS' - W^T Y + Qe^T dO   (element (i, j) reads only its own dS')
        {   // thread: column j, state rows i0 .. i0 + NI - 1 (contiguous, so the Qe and W rows
            // load as float4); dO[r][j], Y[r][j] read once per r
            const int j = tid % kW, i0 = (tid / kW) * NI;
            float acc[NI];
#pragma unroll
            for (int m = 0; m < NI; ++m) acc[m] = gc[i0 + m] * dS[(size_t)(i0 + m) * kW + j];
            for (int r = 0; r < C; ++r) {
                const float d = load_in(dOs, (size_t)r * kW + j), y = Y[(size_t)r * kW + j];
                const float4* qv = reinterpret_cast<const float4*>(Qc + (size_t)r * dk + i0);
                const float4* wv = reinterpret_cast<const float4*>(Wc + (size_t)r * dk + i0);
#pragma unroll
                for (int m4 = 0; m4 < NI / 4; ++m4) {
                    const float4 qq = qv[m4], ww = wv[m4];
                    acc[4 * m4 + 0] = fmaf(-ww.x, y, fmaf(qq.x, d, acc[4 * m4 + 0]));
                    acc[4 * m4 + 1] = fmaf(-ww.y, y, fmaf(qq.y, d, acc[4 * m4 + 1]));
                    acc[4 * m4 + 2] = fmaf(-ww.z, y, fmaf(qq.z, d, acc[4 * m4 + 2]));
                    acc[4 * m4 + 3] = fmaf(-ww.w, y, fmaf(qq.w, d, acc[4 * m4 + 3]));
                }
            }
#pragma unroll
            for (int m = 0; m < NI; ++m) dS[(size_t)(i0 + m) * kW + j] = acc[m];
        }
        __syncthreads();                     // W, Qe, e^{g_C}, dO buffers free
        fetch_b(c - 1);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (gr.dS0) {
        for (int idx = tid; idx < dk * kW; idx += NT) {
            const int i = idx / kW, j = idx % kW;
            gr.dS0[((size_t)bh * dk + i) * dv + j0 + j] = dS[idx];
        }
    }
}

__host__ __device__ inline size_t grad_smem(int C, int dk, int dv) {
    return sizeof(float) * ((size_t)5 * C * dk + (size_t)4 * C * dv + (size_t)4 * C * C +
                            (size_t)2 * dk * kLd + 2 * C + dk);
}

// One CTA per (chunk, head).  kC, kDK, kDV: the sizes as compile-time constants (0: read from
// the problem), so that the common shapes' loops unroll with constant offsets.  At d = 128 and
// chunk 16 the shared memory allows two CTAs per SM, which the register budget is then sized
// for (at chunk 32 it allows one).
template <typename Tin, int RPT, int kC = 0, int kDK = 0, int kDV = 0>
__global__ void __launch_bounds__(NT, (kDK == 128 && kC == 16) ? 2 : 1) grad_chunk_kernel(Problem p, Grads gr) {
    const int c = blockIdx.x;
    const int bh = blockIdx.y;
    const int C = kC ? kC : p.C, dk = kDK ? kDK : p.dk, dv = kDV ? kDV : p.dv;
    if (!GDN_IN_BOUNDS(c < p.NC && bh < p.B * p.H && C == p.C && dk == p.dk && dv == p.dv, p.status)) return;
    const int b = bh / p.H, h = bh % p.H;
    const int s0 = c * C;
    const int Cv = min(C, p.L - s0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int nwarps = NT / 32;

    extern __shared__ __align__(16) float sm[];
    float* qh = sm;                          // q^                      C x dk
    float* kt = qh + (size_t)C * dk;         // k~
    float* g = kt + (size_t)C * dk;          // log alpha, then cumulative
    float* KG = g + (size_t)C * dk;          // k~ e^g,          later dq^
    float* KE = KG + (size_t)C * dk;         // k~ e^{g_C - g},  later dk~
    float* vt = KE + (size_t)C * dk;         // v~                      C x dv
    float* dOs = vt + (size_t)C * dv;        // dO
    float* U = dOs + (size_t)C * dv;         // R, then U
    float* dR = U + (size_t)C * dv;          // K_E dS', then dU, then dR
    float* A = dR + (size_t)C * dv;          // C x C
    float* P = A + (size_t)C * C;
    float* dP = P + (size_t)C * C;
    float* dA = dP + (size_t)C * C;
    float* St = dA + (size_t)C * C;          // S tile   dk x kLd,  later dg (C x dk)
    float* dSt = St + (size_t)dk * kLd;      // dS' tile dk x kLd
    float* iq = dSt + (size_t)dk * kLd;      // 1 / ||q_r||             C
    float* ik = iq + C;                      // 1 / ||k_r||             C
    float* dgC = ik + C;                     // dk

    const Tin* q = static_cast<const Tin*>(p.q);
    const Tin* k = static_cast<const Tin*>(p.k);
    const Tin* v = static_cast<const Tin*>(p.v);
    const Tin* dO = static_cast<const Tin*>(gr.dO);
    const float* bvsrc = p.beta_v ? p.beta_v : p.beta;
    const int bvstride = p.beta_v ? dv : dk;

    // The chunk's S and dS' (read by phases 3 and 6, each twice) into L2 while the rows and the
    // Gram products are formed.
    if (tid == 0) {
        const size_t n = (size_t)dk * dv;
        bulk_prefetch_l2(p.S_chunks + ((size_t)bh * p.NC + c) * n, (uint32_t)(n * sizeof(float)));
        bulk_prefetch_l2(gr.dS_chunks + ((size_t)bh * p.NC + c) * n, (uint32_t)(n * sizeof(float)));
    }
    // 1. rows: q^, k~, v~, log alpha, dO.  Every load of a row is issued before any is used (one
    // round trip to memory per row).
    constexpr int kJ = 4;                    // channels per lane (d <= 128)
    for (int r = warp; r < C; r += nwarps) {
        float* qr = qh + (size_t)r * dk;
        float* kr = kt + (size_t)r * dk;
        float* gq = g + (size_t)r * dk;
        if (r < Cv) {
            const RowRef rr = row_ref(p, b, h, s0 + r);
            float xq[kJ], xk[kJ], xa[kJ], xb[kJ], xv[kJ], xo[kJ], xbv[kJ];
#pragma unroll
            for (int u = 0; u < kJ; ++u) {
                const int j = lane + 32 * u;
                if (j < dk) {
                    xq[u] = load_in(q, rr.tok * dk + j);
                    xk[u] = load_in(k, rr.tok * dk + j);
                    xa[u] = p.alpha_scalar ? 0.f : p.alpha[rr.tok * dk + j];
                    xb[u] = p.beta_scalar ? 0.f : p.beta[rr.tok * dk + j];
                }
                if (j < dv) {
                    xv[u] = load_in(v, rr.tok * dv + j);
                    xo[u] = load_in(dO, rr.tok * dv + j);
                    xbv[u] = p.beta_scalar ? 0.f : bvsrc[rr.tok * bvstride + j];
                }
            }
            const float as = p.alpha_scalar ? p.alpha[rr.tok] : 0.f;
            const float bsr = p.beta_scalar ? p.beta[rr.tok] : 0.f;
            const float bvr = p.beta_scalar ? bvsrc[rr.tok] : 0.f;
            float ssq = 0.f, ssk = 0.f;
#pragma unroll
            for (int u = 0; u < kJ; ++u)
                if (lane + 32 * u < dk) {
                    ssq += xq[u] * xq[u];
                    ssk += xk[u] * xk[u];
                }
            const float a = rsqrtf(warp_sum(ssq) + kNormEps);
            const float bk = rsqrtf(warp_sum(ssk) + kNormEps);
            if (lane == 0) {
                iq[r] = a;
                ik[r] = bk;
            }
            const float bs = p.beta_scalar ? sqrtf(bsr) : 0.f;
            const float la = p.alpha_scalar ? logf(as) : 0.f;
            const float bvs = p.beta_scalar ? sqrtf(bvr) : 0.f;
#pragma unroll
            for (int u = 0; u < kJ; ++u) {
                const int j = lane + 32 * u;
                if (j < dk) {
                    qr[j] = xq[u] * a;
                    kr[j] = xk[u] * (bk * (p.beta_scalar ? bs : sqrtf(xb[u])));
                    gq[j] = p.alpha_scalar ? la : logf(xa[u]);
                }
                if (j < dv) {
                    const float sb = p.beta_scalar ? bvs : sqrtf(xbv[u]);
                    vt[(size_t)r * dv + j] = xv[u] * sb;
                    dOs[(size_t)r * dv + j] = xo[u];
                }
            }
        } else {
            for (int j = lane; j < dk; j += 32) { qr[j] = 0.f; kr[j] = 0.f; gq[j] = 0.f; }
            for (int j = lane; j < dv; j += 32) { vt[(size_t)r * dv + j] = 0.f; dOs[(size_t)r * dv + j] = 0.f; }
            if (lane == 0) { iq[r] = 0.f; ik[r] = 0.f; }
        }
    }
    __syncthreads();
    for (int j = tid; j < dk; j += NT) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += g[(size_t)r * dk + j];
            g[(size_t)r * dk + j] = acc;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * dk; idx += NT) {
        const int j = idx % dk;
        const float gl = g[(size_t)(C - 1) * dk + j];
        KG[idx] = kt[idx] * expf(g[idx]);
        KE[idx] = kt[idx] * expf(gl - g[idx]);
    }
    // 2. A (i < r) and P (i <= r), decay formed element by element.  Warp w takes rows
    // 16 m + w and 16 m + 15 - w (the same number of pairs for every warp); its lanes run over
    // channels and hold the partial sums of 16 A and 16 P entries at a time, which one butterfly
    // of 31 shuffles reduces (lane l ends with entry l; the same pairing as a warp sum per entry).
    {
        const unsigned full = 0xffffffffu;
        for (int k = 0; k < C / 8; ++k) {
            const int r = 16 * (k >> 1) + ((k & 1) ? 15 - warp : warp);
            float kr_[kJ], qr_[kJ], gr_[kJ];
#pragma unroll
            for (int u = 0; u < kJ; ++u) {
                const int j = lane + 32 * u;
                if (j < dk) {
                    kr_[u] = kt[(size_t)r * dk + j];
                    qr_[u] = qh[(size_t)r * dk + j];
                    gr_[u] = g[(size_t)r * dk + j];
                }
            }
            for (int ih = 0; ih < C; ih += 16) {
                float v[32];                 // v[t]: A[r][ih + t], v[16 + t]: P[r][ih + t]
#pragma unroll
                for (int t = 0; t < 32; ++t) v[t] = 0.f;
                if (ih <= r) {
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int i = ih + t;
                        if (i <= r) {
#pragma unroll
                            for (int u = 0; u < kJ; ++u) {
                                const int j = lane + 32 * u;
                                if (j < dk) {
                                    const float ke = kt[(size_t)i * dk + j] * expf(gr_[u] - g[(size_t)i * dk + j]);
                                    v[16 + t] += qr_[u] * ke;
                                    v[t] += kr_[u] * ke;
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int off = 16; off >= 1; off >>= 1) {
                        const bool upper = (lane & off) != 0;
#pragma unroll
                        for (int t = 0; t < off; ++t) {
                            const float send = upper ? v[t] : v[t + off];
                            const float keep = upper ? v[t + off] : v[t];
                            v[t] = keep + __shfl_xor_sync(full, send, off);
                        }
                    }
                }
                const int i = ih + (lane & 15);
                if (lane < 16) A[(size_t)r * C + i] = (i < r) ? v[0] : 0.f;
                else P[(size_t)r * C + i] = (i <= r) ? v[0] : 0.f;
            }
        }
    }
    __syncthreads();

    const float* Sg = p.S_chunks + ((size_t)bh * p.NC + c) * dk * dv;
    const float* dSg = gr.dS_chunks + ((size_t)bh * p.NC + c) * dk * dv;
    // A dk x kNS tile of S and dS' (columns jt ..): this thread's share, loaded into registers
    // one tile ahead of its use (the load is in flight while the previous tile is worked on)
    constexpr int kTV = (kDK ? kDK : 128) * kNS / NT;     // values per thread (dk <= 128)
    float ts[kTV], tds[kTV];
    auto tile_load = [&](int jt) {
#pragma unroll
        for (int m = 0; m < kTV; ++m) {
            const int idx = tid + m * NT;
            if (idx < dk * kNS) {
                const int i = idx / kNS, jj = idx % kNS;
                ts[m] = Sg[(size_t)i * dv + jt + jj];
                tds[m] = dSg[(size_t)i * dv + jt + jj];
            }
        }
    };
    auto tile_store = [&]() {
#pragma unroll
        for (int m = 0; m < kTV; ++m) {
            const int idx = tid + m * NT;
            if (idx < dk * kNS) {
                const int i = idx / kNS, jj = idx % kNS;
                St[i * kLd + jj] = ts[m];
                dSt[i * kLd + jj] = tds[m];
            }
        }
    };
    // 3. R = V~ - K_G S and K_E dS', tile by tile over d_v
    tile_load(0);
    for (int jt = 0; jt < dv; jt += kNS) {
        tile_store();
        __syncthreads();
        if (jt + kNS < dv) tile_load(jt + kNS);
        {   // thread: column jj, rows r0, r0 + 8, ... (C / 8 of them, at most 4); each S and dS'
            // element is read once for all of them, K_G and K_E rows as float4 along i
            constexpr int kMaxRows = 4, kRowStep = NT / kNS;
            const int jj = tid % kNS, r0 = tid / kNS, nr = C / kRowStep;
            float ks[kMaxRows], kd[kMaxRows];
#pragma unroll
            for (int m = 0; m < kMaxRows; ++m) { ks[m] = 0.f; kd[m] = 0.f; }
            for (int i = 0; i < dk; i += 4) {
                const float s0 = St[i * kLd + jj], s1 = St[(i + 1) * kLd + jj];
                const float s2 = St[(i + 2) * kLd + jj], s3 = St[(i + 3) * kLd + jj];
                const float d0 = dSt[i * kLd + jj], d1 = dSt[(i + 1) * kLd + jj];
                const float d2 = dSt[(i + 2) * kLd + jj], d3 = dSt[(i + 3) * kLd + jj];
#pragma unroll
                for (int m = 0; m < kMaxRows; ++m) {
                    if (m < nr) {
                        const size_t ro = (size_t)(r0 + kRowStep * m) * dk + i;
                        const float4 g4 = *reinterpret_cast<const float4*>(KG + ro);
                        const float4 e4 = *reinterpret_cast<const float4*>(KE + ro);
                        ks[m] = fmaf(g4.w, s3, fmaf(g4.z, s2, fmaf(g4.y, s1, fmaf(g4.x, s0, ks[m]))));
                        kd[m] = fmaf(e4.w, d3, fmaf(e4.z, d2, fmaf(e4.y, d1, fmaf(e4.x, d0, kd[m]))));
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < kMaxRows; ++m) {
                if (m < nr) {
                    const size_t o = (size_t)(r0 + kRowStep * m) * dv + jt + jj;
                    U[o] = vt[o] - ks[m];
                    dR[o] = kd[m];
                }
            }
        }
        __syncthreads();
    }
    // 4. dU = K_E dS' + P^T dO, then U = (I + A)^{-1} R (forward substitution) and
    //    dR = (I + A)^{-T} dU (back substitution).  Each substitution runs down one column per
    //    thread, in registers: threads 0 .. NT/2 - 1 take U's columns, the others dR's (the two
    //    are independent), so no barrier is needed between rows.
    for (int idx = tid; idx < C * dv; idx += NT) {
        const int i = idx / dv, j = idx % dv;
        float acc = dR[idx];
        for (int r = i; r < C; ++r) acc += P[(size_t)r * C + i] * dOs[(size_t)r * dv + j];
        dR[idx] = acc;
    }
    __syncthreads();
    {
        constexpr int kMaxC = kC ? kC : 32;  // rows (the chunk; at most 32)
        constexpr int half = NT / 2;
        const bool second = tid >= half;
        float* X = second ? dR : U;
        for (int j = second ? tid - half : tid; j < dv; j += half) {
            float x[kMaxC];
#pragma unroll
            for (int r = 0; r < kMaxC; ++r)
                if (r < C) x[r] = X[(size_t)r * dv + j];
            if (!second) {
#pragma unroll
                for (int r = 1; r < kMaxC; ++r) {
                    if (r < C) {
                        float acc = x[r];
#pragma unroll
                        for (int i = 0; i < r; ++i) acc -= A[(size_t)r * C + i] * x[i];
                        x[r] = acc;
                    }
                }
            } else {
#pragma unroll
                for (int r = kMaxC - 2; r >= 0; --r) {
                    if (r <= C - 2) {
                        float acc = x[r];
#pragma unroll
                        for (int i = r + 1; i < kMaxC; ++i)
                            if (i < C) acc -= A[(size_t)i * C + r] * x[i];
                        x[r] = acc;
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < kMaxC; ++r)
                if (r < C) X[(size_t)r * dv + j] = x[r];
        }
    }
    __syncthreads();
    // 5. dP = lower(dO U^T), dA = strictly-lower(-dR U^T).  Where U^T (rows padded to C + 1)
    //    fits the free tile buffers: one thread per (r, i) pair with no cross-lane reduction
    //    (a warp's lanes read consecutive i of U^T; dO and dR rows are broadcasts); otherwise
    //    one warp per pair.
    if ((size_t)dv * (C + 1) <= (size_t)2 * dk * kLd) {
        float* Ut = St;
        for (int idx = tid; idx < C * dv; idx += NT) {
            const int i = idx / dv, j = idx % dv;
            Ut[(size_t)j * (C + 1) + i] = U[idx];
        }
        __syncthreads();
        for (int pr = tid; pr < C * C; pr += NT) {
            const int r = pr / C, i = pr % C;
            float a = 0.f, pp = 0.f;
            if (i <= r) {
                for (int j = 0; j < dv; ++j) {
                    const float u = Ut[(size_t)j * (C + 1) + i];
                    pp += dOs[(size_t)r * dv + j] * u;
                    a -= dR[(size_t)r * dv + j] * u;
                }
            }
            dA[pr] = (i < r) ? a : 0.f;
            dP[pr] = pp;
        }
    } else {
        for (int pr = warp; pr < C * C; pr += nwarps) {
            const int r = pr / C, i = pr % C;
            float a = 0.f, pp = 0.f;
            if (i <= r) {
                for (int j = lane; j < dv; j += 32) {
                    const float u = U[(size_t)i * dv + j];
                    pp += dOs[(size_t)r * dv + j] * u;
                    a -= dR[(size_t)r * dv + j] * u;
                }
                a = warp_sum(a);
                pp = warp_sum(pp);
            }
            if (lane == 0) {
                dA[pr] = (i < r) ? a : 0.f;
                dP[pr] = pp;
            }
        }
    }
    // 6. dO S^T, dR S^T, U dS'^T (thread: column cc, rows r0 + rstep * m) and rowsum(S (.) dS')
    const int cc = tid % dk, r0 = tid / dk, rstep = NT / dk;
    float G1[RPT], G2[RPT], G3[RPT], G4 = 0.f;
#pragma unroll
    for (int m = 0; m < RPT; ++m) { G1[m] = 0.f; G2[m] = 0.f; G3[m] = 0.f; }
    tile_load(0);
    for (int jt = 0; jt < dv; jt += kNS) {
        __syncthreads();
        tile_store();
        __syncthreads();
        if (jt + kNS < dv) tile_load(jt + kNS);
        for (int jj = 0; jj < kNS; jj += 4) {   // four columns at a time: row data as float4
            float sv[4], dv4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sv[e] = St[cc * kLd + jj + e];
                dv4[e] = dSt[cc * kLd + jj + e];
                if (r0 == 0) G4 += sv[e] * dv4[e];
            }
#pragma unroll
            for (int m = 0; m < RPT; ++m) {
                const size_t o = (size_t)(r0 + rstep * m) * dv + jt + jj;
                const float4 a = *reinterpret_cast<const float4*>(dOs + o);
                const float4 rr4 = *reinterpret_cast<const float4*>(dR + o);
                const float4 u = *reinterpret_cast<const float4*>(U + o);
                G1[m] = fmaf(a.w, sv[3], fmaf(a.z, sv[2], fmaf(a.y, sv[1], fmaf(a.x, sv[0], G1[m]))));
                G2[m] = fmaf(rr4.w, sv[3], fmaf(rr4.z, sv[2], fmaf(rr4.y, sv[1], fmaf(rr4.x, sv[0], G2[m]))));
                G3[m] = fmaf(u.w, dv4[3], fmaf(u.z, dv4[2], fmaf(u.y, dv4[1], fmaf(u.x, dv4[0], G3[m]))));
            }
        }
    }
    __syncthreads();
    const float gCc = g[(size_t)(C - 1) * dk + cc];
    if (r0 == 0) dgC[cc] = expf(gCc) * G4;
    __syncthreads();
    // 7. dq^, dk~ and dg per element
    float* Dg = St;
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int r = r0 + rstep * m;
        const size_t e = (size_t)r * dk + cc;
        const float grc = g[e];
        float dq = expf(grc) * G1[m];
        float dkp = -expf(grc) * G2[m];
        float dkm = expf(gCc - grc) * G3[m];
        const float ke3 = KE[e] * G3[m];
        for (int i = 0; i <= r; ++i) {
            const float w = kt[(size_t)i * dk + cc] * expf(grc - g[(size_t)i * dk + cc]);
            dq += dP[(size_t)r * C + i] * w;
            if (i < r) dkp += dA[(size_t)r * C + i] * w;
        }
        for (int i = r; i < C; ++i) {
            const float ex = expf(g[(size_t)i * dk + cc] - grc);
            dkm += dP[(size_t)i * C + r] * qh[(size_t)i * dk + cc] * ex;
            if (i > r) dkm += dA[(size_t)i * C + r] * kt[(size_t)i * dk + cc] * ex;
        }
        atomicAdd(&dgC[cc], ke3);
        Dg[e] = qh[e] * dq + kt[e] * (dkp - dkm);
        KG[e] = dq;
        KE[e] = dkp + dkm;
    }
    __syncthreads();
    // 8. d log alpha = reverse cumulative sum of dg (dg_C at the last row)
    for (int j = tid; j < dk; j += NT) {
        float acc = dgC[j];
        for (int r = C - 1; r >= 0; --r) {
            acc += Dg[(size_t)r * dk + j];
            Dg[(size_t)r * dk + j] = acc;
        }
    }
    __syncthreads();
    // 9. chain through the rates, alpha and the normalisations, one row per warp
    for (int r = warp; r < Cv; r += nwarps) {
        const size_t t = row_ref(p, b, h, s0 + r).tok;
        const float* qr = qh + (size_t)r * dk;
        const float* dqr = KG + (size_t)r * dk;      // dq^
        const float* dkr = KE + (size_t)r * dk;      // dk~
        const float sbk_s = p.beta_scalar ? sqrtf(p.beta[t]) : 0.f;
        const float sbv_s = p.beta_scalar ? sqrtf(bvsrc[t]) : 0.f;
        float dotq = 0.f, dotk = 0.f;
        for (int j = lane; j < dk; j += 32) {
            const float sb = p.beta_scalar ? sbk_s : sqrtf(p.beta[t * dk + j]);
            dotq += qr[j] * dqr[j];
            dotk += load_in(k, t * dk + j) * ik[r] * sb * dkr[j];
        }
        dotq = warp_sum(dotq);
        dotk = warp_sum(dotk);
        float dbk = 0.f, dbv = 0.f, dal = 0.f;
        for (int j = lane; j < dk; j += 32) {
            const float sb = p.beta_scalar ? sbk_s : sqrtf(p.beta[t * dk + j]);
            const float khat = load_in(k, t * dk + j) * ik[r];
            if (gr.dq) gr.dq[t * dk + j] = (dqr[j] - qr[j] * dotq) * iq[r];
            if (gr.dk) gr.dk[t * dk + j] = (sb * dkr[j] - khat * dotk) * ik[r];
            float db = dkr[j] * khat * 0.5f / sb;             // d sqrt(b) / db = 1 / (2 sqrt(b))
            if (!p.beta_v && !p.beta_scalar)                   // one rate on k and v (dk == dv)
                db += dR[(size_t)r * dv + j] * load_in(v, t * dv + j) * 0.5f / sb;
            if (p.beta_scalar) dbk += db;
            else if (gr.dbeta) gr.dbeta[t * dk + j] = db;
            const float dla = Dg[(size_t)r * dk + j];          // d log alpha
            if (p.alpha_scalar) dal += dla;
            else if (gr.dalpha) gr.dalpha[t * dk + j] = dla / p.alpha[t * dk + j];
        }
        for (int j = lane; j < dv; j += 32) {
            const float sb = p.beta_scalar ? sbv_s : sqrtf(bvsrc[t * bvstride + j]);
            const float dvt = dR[(size_t)r * dv + j];
            if (gr.dv) gr.dv[t * dv + j] = sb * dvt;
            const float db = dvt * load_in(v, t * dv + j) * 0.5f / sb;
            if (p.beta_scalar) dbv += db;
            else if (p.beta_v && gr.dbeta_v) gr.dbeta_v[t * dv + j] = db;
        }
        if (p.alpha_scalar) {
            dal = warp_sum(dal);
            if (lane == 0 && gr.dalpha) gr.dalpha[t] = dal / p.alpha[t];
        }
        if (p.beta_scalar) {
            dbk = warp_sum(dbk);
            dbv = warp_sum(dbv);
            if (lane == 0) {
                if (p.beta_v) {
                    if (gr.dbeta) gr.dbeta[t] = dbk;
                    if (gr.dbeta_v) gr.dbeta_v[t] = dbv;
                } else if (gr.dbeta) {
                    gr.dbeta[t] = dbk + dbv;
                }
            }
        }
    }
}

template <typename Tin, int NR, int NI, int NSC = kNS>
cudaError_t launch_rev(const Problem& p, const Grads& gr, cudaStream_t stream) {
    const size_t s3 = rev_smem(p.C, p.dk, NSC);
    auto kern = rev_scan_kernel<Tin, NR, NI, NSC>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3);
    if (e != cudaSuccess) return e;
    kern<<<dim3(p.dv / NSC, p.B * p.H), NT, s3, stream>>>(p, gr);
    return cudaGetLastError();
}

template <typename Tin, int NR>
cudaError_t launch_rev_nr(const Problem& p, const Grads& gr, cudaStream_t stream) {
    switch (p.dk / kGroups) {
        case 4: return launch_rev<Tin, NR, 4>(p, gr, stream);
        case 8: return launch_rev<Tin, NR, 8>(p, gr, stream);
        case 16: return launch_rev<Tin, NR, 16>(p, gr, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin, int RPT, int kC = 0, int kDK = 0, int kDV = 0>
cudaError_t launch_grad(const Problem& p, const Grads& gr, cudaStream_t stream) {
    const size_t s4 = grad_smem(p.C, p.dk, p.dv);
    auto kern = grad_chunk_kernel<Tin, RPT, kC, kDK, kDV>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s4);
    if (e != cudaSuccess) return e;
    kern<<<dim3(p.NC, p.B * p.H), NT, s4, stream>>>(p, gr);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_rev_t(const Problem& p, const Grads& gr, cudaStream_t stream) {
    // d_k = 128: slices of 16 columns (16 threads per column), twice the CTAs of 32-column
    // slices for the same serial chain, each step with half the work
    if (p.dk == 128) {
        if (p.C == 16) return launch_rev<Tin, 1, 8, 16>(p, gr, stream);
        if (p.C == 32) return launch_rev<Tin, 2, 8, 16>(p, gr, stream);
    }
    return (p.C / kGroups == 2) ? launch_rev_nr<Tin, 2>(p, gr, stream)
         : (p.C / kGroups == 4) ? launch_rev_nr<Tin, 4>(p, gr, stream) : cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t launch_grad_t(const Problem& p, const Grads& gr, cudaStream_t stream) {
    if (p.dk == 128 && p.dv == 128) {        // d = 128: the sizes as constants
        if (p.C == 16) return launch_grad<Tin, 8, 16, 128, 128>(p, gr, stream);
        if (p.C == 32) return launch_grad<Tin, 16, 32, 128, 128>(p, gr, stream);
    }
    switch (p.C * p.dk / NT) {
        case 2: return launch_grad<Tin, 2>(p, gr, stream);
        case 4: return launch_grad<Tin, 4>(p, gr, stream);
        case 8: return launch_grad<Tin, 8>(p, gr, stream);
        case 16: return launch_grad<Tin, 16>(p, gr, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace bwd

bool bwd_supported(int C, int dk, int dv) {
    return (C == 16 || C == 32) && (size_t)C * dk <= (size_t)bwd::kMaxRPT * bwd::NT &&
           bwd::grad_smem(C, dk, dv) <= 227 * 1024 && bwd::rev_smem(C, dk) <= 227 * 1024;
}

// Workspace after the header: the forward's chunk quantities, then the states at
// every chunk start, then the state gradients at every chunk end (each 256-aligned).
size_t bwd_inter_bytes(const Problem& p, size_t fwd_inter) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t states = (size_t)p.B * p.H * p.NC * p.dk * p.dv * sizeof(float);
    return up(fwd_inter) + 2 * up(states);
}

int bwd_launches(const Problem& p) { return p.NC > 0 ? 4 : 1; }

cudaError_t launch_bwd(Problem p, const void* dO, const float* dS_final, float* dq, float* dk,
                       float* dv, float* dalpha, float* dbeta, float* dbeta_v, float* dS0,
                       size_t fwd_inter, bool bf16, cudaStream_t stream) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t states = (size_t)p.B * p.H * p.NC * p.dk * p.dv * sizeof(float);
    char* base = static_cast<char*>(p.inter);
    p.S_chunks = reinterpret_cast<float*>(base + up(fwd_inter));
    bwd::Grads gr{dO, dS_final, dq, dk, dv, dalpha, dbeta, dbeta_v, dS0,
                  reinterpret_cast<float*>(base + up(fwd_inter) + up(states))};
    auto rev = [&](cudaStream_t st) {
        return bf16 ? bwd::launch_rev_t<__nv_bfloat16>(p, gr, st) : bwd::launch_rev_t<float>(p, gr, st);
    };
    if (p.NC == 0) return rev(stream);        // dS0 = dS_final
    Problem f = p;                             // state recompute: no outputs, chunk-start states kept
    f.out = nullptr;
    f.S_final = nullptr;
    cudaError_t e = launch_simt_intra(f, bf16, stream);
    if (e != cudaSuccess) return e;
    {
        // The recompute scan (forward over chunks) and the state-gradient scan (backward over
        // chunks) both read only the chunk blocks: run them side by side, the second on the
        // side stream, and join before the gradient kernel.
        std::unique_lock<std::mutex> lock;
        SideStream* ss = side_stream_lock(lock);
        if (!ss) {
            e = launch_simt_scan(f, bf16, stream);
            if (e == cudaSuccess) e = rev(stream);
        } else {
            e = cudaEventRecord(ss->fork, stream);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->stream, ss->fork, 0);
            if (e == cudaSuccess) e = rev(ss->stream);
            if (e == cudaSuccess) e = launch_simt_scan(f, bf16, stream);
            cudaError_t j = cudaEventRecord(ss->join, ss->stream);
            if (j == cudaSuccess) j = cudaStreamWaitEvent(stream, ss->join, 0);
            if (e == cudaSuccess) e = j;
        }
    }
    if (e != cudaSuccess) return e;
    return bf16 ? bwd::launch_grad_t<__nv_bfloat16>(p, gr, stream) : bwd::launch_grad_t<float>(p, gr, stream);
}

}  // namespace gdn
