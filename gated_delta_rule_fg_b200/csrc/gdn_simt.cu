// gdn_simt.cu -- float32 CUDA-core kernels for the two roles of the chunkwise
// FG^2-GDN forward (see gdn_common.cuh).  This is the float32 precision path
// (every product in fp32 FMA, decay factors exp(g_r - g_i) formed element by
// element so nothing overflows for any alpha in (0,1]) and the path for shapes
// the tensor-core kernels do not cover.
#include "gdn_common.cuh"

namespace gdn {

constexpr int kSimtThreads = 256;
constexpr int kScanCols = 32;   // d_v columns of the state owned by one scan CTA
constexpr int kRowGroups = kSimtThreads / kScanCols;   // 8: threads per column in the scan
// The scan kernel is instantiated per (chunk rows, state rows) a thread carries:
// NR = C / 8 and NI = dk / 8, so its unrolled loops carry no idle iterations.

// Shared memory of the intra kernel: qh, kt, g (C x dk), vt, Up (C x dv), A, Tm, P (C x C),
// and for GDN2 the erase vectors (C x dk).
__host__ __device__ inline size_t intra_simt_smem(int C, int dk, int dv, bool gdn2 = false) {
    return sizeof(float) * ((size_t)(gdn2 ? 4 : 3) * C * dk + (size_t)2 * C * dv + (size_t)3 * C * C);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// One CTA per (chunk, head).  kC, kDK, kDV: the sizes as compile-time constants (0: read from
// the problem), so that the common shapes' loops unroll with constant offsets.
template <typename Tin, int kC = 0, int kDK = 0, int kDV = 0>
__global__ void __launch_bounds__(kSimtThreads)
intra_simt_kernel(Problem p) {
    const int c = blockIdx.x;
    const int bh = blockIdx.y;
    const int C = kC ? kC : p.C, dk = kDK ? kDK : p.dk, dv = kDV ? kDV : p.dv;
    if (!GDN_IN_BOUNDS(c < p.NC && bh < p.B * p.H && C == p.C && dk == p.dk && dv == p.dv, p.status))
        return;                                                          // the whole CTA, before any barrier
    const int b = bh / p.H, h = bh % p.H;
    const int s0 = c * C;
    const int Cv = min(C, p.L - s0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int nwarps = kSimtThreads / 32;

    extern __shared__ float sm[];
    float* qh = sm;                      // q^ rows, later q^ (.) e^g
    float* kt = qh + (size_t)C * dk;     // k~ rows, later k~ (.) e^g
    float* g = kt + (size_t)C * dk;      // log alpha, cumulative; later W
    float* vt = g + (size_t)C * dk;      // v~ rows
    float* Up = vt + (size_t)C * dv;     // U' = T V~
    float* A = Up + (size_t)C * dv;      // strictly lower A
    float* Tm = A + (size_t)C * C;       // T = (I + A)^{-1}
    float* P = Tm + (size_t)C * C;       // lower P
    const bool gdn2 = p.gdn2_eta != nullptr;
    // erase vectors: the rows A and the state read use (j' for GDN2; k~ itself otherwise)
    float* ew = gdn2 ? P + (size_t)C * C : kt;

    const Tin* q = static_cast<const Tin*>(p.q);
    const Tin* k = static_cast<const Tin*>(p.k);
    const Tin* v = static_cast<const Tin*>(p.v);

    // 1. rows: normalise q, k; sqrt(beta) scaling; log alpha.
    for (int r = warp; r < C; r += nwarps) {
        float* qr = qh + (size_t)r * dk;
        float* kr = kt + (size_t)r * dk;
        float* gr = g + (size_t)r * dk;
        float* vr = vt + (size_t)r * dv;
        if (r < Cv) {
            RowRef rr = row_ref(p, b, h, s0 + r);
            size_t krow = p.dp ? (rr.tok * p.nh + rr.m) : rr.tok;
            float ssq = 0.f, ssk = 0.f;
            for (int j = lane; j < dk; j += 32) {
                float xq = rr.has_q ? load_in(q, rr.tok * dk + j) : 0.f;
                float xk = load_in(k, krow * dk + j);
                qr[j] = xq;
                kr[j] = xk;
                ssq += xq * xq;
                ssk += xk * xk;
            }
            ssq = warp_sum(ssq);
            ssk = warp_sum(ssk);
            const float iq = rsqrtf(ssq + kNormEps);
            const float ik = rsqrtf(ssk + kNormEps);
            float bscal = 0.f, ascal = 0.f;
            if (p.dp) {
                bscal = p.beta[rr.tok * p.nh + rr.m];
                ascal = rr.m == 0 ? logf(p.alpha[rr.tok]) : 0.f;
            } else {
                if (p.beta_scalar) bscal = p.beta[rr.tok];
                if (p.alpha_scalar) ascal = logf(p.alpha[rr.tok]);
            }
            const bool bs = p.dp || p.beta_scalar;
            const bool as = p.dp || p.alpha_scalar;
            for (int j = lane; j < dk; j += 32) {
                float bj = gdn2 ? 1.f : (bs ? bscal : p.beta[rr.tok * dk + j]);
                qr[j] *= iq;
                kr[j] *= ik * sqrtf(bj);
                gr[j] = as ? ascal : logf(p.alpha[rr.tok * dk + j]);
            }
            if (gdn2) {
                // GDN2 (Su Jianlin's GDN2 stability note, in the d_k x d_v convention): write
                // vector k^, erase vector j' = eta k^ (.) b after the token-wise transform,
                // values eta v.  kr already holds k^ (beta is not used).
                const float eta = p.gdn2_eta[rr.tok];
                float* er = ew + (size_t)r * dk;
                float cdot = 0.f, nj2 = 0.f, amax = 0.f;
                for (int j = lane; j < dk; j += 32) {
                    kr[j] = load_in(k, krow * dk + j) * ik;
                    const float jp = eta * kr[j] * p.gdn2_b[rr.tok * dk + j];
                    er[j] = jp;
                    cdot += jp * kr[j];
                    nj2 += jp * jp;
                    amax = fmaxf(amax, p.alpha_scalar ? p.alpha[rr.tok] : p.alpha[rr.tok * dk + j]);
                }
                cdot = warp_sum(cdot);
                nj2 = warp_sum(nj2);
                amax = warp_max(amax);
                if (p.gdn2_mode == 1) {          // D -> min(D, 1/rho), rho = ||I - j' k^T||_2
                    const float rho = 0.5f * (sqrtf(nj2) + sqrtf(fmaxf(nj2 - 4.f * cdot + 4.f, 0.f)));
                    const float lr = -logf(rho);
                    for (int j = lane; j < dk; j += 32) gr[j] = fminf(gr[j], lr);
                } else if (p.gdn2_mode == 2) {   // j* = c k + lambda* (j' - c k)
                    const float tau = (cdot - 1.f) * amax + 1.f / amax;
                    const float den = nj2 - cdot * cdot;
                    const float lam = den > 0.f ? fminf(1.f, sqrtf(fmaxf(tau * tau - cdot * cdot, 0.f) / den)) : 1.f;
                    for (int j = lane; j < dk; j += 32) er[j] = cdot * kr[j] + lam * (er[j] - cdot * kr[j]);
                }
                for (int j = lane; j < dv; j += 32) vr[j] = load_in(v, krow * dv + j) * eta;
            } else {
                for (int j = lane; j < dv; j += 32) {
                    float bj;
                    if (p.beta_v) bj = bs ? p.beta_v[rr.tok] : p.beta_v[rr.tok * dv + j];
                    else bj = bs ? bscal : p.beta[rr.tok * dk + j];   // channel-wise beta needs dk == dv
                    vr[j] = load_in(v, krow * dv + j) * sqrtf(bj);
                }
            }
        } else {
            if (gdn2) for (int j = lane; j < dk; j += 32) ew[(size_t)r * dk + j] = 0.f;
            for (int j = lane; j < dk; j += 32) { qr[j] = 0.f; kr[j] = 0.f; gr[j] = 0.f; }
            for (int j = lane; j < dv; j += 32) vr[j] = 0.f;
        }
    }
    __syncthreads();

    // 2. cumulative log-decay inside the chunk, per channel.
    for (int j = tid; j < dk; j += kSimtThreads) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += g[(size_t)r * dk + j];
            g[(size_t)r * dk + j] = acc;
        }
    }
    __syncthreads();

    // 3. A (i < r) and P (i <= r) with the decay formed element by element.  Warp w takes rows
    // 16 m + w and 16 m + 15 - w (the same number of pairs for every warp); its lanes run over
    // channels and hold the partial sums of 16 A and 16 P entries at a time, which one butterfly
    // of 31 shuffles reduces (lane l ends with entry l; the same pairing as a warp sum per entry).
    {
        const unsigned full = 0xffffffffu;
        constexpr int kJ = 4;                // channels per lane (d <= 128)
        for (int k = 0; k < C / 8; ++k) {
            const int r = 16 * (k >> 1) + ((k & 1) ? 15 - warp : warp);
            float er_[kJ], qr_[kJ], gr_[kJ];
#pragma unroll
            for (int u = 0; u < kJ; ++u) {
                const int j = lane + 32 * u;
                if (j < dk) {
                    er_[u] = ew[(size_t)r * dk + j];
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
                                    const float e = expf(gr_[u] - g[(size_t)i * dk + j]);
                                    const float ke = kt[(size_t)i * dk + j] * e;
                                    v[16 + t] += qr_[u] * ke;
                                    v[t] += er_[u] * ke;
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

    // 4. T = (I + A)^{-1} by forward substitution, one column per thread in registers:
    //    T[r][j] = delta_rj - sum_{j <= i < r} A[r][i] T[i][j].
    {
        constexpr int kMaxC = kC ? kC : 64;  // rows (the chunk; at most 64)
        const int j = tid;
        if (j < C) {
            float t[kMaxC];
#pragma unroll
            for (int r = 0; r < kMaxC; ++r) {
                if (r < C) {
                    float acc = (j == r) ? 1.f : 0.f;
                    if (j < r) {
#pragma unroll
                        for (int i = 0; i < r; ++i)
                            if (i >= j) acc -= A[(size_t)r * C + i] * t[i];
                    }
                    t[r] = acc;
                }
            }
#pragma unroll
            for (int r = 0; r < kMaxC; ++r)
                if (r < C) Tm[(size_t)r * C + j] = t[r];
        }
    }
    __syncthreads();

    // 5. chunk-end decay, K', and the e^g-scaled operands.
    InterF32 L{C, dk, dv};
    float* outp = static_cast<float*>(p.inter) + ((size_t)bh * p.NC + c) * L.floats();
    for (int j = tid; j < dk; j += kSimtThreads) outp[L.gC() + j] = expf(g[(size_t)(C - 1) * dk + j]);
    for (int idx = tid; idx < C * dk; idx += kSimtThreads) {
        const int r = idx / dk, j = idx % dk;
        const float gl = g[(size_t)(C - 1) * dk + j];
        const float gr = g[idx];
        outp[L.Kp() + idx] = kt[idx] * expf(gl - gr);
        const float eg = expf(gr);
        ew[idx] *= eg;            // the state read: k~ e^g (tied) or j' e^g (GDN2)
        qh[idx] *= eg;
        (void)r;
    }
    __syncthreads();

    // 6. W = T (K~ e^g) into g's buffer; U' = T V~.
    float* W = g;
    for (int idx = tid; idx < C * dk; idx += kSimtThreads) {
        const int r = idx / dk, j = idx % dk;
        float acc = 0.f;
        for (int i = 0; i <= r; ++i) acc += Tm[(size_t)r * C + i] * ew[(size_t)i * dk + j];
        W[idx] = acc;
        outp[L.W() + idx] = acc;
    }
    for (int idx = tid; idx < C * dv; idx += kSimtThreads) {
        const int r = idx / dv, j = idx % dv;
        float acc = 0.f;
        for (int i = 0; i <= r; ++i) acc += Tm[(size_t)r * C + i] * vt[(size_t)i * dv + j];
        Up[idx] = acc;
        outp[L.Up() + idx] = acc;
    }
    __syncthreads();

    // 7. Qe = Q^ e^g - P W;  PU' = P U'.
    for (int idx = tid; idx < C * dk; idx += kSimtThreads) {
        const int r = idx / dk, j = idx % dk;
        float acc = qh[idx];
        for (int i = 0; i <= r; ++i) acc -= P[(size_t)r * C + i] * W[(size_t)i * dk + j];
        outp[L.Qe() + idx] = acc;
    }
    for (int idx = tid; idx < C * dv; idx += kSimtThreads) {
        const int r = idx / dv, j = idx % dv;
        float acc = 0.f;
        for (int i = 0; i <= r; ++i) acc += P[(size_t)r * C + i] * Up[(size_t)i * dv + j];
        outp[L.PUp() + idx] = acc;
    }
}

// Shared memory of the scan kernel: S (dk x NS), U and the U', PU' slices (C x NS each),
// W, Qe, K' (C x dk each), e^{g_C} (dk).
__host__ __device__ inline size_t scan_simt_smem(int C, int dk, int ns = kScanCols) {
    return sizeof(float) * ((size_t)dk * ns + (size_t)3 * C * ns + (size_t)3 * C * dk + dk);
}

// 16-byte asynchronous copy of n floats (n % 4 == 0, both sides 16-byte aligned), spread
// over the CTA's threads.
__device__ __forceinline__ void cp_async_floats(float* dst, const float* src, int n, int tid) {
    for (int i = 4 * tid; i < n; i += 4 * kSimtThreads)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((unsigned)__cvta_generic_to_shared(dst + i)),
                     "l"(src + i) : "memory");
}
// Rows of a column slice: rows x NSC floats from a row-major source of row stride ld.
template <int NSC>
__device__ __forceinline__ void cp_async_slice(float* dst, const float* src, int rows, int ld, int tid) {
    for (int i = tid; i < rows * (NSC / 4); i += kSimtThreads) {
        const int r = i / (NSC / 4), q4 = i % (NSC / 4);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                     ::"r"((unsigned)__cvta_generic_to_shared(dst + r * NSC + 4 * q4)),
                     "l"(src + (size_t)r * ld + 4 * q4) : "memory");
    }
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// One CTA per (d_v slice of NSC columns, head); serial over chunks.  The chunk
// quantities are fetched one phase ahead with asynchronous copies: W, Qe, U', PU' (used
// only by the U / output phase) for chunk c+1 while the state update of chunk c runs, and
// K', e^{g_C} (used only by the state update) for chunk c+1 while the U phase of c+1 runs.
// Every iteration commits both groups (possibly empty), so "all but the newest group have
// landed" always names the one needed next.
template <typename Tout, int NR, int NI, int NSC = kScanCols>
__global__ void __launch_bounds__(kSimtThreads)
scan_simt_kernel(Problem p) {
    constexpr int NS = NSC;                         // columns of this CTA
    constexpr int kRG = kSimtThreads / NSC;         // threads per column
    const int j0 = blockIdx.x * NS;
    const int bh = blockIdx.y;
    // the launcher picks NR = C / kRG and NI = dk / kRG (C and dk are multiples of it), so both
    // sizes are compile-time here and the loops over them unroll
    constexpr int C = kRG * NR, dk = kRG * NI;
    if (!GDN_IN_BOUNDS(j0 + NS <= p.dv && bh < p.B * p.H && p.C == C && p.dk == dk, p.status)) return;
    const int b = bh / p.H, h = bh % p.H;
    const int dv = p.dv;
    const int tid = threadIdx.x;

    extern __shared__ __align__(16) float sm[];
    float* S = sm;                        // dk x NS
    float* U = S + (size_t)dk * NS;       // C x NS
    float* Upc = U + (size_t)C * NS;      // C x NS: U' slice
    float* PUc = Upc + (size_t)C * NS;    // C x NS: PU' slice
    float* Wc = PUc + (size_t)C * NS;     // C x dk
    float* Qc = Wc + (size_t)C * dk;      // C x dk
    float* Kc = Qc + (size_t)C * dk;      // C x dk
    float* gc = Kc + (size_t)C * dk;      // dk

    InterF32 L{C, dk, dv};
    const float* inter = static_cast<const float*>(p.inter);
    auto block = [&](int c) { return inter + ((size_t)bh * p.NC + c) * L.floats(); };
    auto fetch_uo = [&](int c) {          // group: what the U / output phase reads
        if (c < p.NC) {
            const float* in = block(c);
            cp_async_floats(Wc, in + L.W(), C * dk, tid);
            cp_async_floats(Qc, in + L.Qe(), C * dk, tid);
            cp_async_slice<NS>(Upc, in + L.Up() + j0, C, dv, tid);
            cp_async_slice<NS>(PUc, in + L.PUp() + j0, C, dv, tid);
        }
        cp_async_commit_group();
    };
    auto fetch_s = [&](int c) {           // group: what the state update reads
        if (c < p.NC) {
            const float* in = block(c);
            cp_async_floats(Kc, in + L.Kp(), C * dk, tid);
            cp_async_floats(gc, in + L.gC(), dk, tid);
        }
        cp_async_commit_group();
    };

    for (int idx = tid; idx < dk * NS; idx += kSimtThreads) {
        const int i = idx / NS, j = idx % NS;
        S[idx] = p.S0 ? p.S0[((size_t)bh * dk + i) * dv + j0 + j] : 0.f;
    }
    fetch_uo(0);
    fetch_s(0);
    Tout* out = static_cast<Tout*>(p.out);
    for (int c = 0; c < p.NC; ++c) {
        cp_async_wait_one();              // W, Qe, U', PU' of chunk c
        __syncthreads();                  // ... for every thread; S of chunk c is complete
        if (p.S_chunks) {
            float* dst = p.S_chunks + ((size_t)bh * p.NC + c) * dk * dv;
            for (int idx = tid; idx < dk * NS; idx += kSimtThreads) {
                const int i = idx / NS, j = idx % NS;
                dst[(size_t)i * dv + j0 + j] = S[idx];
            }
        }
        const int s0 = c * C;
        {   // thread: column j, rows rg, rg + 8, ...; each S[i][j] is read once for all its rows
            const int j = tid % NS, rg = tid / NS;
            float ws[NR], qs[NR];
#pragma unroll
            for (int m = 0; m < NR; ++m) { ws[m] = 0.f; qs[m] = 0.f; }
            if (out) {
                for (int i = 0; i < dk; ++i) {
                    const float sij = S[(size_t)i * NS + j];
#pragma unroll
                    for (int m = 0; m < NR; ++m) {
                        const int r = rg + kRG * m;
                        ws[m] += Wc[(size_t)r * dk + i] * sij;
                        qs[m] += Qc[(size_t)r * dk + i] * sij;
                    }
                }
            } else {                      // state recompute only: no outputs
                for (int i = 0; i < dk; i += 4) {   // W rows as float4 along i
                    const float s0 = S[(size_t)i * NS + j], s1 = S[(size_t)(i + 1) * NS + j];
                    const float s2 = S[(size_t)(i + 2) * NS + j], s3 = S[(size_t)(i + 3) * NS + j];
#pragma unroll
                    for (int m = 0; m < NR; ++m) {
                        const float4 w = *reinterpret_cast<const float4*>(Wc + (size_t)(rg + kRG * m) * dk + i);
                        ws[m] = fmaf(w.w, s3, fmaf(w.z, s2, fmaf(w.y, s1, fmaf(w.x, s0, ws[m]))));
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                {
                    const int r = rg + kRG * m;
                    const int idx = r * NS + j;
                    U[idx] = Upc[idx] - ws[m];
                    const int s = s0 + r;
                    if (out && s < p.L) {
                        RowRef rr = row_ref(p, b, h, s);
                        if (rr.has_q) store_out(out, rr.tok * dv + j0 + j, PUc[idx] + qs[m]);
                    }
                }
            }
        }
        __syncthreads();                  // W, Qe, U', PU' buffers are free; U is complete
        fetch_uo(c + 1);
        cp_async_wait_one();              // K', e^{g_C} of chunk c
        __syncthreads();
        {   // thread: column j, state rows i0 .. i0 + NI - 1 (contiguous: K' rows load as
            // float4); each U[r][j] is read once
            const int j = tid % NS, i0 = (tid / NS) * NI;
            float acc[NI];
#pragma unroll
            for (int m = 0; m < NI; ++m) acc[m] = gc[i0 + m] * S[(size_t)(i0 + m) * NS + j];
            for (int r = 0; r < C; ++r) {
                const float u = U[(size_t)r * NS + j];
                const float4* kv = reinterpret_cast<const float4*>(Kc + (size_t)r * dk + i0);
#pragma unroll
                for (int m4 = 0; m4 < NI / 4; ++m4) {
                    const float4 kk = kv[m4];
                    acc[4 * m4 + 0] += kk.x * u;
                    acc[4 * m4 + 1] += kk.y * u;
                    acc[4 * m4 + 2] += kk.z * u;
                    acc[4 * m4 + 3] += kk.w * u;
                }
            }
#pragma unroll
            for (int m = 0; m < NI; ++m) S[(size_t)(i0 + m) * NS + j] = acc[m];
        }
        __syncthreads();                  // K', e^{g_C} buffers are free
        fetch_s(c + 1);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (p.S_final) {
        for (int idx = tid; idx < dk * NS; idx += kSimtThreads) {
            const int i = idx / NS, j = idx % NS;
            p.S_final[((size_t)bh * dk + i) * dv + j0 + j] = S[idx];
        }
    }
}

size_t simt_inter_bytes(const Problem& p) {
    InterF32 L{p.C, p.dk, p.dv};
    return (size_t)p.B * p.H * p.NC * L.floats() * sizeof(float);
}

size_t simt_intra_smem_bytes(int C, int dk, int dv, bool gdn2) { return intra_simt_smem(C, dk, dv, gdn2); }

bool simt_supported(int C, int dk, int dv) {
    return intra_simt_smem(C, dk, dv) <= 227 * 1024 && scan_simt_smem(C, dk) <= 227 * 1024 &&
           dv % kScanCols == 0;
}

template <typename Tout, int NR, int NI, int NSC = kScanCols>
cudaError_t launch_scan_nr_ni(const Problem& p, dim3 grid, size_t smem, cudaStream_t stream) {
    auto kern = scan_simt_kernel<Tout, NR, NI, NSC>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kSimtThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <typename Tout, int NR>
cudaError_t launch_scan_nr(const Problem& p, dim3 grid, size_t smem, cudaStream_t stream) {
    switch (p.dk / kRowGroups) {
        case 4: return launch_scan_nr_ni<Tout, NR, 4>(p, grid, smem, stream);
        case 8: return launch_scan_nr_ni<Tout, NR, 8>(p, grid, smem, stream);
        case 16: return launch_scan_nr_ni<Tout, NR, 16>(p, grid, smem, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename Tout>
cudaError_t launch_scan_t(const Problem& p, dim3 grid, size_t smem, cudaStream_t stream) {
    switch (p.C / kRowGroups) {
        case 2: return launch_scan_nr<Tout, 2>(p, grid, smem, stream);
        case 4: return launch_scan_nr<Tout, 4>(p, grid, smem, stream);
        case 8: return launch_scan_nr<Tout, 8>(p, grid, smem, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin, int kC = 0, int kDK = 0, int kDV = 0>
cudaError_t launch_intra_k(const Problem& p, size_t smem, cudaStream_t stream) {
    auto kern = intra_simt_kernel<Tin, kC, kDK, kDV>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(p.NC, p.B * p.H), kSimtThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_intra_t(const Problem& p, size_t smem, cudaStream_t stream) {
    if (p.dk == 128 && p.dv == 128) {        // d = 128: the sizes as constants
        if (p.C == 16) return launch_intra_k<Tin, 16, 128, 128>(p, smem, stream);
        if (p.C == 32) return launch_intra_k<Tin, 32, 128, 128>(p, smem, stream);
    }
    return launch_intra_k<Tin>(p, smem, stream);
}

cudaError_t launch_simt_intra(const Problem& p, bool bf16, cudaStream_t stream) {
    const size_t s1 = intra_simt_smem(p.C, p.dk, p.dv, p.gdn2_eta != nullptr);
    if (p.NC > 0)
        return bf16 ? launch_intra_t<__nv_bfloat16>(p, s1, stream) : launch_intra_t<float>(p, s1, stream);
    return cudaSuccess;
}

// d_k = 128: slices of 16 columns (16 threads per column), twice the CTAs of 32-column slices
// for the same serial chain, each step with half the work
template <typename Tout>
cudaError_t launch_scan16(const Problem& p, cudaStream_t stream) {
    constexpr int W = 16, RG = kSimtThreads / W;
    const size_t smem = scan_simt_smem(p.C, p.dk, W);
    const dim3 grid(p.dv / W, p.B * p.H);
    switch (p.C / RG) {
        case 1: return launch_scan_nr_ni<Tout, 1, 128 / RG, W>(p, grid, smem, stream);
        case 2: return launch_scan_nr_ni<Tout, 2, 128 / RG, W>(p, grid, smem, stream);
        case 4: return launch_scan_nr_ni<Tout, 4, 128 / RG, W>(p, grid, smem, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_simt_scan(const Problem& p, bool bf16, cudaStream_t stream) {
    if (p.dk == 128 && p.dv % 16 == 0)
        return bf16 ? launch_scan16<__nv_bfloat16>(p, stream) : launch_scan16<float>(p, stream);
    const size_t s2 = scan_simt_smem(p.C, p.dk);
    dim3 g2(p.dv / kScanCols, p.B * p.H);
    return bf16 ? launch_scan_t<__nv_bfloat16>(p, g2, s2, stream) : launch_scan_t<float>(p, g2, s2, stream);
}

cudaError_t launch_simt(const Problem& p, bool bf16, cudaStream_t stream) {
    cudaError_t e = launch_simt_intra(p, bf16, stream);
    return e != cudaSuccess ? e : launch_simt_scan(p, bf16, stream);
}

}  // namespace gdn
