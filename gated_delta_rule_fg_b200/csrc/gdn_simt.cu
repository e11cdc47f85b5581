// gdn_simt.cu -- float32 CUDA-core kernels for the two roles of the chunkwise
// FG^2-GDN forward (see gdn_common.cuh).  This is the float32 precision path
// (every product in fp32 FMA, decay factors exp(g_r - g_i) formed element by
// element so nothing overflows for any alpha in (0,1]) and the path for shapes
// the tensor-core kernels do not cover.
#include "gdn_common.cuh"

namespace gdn {

constexpr int kSimtThreads = 256;
constexpr int kScanCols = 32;   // d_v columns of the state owned by one scan CTA

// Shared memory of the intra kernel: qh, kt, g (C x dk), vt, Up (C x dv), A, Tm, P (C x C).
__host__ __device__ inline size_t intra_simt_smem(int C, int dk, int dv) {
    return sizeof(float) * ((size_t)3 * C * dk + (size_t)2 * C * dv + (size_t)3 * C * C);
}

// One CTA per (chunk, head).
template <typename Tin>
__global__ void __launch_bounds__(kSimtThreads)
intra_simt_kernel(Problem p) {
    const int c = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int C = p.C, dk = p.dk, dv = p.dv;
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
                float bj = bs ? bscal : p.beta[rr.tok * dk + j];
                qr[j] *= iq;
                kr[j] *= ik * sqrtf(bj);
                gr[j] = as ? ascal : logf(p.alpha[rr.tok * dk + j]);
            }
            for (int j = lane; j < dv; j += 32) {
                float bj;
                if (p.beta_v) bj = bs ? p.beta_v[rr.tok] : p.beta_v[rr.tok * dv + j];
                else bj = bs ? bscal : p.beta[rr.tok * dk + j];   // channel-wise beta needs dk == dv
                vr[j] = load_in(v, krow * dv + j) * sqrtf(bj);
            }
        } else {
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

    // 3. A (i < r) and P (i <= r) with the decay formed element by element.
    for (int pr = warp; pr < C * C; pr += nwarps) {
        const int r = pr / C, i = pr % C;
        float a = 0.f, pp = 0.f;
        if (i <= r) {
            for (int j = lane; j < dk; j += 32) {
                const float e = expf(g[(size_t)r * dk + j] - g[(size_t)i * dk + j]);
                const float ke = kt[(size_t)i * dk + j] * e;
                pp += qh[(size_t)r * dk + j] * ke;
                a += kt[(size_t)r * dk + j] * ke;
            }
            a = warp_sum(a);
            pp = warp_sum(pp);
        }
        if (lane == 0) {
            A[pr] = (i < r) ? a : 0.f;
            P[pr] = pp;
        }
    }
    __syncthreads();

    // 4. T = (I + A)^{-1} by forward substitution, one row at a time:
    //    T[r][j] = delta_rj - sum_{j <= i < r} A[r][i] T[i][j].
    for (int r = 0; r < C; ++r) {
        for (int j = tid; j < C; j += kSimtThreads) {
            float acc = (j == r) ? 1.f : 0.f;
            if (j < r) {
                for (int i = j; i < r; ++i) acc -= A[(size_t)r * C + i] * Tm[(size_t)i * C + j];
            }
            Tm[(size_t)r * C + j] = acc;
        }
        __syncthreads();
    }

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
        kt[idx] *= eg;
        qh[idx] *= eg;
        (void)r;
    }
    __syncthreads();

    // 6. W = T (K~ e^g) into g's buffer; U' = T V~.
    float* W = g;
    for (int idx = tid; idx < C * dk; idx += kSimtThreads) {
        const int r = idx / dk, j = idx % dk;
        float acc = 0.f;
        for (int i = 0; i <= r; ++i) acc += Tm[(size_t)r * C + i] * kt[(size_t)i * dk + j];
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

__host__ __device__ inline size_t scan_simt_smem(int C, int dk) {
    return sizeof(float) * ((size_t)dk * kScanCols + (size_t)C * kScanCols + (size_t)3 * C * dk + dk);
}

// One CTA per (d_v slice of kScanCols columns, head); serial over chunks.
template <typename Tout>
__global__ void __launch_bounds__(kSimtThreads)
scan_simt_kernel(Problem p) {
    const int j0 = blockIdx.x * kScanCols;
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int C = p.C, dk = p.dk, dv = p.dv;
    const int tid = threadIdx.x;
    constexpr int NS = kScanCols;

    extern __shared__ float sm[];
    float* S = sm;                        // dk x NS
    float* U = S + (size_t)dk * NS;       // C x NS
    float* Wc = U + (size_t)C * NS;       // C x dk
    float* Qc = Wc + (size_t)C * dk;      // C x dk
    float* Kc = Qc + (size_t)C * dk;      // C x dk
    float* gc = Kc + (size_t)C * dk;      // dk

    for (int idx = tid; idx < dk * NS; idx += kSimtThreads) {
        const int i = idx / NS, j = idx % NS;
        S[idx] = p.S0 ? p.S0[((size_t)bh * dk + i) * dv + j0 + j] : 0.f;
    }
    InterF32 L{C, dk, dv};
    Tout* out = static_cast<Tout*>(p.out);
    for (int c = 0; c < p.NC; ++c) {
        const float* in = static_cast<const float*>(p.inter) + ((size_t)bh * p.NC + c) * L.floats();
        __syncthreads();   // previous chunk's S update and U reads are done
        if (p.S_chunks) {
            float* dst = p.S_chunks + ((size_t)bh * p.NC + c) * dk * dv;
            for (int idx = tid; idx < dk * NS; idx += kSimtThreads) {
                const int i = idx / NS, j = idx % NS;
                dst[(size_t)i * dv + j0 + j] = S[idx];
            }
        }
        for (int idx = tid; idx < C * dk; idx += kSimtThreads) {
            Wc[idx] = in[L.W() + idx];
            Qc[idx] = in[L.Qe() + idx];
            Kc[idx] = in[L.Kp() + idx];
        }
        for (int i = tid; i < dk; i += kSimtThreads) gc[i] = in[L.gC() + i];
        __syncthreads();
        const int s0 = c * C;
        for (int idx = tid; idx < C * NS; idx += kSimtThreads) {
            const int r = idx / NS, j = idx % NS;
            float ws = 0.f, qs = 0.f;
            for (int i = 0; i < dk; ++i) {
                const float sij = S[(size_t)i * NS + j];
                ws += Wc[(size_t)r * dk + i] * sij;
                qs += Qc[(size_t)r * dk + i] * sij;
            }
            U[idx] = in[L.Up() + (size_t)r * dv + j0 + j] - ws;
            const int s = s0 + r;
            if (out && s < p.L) {     // no outputs in the backward's state recompute
                RowRef rr = row_ref(p, b, h, s);
                if (rr.has_q) store_out(out, rr.tok * dv + j0 + j, in[L.PUp() + (size_t)r * dv + j0 + j] + qs);
            }
        }
        __syncthreads();
        for (int idx = tid; idx < dk * NS; idx += kSimtThreads) {
            const int i = idx / NS, j = idx % NS;
            float acc = gc[i] * S[idx];
            for (int r = 0; r < C; ++r) acc += Kc[(size_t)r * dk + i] * U[(size_t)r * NS + j];
            S[idx] = acc;
        }
    }
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

bool simt_supported(int C, int dk, int dv) {
    return intra_simt_smem(C, dk, dv) <= 227 * 1024 && scan_simt_smem(C, dk) <= 227 * 1024 &&
           dv % kScanCols == 0;
}

cudaError_t launch_simt(const Problem& p, bool bf16, cudaStream_t stream) {
    const size_t s1 = intra_simt_smem(p.C, p.dk, p.dv);
    const size_t s2 = scan_simt_smem(p.C, p.dk);
    if (p.NC > 0) {
        dim3 g1(p.NC, p.B * p.H);
        if (bf16) {
            cudaFuncSetAttribute(intra_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
            intra_simt_kernel<__nv_bfloat16><<<g1, kSimtThreads, s1, stream>>>(p);
        } else {
            cudaFuncSetAttribute(intra_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
            intra_simt_kernel<float><<<g1, kSimtThreads, s1, stream>>>(p);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    dim3 g2(p.dv / kScanCols, p.B * p.H);
    if (bf16) {
        cudaFuncSetAttribute(scan_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
        scan_simt_kernel<__nv_bfloat16><<<g2, kSimtThreads, s2, stream>>>(p);
    } else {
        cudaFuncSetAttribute(scan_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
        scan_simt_kernel<float><<<g2, kSimtThreads, s2, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace gdn
