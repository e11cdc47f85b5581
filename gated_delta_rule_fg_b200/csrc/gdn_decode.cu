// gdn_decode.cu -- one recurrent step of FG^2-GDN per head (single-token decode).
//
// For each (batch b, head h) with state S (dk x dv, float32) and one new token:
//     q^ = q / ||q||,  k^ = k / ||k||              (||x|| = sqrt(sum x^2 + 1e-6))
//     k~ = sqrt(beta^k) (.) k^,  v~ = sqrt(beta^v) (.) v   (beta^v = beta without FG^2-GDN+)
//     S' = (I - k~ k~^T) Diag(alpha) S + k~ v~^T,  o = S'^T q^
// (FG^2-GDN reading notes, sec. 2.2 eq. (11), one token; eq. (13) for the split rates).
//
// Columns of S are independent: with X = Diag(alpha) S and u_j = v~_j - k~^T X[:, j],
//     S'[:, j] = X[:, j] + k~ u_j,     o_j = (alpha (.) q^)^T S[:, j] + (q^ . k~) u_j,
// so one CTA takes a 32-column slice of one head's state, reads it once into registers,
// forms both column dot products in the same pass, and writes S' and o.  The step moves
// 2 * dk * dv * 4 bytes of state per head and is bound by HBM bandwidth.
#include "gdn.h"
#include "gdn_common.cuh"

namespace gdn {
namespace dec {

constexpr int NT = 128;          // threads per CTA
constexpr int kCols = 32;        // state columns per CTA
constexpr int kG = kCols / 4;    // float4 column groups per row
constexpr int kR = NT / kG;      // row groups (16)

template <typename Tin, int DK>
__global__ void __launch_bounds__(NT) step_kernel(Problem p) {
    constexpr int RPT = DK / kR;             // rows per thread
    __shared__ float s_qa[DK], s_ka[DK], s_kt[DK], s_al[DK];
    __shared__ float s_red[3][NT / 32];
    __shared__ float s_pa[kR][kCols], s_pc[kR][kCols];
    __shared__ float s_u[kCols];

    const int slices = p.dv / kCols;
    const int bh = blockIdx.x / slices;
    const int col0 = (blockIdx.x % slices) * kCols;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int dk = DK, dv = p.dv;
    const Tin* q = static_cast<const Tin*>(p.q) + (size_t)bh * dk;
    const Tin* k = static_cast<const Tin*>(p.k) + (size_t)bh * dk;

    // the state slice first: its loads do not depend on the token prep, so they are in
    // flight while the prep's loads and reductions run
    const int rg = tid / kG, cg = tid % kG;
    const int c = col0 + 4 * cg;
    float4 s[RPT];
    const size_t sbase = (size_t)bh * dk * dv;
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg + kR * m;
        s[m] = p.S0 ? *reinterpret_cast<const float4*>(p.S0 + sbase + (size_t)i * dv + c)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // token prep: norms of q and k, and q^ . k~ (needs sqrt(beta^k) per channel)
    float xq = 0.f, xk = 0.f, a = 1.f, sb = 0.f;
    if (tid < DK) {
        xq = load_in(q, tid);
        xk = load_in(k, tid);
        a = p.alpha_scalar ? p.alpha[bh] : p.alpha[(size_t)bh * dk + tid];
        sb = sqrtf(p.beta_scalar ? p.beta[bh] : p.beta[(size_t)bh * dk + tid]);
    }
    float ssq = warp_sum(xq * xq), ssk = warp_sum(xk * xk), sqk = warp_sum(xq * xk * sb);
    if (lane == 0) {
        s_red[0][warp] = ssq;
        s_red[1][warp] = ssk;
        s_red[2][warp] = sqk;
    }
    __syncthreads();
    ssq = ssk = sqk = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        ssq += s_red[0][w];
        ssk += s_red[1][w];
        sqk += s_red[2][w];
    }
    const float iq = rsqrtf(ssq + kNormEps), ik = rsqrtf(ssk + kNormEps);
    const float qk = sqk * iq * ik;          // q^ . k~
    if (tid < DK) {
        const float kt = xk * ik * sb;
        s_qa[tid] = xq * iq * a;
        s_ka[tid] = kt * a;
        s_kt[tid] = kt;
        s_al[tid] = a;
    }
    __syncthreads();

    // one pass over the slice: X^T k~ and (alpha (.) q^)^T S per column
    float pa[4] = {0.f, 0.f, 0.f, 0.f}, pc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg + kR * m;
        const float ka = s_ka[i], qa = s_qa[i];
        pa[0] += ka * s[m].x; pa[1] += ka * s[m].y; pa[2] += ka * s[m].z; pa[3] += ka * s[m].w;
        pc[0] += qa * s[m].x; pc[1] += qa * s[m].y; pc[2] += qa * s[m].z; pc[3] += qa * s[m].w;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        s_pa[rg][4 * cg + e] = pa[e];
        s_pc[rg][4 * cg + e] = pc[e];
    }
    __syncthreads();
    if (tid < kCols) {
        float d = 0.f, o = 0.f;
#pragma unroll
        for (int r = 0; r < kR; ++r) {
            d += s_pa[r][tid];
            o += s_pc[r][tid];
        }
        const int j = col0 + tid;
        const float* bv = p.beta_v ? p.beta_v : p.beta;     // without beta_v: beta (dk == dv)
        const float rate = p.beta_scalar ? bv[bh] : bv[(size_t)bh * (p.beta_v ? dv : dk) + j];
        const float vt = load_in(static_cast<const Tin*>(p.v), (size_t)bh * dv + j) * sqrtf(rate);
        const float u = vt - d;
        s_u[tid] = u;
        store_out(static_cast<Tin*>(p.out), (size_t)bh * dv + j, o + qk * u);
    }
    __syncthreads();

    // S'[i, j] = alpha_i S[i, j] + k~_i u_j
    const float u0 = s_u[4 * cg], u1 = s_u[4 * cg + 1], u2 = s_u[4 * cg + 2], u3 = s_u[4 * cg + 3];
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg + kR * m;
        const float al = s_al[i];
        const float kt = s_kt[i];
        float4 r;
        r.x = al * s[m].x + kt * u0;
        r.y = al * s[m].y + kt * u1;
        r.z = al * s[m].z + kt * u2;
        r.w = al * s[m].w + kt * u3;
        *reinterpret_cast<float4*>(p.S_final + sbase + (size_t)i * dv + c) = r;
    }
}

template <typename Tin>
cudaError_t launch_t(const Problem& p, cudaStream_t stream) {
    const unsigned grid = (unsigned)((size_t)p.B * p.H * (p.dv / kCols));
    switch (p.dk) {
        case 32: step_kernel<Tin, 32><<<grid, NT, 0, stream>>>(p); break;
        case 64: step_kernel<Tin, 64><<<grid, NT, 0, stream>>>(p); break;
        case 128: step_kernel<Tin, 128><<<grid, NT, 0, stream>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace dec

// p.T is unused (one token); p.S0 is the state read (may be null: zero state),
// p.S_final the state written (may equal p.S0).
cudaError_t launch_decode(const Problem& p, bool bf16, cudaStream_t stream) {
    return bf16 ? dec::launch_t<__nv_bfloat16>(p, stream) : dec::launch_t<float>(p, stream);
}

}  // namespace gdn
