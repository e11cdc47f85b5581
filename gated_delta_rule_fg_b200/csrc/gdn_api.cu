// gdn_api.cu -- the C ABI declared in include/gdn.h: argument validation,
// workspace sizing and kernel dispatch.  Every step of the computation runs in
// the CUDA kernels of this library; there is no host or CPU fallback.
#include <cstdlib>

#include "gdn.h"
#include "gdn_common.cuh"
#include "gdn_nvtx.h"

namespace gdn {
// gdn_simt.cu
size_t simt_inter_bytes(const Problem& p);
bool simt_supported(int C, int dk, int dv);
size_t simt_intra_smem_bytes(int C, int dk, int dv, bool gdn2);
cudaError_t launch_simt(const Problem& p, bool bf16, cudaStream_t stream);
// gdn_tc.cu
bool tc_supported(const Problem& p, bool bf16);
size_t tc_inter_bytes(const Problem& p);
cudaError_t launch_tc(const Problem& p, cudaStream_t stream);
int tc_launches(const Problem& p);
// gdn_decode.cu
cudaError_t launch_decode(const Problem& p, bool bf16, cudaStream_t stream);
// gdn_bwd.cu
bool bwd_supported(int C, int dk, int dv);
size_t bwd_inter_bytes(const Problem& p, size_t fwd_inter);
int bwd_launches(const Problem& p);
cudaError_t launch_bwd(Problem p, const void* dO, const float* dS_final, float* dq, float* dk,
                       float* dv, float* dalpha, float* dbeta, float* dbeta_v, float* dS0,
                       size_t fwd_inter, bool bf16, cudaStream_t stream);
}  // namespace gdn

using namespace gdn;

namespace {

constexpr size_t kHeaderBytes = 256;     // status word + reserved, keeps the rest 256-aligned

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

// Fills `p` (without pointers) and checks sizes.  Returns GDN_OK or the error.
gdn_status_t make_problem(Problem& p, int B, int H, int T, int nh, int dk, int dv, int chunk,
                          gdn_dtype_t dtype, unsigned flags, bool dp, bool plus = false) {
    if (B < 0 || H < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (flags & ~(unsigned)(GDN_ALPHA_SCALAR | GDN_BETA_SCALAR | GDN_SINGLE_STREAM)) return GDN_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return GDN_ERR_UNSUPPORTED;
    // chunk 128 is evaluated as 64-row chunks: the chunk length changes only the order of the
    // rounding, not what is computed, and the kernels tile at most 64 rows
    if (chunk == 128) chunk = 64;
    if (dp && (nh < 1 || nh > 4)) return GDN_ERR_UNSUPPORTED;
    const bool beta_scalar = dp || (flags & GDN_BETA_SCALAR);
    if (!beta_scalar && !plus && dk != dv) return GDN_ERR_INVALID_ARG;   // sqrt(beta) scales v too
    if (!simt_supported(chunk, dk, dv)) return GDN_ERR_UNSUPPORTED;
    p = Problem{};
    p.B = B; p.H = H; p.T = T;
    p.nh = dp ? nh : 1;
    p.L = T * p.nh;
    p.dk = dk; p.dv = dv; p.C = chunk;
    p.NC = (p.L + chunk - 1) / chunk;
    p.alpha_scalar = dp ? 1 : ((flags & GDN_ALPHA_SCALAR) ? 1 : 0);
    p.beta_scalar = beta_scalar ? 1 : 0;
    p.dp = dp ? 1 : 0;
    p.single_stream = (flags & GDN_SINGLE_STREAM) ? 1 : 0;
    p.test_skip_chunk = -1;
    if (const char* e = std::getenv("GDN_TEST_SCAN_SKIP_CHUNK")) {
        char* end = nullptr;
        const long c = std::strtol(e, &end, 10);
        if (end != e && c >= 0 && c < (1L << 30)) {
            p.test_skip_chunk = (int)c;
            p.test_wait_ns = 1000000ull;        // 1 ms
        }
    }
    return GDN_OK;
}

size_t workspace_bytes_for(const Problem& p, bool bf16) {
    size_t inter = tc_supported(p, bf16) ? tc_inter_bytes(p) : simt_inter_bytes(p);
    return kHeaderBytes + inter;
}

// Pointer checks shared by the forward entry points (NULL token tensors, 16-byte alignment).
gdn_status_t check_pointers(const Problem& p) {
    const bool has_tokens = p.B > 0 && p.H > 0 && p.T > 0;
    if (has_tokens && (!p.q || !p.k || !p.v || !p.alpha || !p.beta || !p.out)) return GDN_ERR_INVALID_ARG;
    if (!aligned16(p.q) || !aligned16(p.k) || !aligned16(p.v) || !aligned16(p.alpha) ||
        !aligned16(p.beta) || !aligned16(p.beta_v) || !aligned16(p.out) || !aligned16(p.S0) ||
        !aligned16(p.S_final))
        return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status_t run(Problem& p, bool bf16, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream) {
    const gdn_status_t pst = check_pointers(p);
    if (pst != GDN_OK) return pst;
    const size_t need = workspace_bytes_for(p, bf16);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return GDN_ERR_WORKSPACE;
    p.status = static_cast<int*>(workspace);
    p.inter = static_cast<char*>(workspace) + kHeaderBytes;
    if (p.B == 0 || p.H == 0) return GDN_OK;
    cudaError_t e = tc_supported(p, bf16) ? launch_tc(p, stream) : launch_simt(p, bf16, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int launches_for(const Problem& p, bool bf16) {
    if (p.B == 0 || p.H == 0) return 0;
    if (tc_supported(p, bf16)) return tc_launches(p);
    return p.NC > 0 ? 2 : 1;
}

}  // namespace

namespace gdn {
// Every check gdn_chunk_fwd makes before it enqueues work, except the workspace ones.
gdn_status_t chunk_fwd_check_args(const void* q, const void* k, const void* v, const float* alpha,
                                  const float* beta, const float* S0, const void* out,
                                  const float* S_final, int B, int H, int T, int dk, int dv, int chunk,
                                  gdn_dtype_t dtype, unsigned flags) {
    Problem p;
    gdn_status_t st = make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false);
    if (st != GDN_OK) return st;
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta;
    p.S0 = S0; p.out = const_cast<void*>(out); p.S_final = const_cast<float*>(S_final);
    return check_pointers(p);
}
}  // namespace gdn

extern "C" {

int gdn_chunk_fwd_launches(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                           unsigned flags) {
    Problem p;
    if (make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false) != GDN_OK) return -1;
    return launches_for(p, dtype == GDN_BF16);
}

int gdn_chunk_fwd_tensor_cores(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                               unsigned flags) {
    Problem p;
    if (make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false) != GDN_OK) return -1;
    // (T == 0 and empty batches enqueue no chunk work; the answer is the path the sizes select)
    Problem q = p;
    if (q.T == 0) q.T = 1;
    return tc_supported(q, dtype == GDN_BF16) ? 1 : 0;
}

int gdn_deltaproduct_fwd_launches(int B, int H, int T, int n_h, int dk, int dv, int chunk,
                                  gdn_dtype_t dtype) {
    Problem p;
    if (make_problem(p, B, H, T, n_h, dk, dv, chunk, dtype, 0u, true) != GDN_OK) return -1;
    return launches_for(p, dtype == GDN_BF16);
}

size_t gdn_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                    gdn_dtype_t dtype, unsigned flags) {
    Problem p;
    if (make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false) != GDN_OK) return 0;
    return workspace_bytes_for(p, dtype == GDN_BF16);
}

gdn_status_t gdn_chunk_fwd(const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta,
                           const float* S0, void* out, float* S_final,
                           int B, int H, int T, int dk, int dv, int chunk,
                           gdn_dtype_t dtype, unsigned flags,
                           void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    NvtxRange nvtx_range("gdn_chunk_fwd");
    Problem p;
    gdn_status_t st = make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false);
    if (st != GDN_OK) return st;
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta;
    p.S0 = S0; p.out = out; p.S_final = S_final;
    return run(p, dtype == GDN_BF16, workspace, workspace_bytes, stream);
}

int gdn_plus_chunk_fwd_launches(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                                unsigned flags) {
    Problem p;
    if (make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, true) != GDN_OK) return -1;
    return launches_for(p, dtype == GDN_BF16);
}

size_t gdn_plus_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                         gdn_dtype_t dtype, unsigned flags) {
    Problem p;
    if (make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, true) != GDN_OK) return 0;
    return workspace_bytes_for(p, dtype == GDN_BF16);
}

gdn_status_t gdn_plus_chunk_fwd(const void* q, const void* k, const void* v,
                                const float* alpha, const float* beta_k, const float* beta_v,
                                const float* S0, void* out, float* S_final,
                                int B, int H, int T, int dk, int dv, int chunk,
                                gdn_dtype_t dtype, unsigned flags,
                                void* workspace, size_t workspace_bytes,
                                cudaStream_t stream) {
    NvtxRange nvtx_range("gdn_plus_chunk_fwd");
    Problem p;
    gdn_status_t st = make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, true);
    if (st != GDN_OK) return st;
    if (B > 0 && H > 0 && T > 0 && !beta_v) return GDN_ERR_INVALID_ARG;
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta_k; p.beta_v = beta_v;
    p.S0 = S0; p.out = out; p.S_final = S_final;
    return run(p, dtype == GDN_BF16, workspace, workspace_bytes, stream);
}

size_t gdn_deltaproduct_fwd_workspace_size(int B, int H, int T, int n_h, int dk, int dv,
                                           int chunk, gdn_dtype_t dtype) {
    Problem p;
    if (make_problem(p, B, H, T, n_h, dk, dv, chunk, dtype, 0u, true) != GDN_OK) return 0;
    return workspace_bytes_for(p, dtype == GDN_BF16);
}

gdn_status_t gdn_deltaproduct_fwd(const void* q, const void* k, const void* v,
                                  const float* gamma, const float* beta,
                                  const float* S0, void* out, float* S_final,
                                  int B, int H, int T, int n_h, int dk, int dv, int chunk,
                                  gdn_dtype_t dtype,
                                  void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream) {
    NvtxRange nvtx_range("gdn_deltaproduct_fwd");
    Problem p;
    gdn_status_t st = make_problem(p, B, H, T, n_h, dk, dv, chunk, dtype, 0u, true);
    if (st != GDN_OK) return st;
    p.q = q; p.k = k; p.v = v; p.alpha = gamma; p.beta = beta;
    p.S0 = S0; p.out = out; p.S_final = S_final;
    return run(p, dtype == GDN_BF16, workspace, workspace_bytes, stream);
}

size_t gdn2_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                     gdn_dtype_t dtype, unsigned flags) {
    Problem p;
    if (flags & ~(unsigned)(GDN_ALPHA_SCALAR | GDN_SINGLE_STREAM)) return 0;
    if (make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, true) != GDN_OK) return 0;
    if (tc_supported(p, dtype == GDN_BF16)) return kHeaderBytes + tc_inter_bytes(p);
    if (simt_intra_smem_bytes(chunk, dk, dv, true) > 227 * 1024) return 0;
    return kHeaderBytes + simt_inter_bytes(p);
}

int gdn2_chunk_fwd_launches(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                            unsigned flags) {
    if (gdn2_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype, flags) == 0) return -1;
    if (B == 0 || H == 0) return 0;
    Problem p;
    make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, true);
    if (tc_supported(p, dtype == GDN_BF16)) return tc_launches(p);
    return T > 0 ? 2 : 1;
}

gdn_status_t gdn2_chunk_fwd(const void* q, const void* k, const void* v, const float* alpha,
                            const float* eta, const float* b_gate, const float* S0, void* out,
                            float* S_final, int B, int H, int T, int dk, int dv, int chunk,
                            gdn_dtype_t dtype, unsigned flags, int mode,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    NvtxRange nvtx_range("gdn2_chunk_fwd");
    Problem p;
    if (flags & ~(unsigned)(GDN_ALPHA_SCALAR | GDN_SINGLE_STREAM)) return GDN_ERR_INVALID_ARG;
    if (mode < 0 || mode > 2) return GDN_ERR_INVALID_ARG;
    gdn_status_t st = make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, true);
    if (st != GDN_OK) return st;
    const bool tc = tc_supported(p, dtype == GDN_BF16);
    if (!tc && simt_intra_smem_bytes(chunk, dk, dv, true) > 227 * 1024) return GDN_ERR_UNSUPPORTED;
    const bool has_tokens = B > 0 && H > 0 && T > 0;
    if (has_tokens && (!q || !k || !v || !alpha || !eta || !b_gate || !out)) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, alpha, eta, b_gate, S0, out, S_final};
    for (const void* x : ptrs)
        if (!aligned16(x)) return GDN_ERR_INVALID_ARG;
    const size_t need = kHeaderBytes + (tc ? tc_inter_bytes(p) : simt_inter_bytes(p));
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return GDN_ERR_WORKSPACE;
    if (B == 0 || H == 0) return GDN_OK;
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = nullptr;
    p.S0 = S0; p.out = out; p.S_final = S_final;
    p.gdn2_eta = eta ? eta : alpha;      // non-null marks GDN2 (eta is only read for T > 0)
    p.gdn2_b = b_gate;
    p.gdn2_mode = mode;
    p.status = static_cast<int*>(workspace);
    p.inter = static_cast<char*>(workspace) + kHeaderBytes;
    const cudaError_t e = tc ? launch_tc(p, stream) : launch_simt(p, dtype == GDN_BF16, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t gdn_chunk_bwd_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                    gdn_dtype_t dtype, unsigned flags) {
    Problem p;
    if (make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, true) != GDN_OK) return 0;
    if (!bwd_supported(chunk, dk, dv)) return 0;
    return kHeaderBytes + bwd_inter_bytes(p, simt_inter_bytes(p));
}

int gdn_chunk_bwd_launches(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                           unsigned flags) {
    Problem p;
    if (make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, true) != GDN_OK) return -1;
    if (!bwd_supported(chunk, dk, dv)) return -1;
    return (B == 0 || H == 0) ? 0 : bwd_launches(p);
}

gdn_status_t gdn_chunk_bwd(const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta_k, const float* beta_v,
                           const float* S0, const void* dout, const float* dS_final,
                           float* dq, float* dk_, float* dv_, float* dalpha, float* dbeta_k,
                           float* dbeta_v, float* dS0,
                           int B, int H, int T, int dk, int dv, int chunk,
                           gdn_dtype_t dtype, unsigned flags,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    NvtxRange nvtx_range("gdn_chunk_bwd");
    Problem p;
    gdn_status_t st = make_problem(p, B, H, T, 1, dk, dv, chunk, dtype, flags, false, beta_v != nullptr);
    if (st != GDN_OK) return st;
    if (!bwd_supported(chunk, dk, dv)) return GDN_ERR_UNSUPPORTED;
    if (dbeta_v && !beta_v) return GDN_ERR_INVALID_ARG;
    const bool has_tokens = B > 0 && H > 0 && T > 0;
    if (has_tokens && (!q || !k || !v || !alpha || !beta_k || !dout)) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, alpha, beta_k, beta_v, S0, dout, dS_final, dq, dk_, dv_,
                          dalpha, dbeta_k, dbeta_v, dS0};
    for (const void* x : ptrs)
        if (!aligned16(x)) return GDN_ERR_INVALID_ARG;
    const size_t fwd = simt_inter_bytes(p);
    const size_t need = kHeaderBytes + bwd_inter_bytes(p, fwd);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return GDN_ERR_WORKSPACE;
    if (B == 0 || H == 0) return GDN_OK;
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta_k; p.beta_v = beta_v; p.S0 = S0;
    p.status = static_cast<int*>(workspace);
    p.inter = static_cast<char*>(workspace) + kHeaderBytes;
    cudaError_t e = launch_bwd(p, dout, dS_final, dq, dk_, dv_, dalpha, dbeta_k, dbeta_v, dS0, fwd,
                               dtype == GDN_BF16, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_recurrent_step(const void* q, const void* k, const void* v,
                                const float* alpha, const float* beta_k, const float* beta_v,
                                const float* S_in, float* S_out, void* out,
                                int B, int H, int dk, int dv, gdn_dtype_t dtype, unsigned flags,
                                cudaStream_t stream) {
    NvtxRange nvtx_range("gdn_recurrent_step");
    if (B < 0 || H < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (flags & ~(unsigned)(GDN_ALPHA_SCALAR | GDN_BETA_SCALAR)) return GDN_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    const bool beta_scalar = (flags & GDN_BETA_SCALAR) != 0;
    if (!beta_scalar && !beta_v && dk != dv) return GDN_ERR_INVALID_ARG;
    if ((size_t)B * H * (dv / 32) > 0x7fffffffull) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return GDN_OK;
    if (!q || !k || !v || !alpha || !beta_k || !S_out || !out) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(beta_k) ||
        !aligned16(beta_v) || !aligned16(S_in) || !aligned16(S_out) || !aligned16(out))
        return GDN_ERR_INVALID_ARG;
    if (S_in && S_in != S_out) {     // in place is allowed; a partial overlap is not
        const size_t n = (size_t)B * H * dk * dv;
        if (S_in < S_out + n && S_out < S_in + n) return GDN_ERR_INVALID_ARG;
    }
    Problem p{};
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta_k; p.beta_v = beta_v;
    p.S0 = S_in; p.S_final = S_out; p.out = out;
    p.B = B; p.H = H; p.T = 1; p.nh = 1; p.L = 1;
    p.dk = dk; p.dv = dv; p.C = 1; p.NC = 1;
    p.alpha_scalar = (flags & GDN_ALPHA_SCALAR) ? 1 : 0;
    p.beta_scalar = beta_scalar ? 1 : 0;
    return launch_decode(p, dtype == GDN_BF16, stream) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_workspace_status(void* workspace, cudaStream_t stream) {
    NvtxRange nvtx_range("gdn_workspace_status");
    if (!workspace) return GDN_ERR_WORKSPACE;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GDN_ERR_CUDA;
    if (word != 0 && cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    switch (word) {
        case 0: return GDN_OK;
        case kDevTimeout: return GDN_ERR_TIMEOUT;
        case kDevRange: return GDN_ERR_RANGE;
        case kDevBounds: return GDN_ERR_BOUNDS;
        default: return GDN_ERR_CUDA;
    }
}

const char* gdn_status_string(gdn_status_t s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported size";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_TIMEOUT: return "device wait timed out";
        case GDN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case GDN_ERR_RANGE: return "value outside the fp16 operand range";
        case GDN_ERR_BOUNDS: return "index outside its buffer (bounds-checking build)";
    }
    return "unknown status";
}

int gdn_version(void) { return 100; }

}  // extern "C"
