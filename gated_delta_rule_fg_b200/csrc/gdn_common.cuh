// gdn_common.cuh -- problem description and helpers shared by the kernels of
// libgdn_b200.so.
//
// The chunkwise evaluation of the FG^2-GDN recurrence (reading notes of
// "FG^2-GDN: Enhancing Long-Context Gated Delta Networks with Doubly
// Fine-Grained Control", sec. 2.2 eq. (11) and sec. 2.4) is split in two roles:
//
//   intra role (independent per chunk): load a chunk of C rows, L2-normalise
//     q and k, scale k and v by sqrt(beta) (FG^2-GDN+, sec. 2.3 eq. (13): k by
//     sqrt(beta^k) and v by sqrt(beta^v)), take the cumulative log-decay
//     g_r = sum_{s<=r} log alpha_s per channel, and build
//       A   = strictly-lower (K~ e^g)(K~ e^-g)^T    P = lower (Q^ e^g)(K~ e^-g)^T
//       T   = (I + A)^{-1}                          (UT transform)
//       W   = T (K~ (.) e^g)        U'  = T V~
//       Qe  = Q^ (.) e^g - P W      PU' = P U'
//       K'  = K~ (.) e^{g_C - g}    gC  = e^{g_C}
//   scan role (serial over chunks, per head and d_v slice), with S the state
//     at the chunk start:
//       U = U' - W S;   O = Qe S + PU';   S <- Diag(gC) S + K'^T U
//
// The scan-role formulas follow from eq. (11): with X_r = Diag(alpha_r) S_{r-1}
// and u_r = v~_r - X_r^T k~_r, (I + A) U = V~ - (K~ (.) e^g) S, the outputs are
// O = (Q^ (.) e^g) S + P U and the next state is Diag(e^{g_C}) S + K'^T U;
// substituting U = U' - W S into O gives O = Qe S + PU'.
#pragma once
#include <mutex>

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gdn {

// Device-side error codes recorded in the workspace header (match gdn_status_t).
enum : int { kDevOk = 0, kDevTimeout = 4, kDevRange = 6, kDevBounds = 7 };

// Bounds checks of the bounds-checking build (-DGDN_DEBUG_BOUNDS): GDN_IN_BOUNDS(cond, status)
// is false, and GDN_ERR_BOUNDS is recorded in the workspace status word, when `cond` does not
// hold; the caller then skips the access.  In the normal build it is the constant true.
#ifdef GDN_DEBUG_BOUNDS
__device__ __forceinline__ bool bounds_ok(bool cond, int* status) {
    if (!cond) atomicCAS(status, (int)kDevOk, (int)kDevBounds);
    return cond;
}
#define GDN_IN_BOUNDS(cond, status) (::gdn::bounds_ok((cond), (status)))
#else
#define GDN_IN_BOUNDS(cond, status) true
#endif

struct Problem {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;     // GDN: alpha; DeltaProduct: gamma (scalar per token)
    const float* beta;      // key rate beta^k (and value rate, unless beta_v is set)
    const float* beta_v;    // FG^2-GDN+ value rate beta^v (eq. (13)); null: beta scales v too
    const float* S0;        // may be null
    void* out;
    float* S_final;         // may be null
    int B, H, T;            // T = tokens
    int nh;                 // sub-steps per token (1 for GDN, n_h for DeltaProduct)
    int L;                  // sub-steps per sequence = T * nh
    int dk, dv, C;          // head dims and chunk length (in sub-steps)
    int NC;                 // chunks per sequence = ceil(L / C)
    int alpha_scalar, beta_scalar;
    int dp;                 // 1: DeltaProduct row mapping
    int single_stream;      // 1: all work on the caller's stream (no side-stream fork)
    // Failure-detection test knob (environment variable GDN_TEST_SCAN_SKIP_CHUNK, read per
    // call; unset in normal use): the tensor-core scan's producer leaves chunk test_skip_chunk
    // unloaded, so the roles that wait for it run out of their bound, which is then
    // test_wait_ns instead of the 2 s default.  -1 / 0: off.
    int test_skip_chunk;
    unsigned long long test_wait_ns;
    int* status;            // workspace header word
    void* inter;            // per-chunk intermediates written by the intra role
    float* S_chunks;        // backward recompute: state at every chunk start,
                            // [B,H,NC,dk,dv]; null in the forward
    // GDN2 (non-tied erase / write, float32 path only): eta [B,T,H] and b [B,T,H,dk]; the
    // erase vector is j' = eta k^ (.) b after the token-wise transform gdn2_mode
    // (0 none, 1 clip D to min(D, 1/rho), 2 shrink j' toward KDA); null eta: not GDN2.
    const float* gdn2_eta;
    const float* gdn2_b;
    int gdn2_mode;
};

// Row source of sub-step s of head (b, h) (DeltaProduct interleaves n_h
// sub-steps per token; the decay gamma_t sits on the first one and the output
// is read at the last one).
struct RowRef {
    size_t tok;        // (b*T + t)*H + h
    int m;             // sub-step within the token
    bool has_q;        // this row produces an output
};

__device__ __forceinline__ RowRef row_ref(const Problem& p, int b, int h, int s) {
    RowRef r;
    int t = s / p.nh;
    r.m = s - t * p.nh;
    r.tok = ((size_t)b * p.T + t) * p.H + h;
    r.has_q = (r.m == p.nh - 1);
    return r;
}

__device__ __forceinline__ float load_in(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_in(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void store_out(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, size_t i, float x) { p[i] = __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

constexpr float kNormEps = 1e-6f;   // ||x|| = sqrt(sum x^2 + eps)

// Layout of the float32 intermediates of one (head, chunk) in the workspace.
struct InterF32 {
    int C, dk, dv;
    __host__ __device__ size_t floats() const { return (size_t)C * (3 * dk + 2 * dv) + dk; }
    __host__ __device__ size_t W() const { return 0; }
    __host__ __device__ size_t Qe() const { return (size_t)C * dk; }
    __host__ __device__ size_t Kp() const { return 2 * (size_t)C * dk; }
    __host__ __device__ size_t Up() const { return 3 * (size_t)C * dk; }
    __host__ __device__ size_t PUp() const { return 3 * (size_t)C * dk + (size_t)C * dv; }
    __host__ __device__ size_t gC() const { return 3 * (size_t)C * dk + 2 * (size_t)C * dv; }
};

// Per device: one high-priority stream and a few events, created on first use, onto which a
// call forks part of its work (fork / join through events on the caller's stream).
constexpr int kSideEvents = 8;
struct SideStream {
    cudaStream_t stream;
    cudaEvent_t fork, join, ready[kSideEvents];
};
// Takes the side-stream lock (held by `lock` for the caller's whole enqueue sequence) and
// returns the current device's side stream, or null if it cannot be created.
SideStream* side_stream_lock(std::unique_lock<std::mutex>& lock);

}  // namespace gdn
