/*
 * gdn.h -- C ABI of the B200 (sm_100a) FG^2-GDN chunkwise forward library
 *          (libgdn_b200.so).
 *
 * The operation.  For every (batch b, head h) pair the library evaluates the
 * FG^2-GDN recurrence ("FG^2-GDN: Enhancing Long-Context Gated Delta Networks
 * with Doubly Fine-Grained Control", sec. 2 "FG2-GDN Update Rule"; reading
 * notes of the same paper, sec. 2.2, eq. (11)):
 *
 *     q^_t = q_t / ||q_t||,   k^_t = k_t / ||k_t||     (||x|| = sqrt(sum x^2 + 1e-6))
 *     k~_t = sqrt(beta_t) (.) k^_t,   v~_t = sqrt(beta_t) (.) v_t
 *     S_t  = (I - k~_t k~_t^T) Diag(alpha_t) S_{t-1} + k~_t v~_t^T
 *     o_t  = S_t^T q^_t
 *
 * with S in R^{dk x dv}, channel-wise decay alpha_t in (0,1]^{dk} and
 * channel-wise write rate beta_t in [0,1]^{dk}.  KDA (scalar beta), GDN
 * (scalar alpha and beta) and DeltaNet (alpha = 1, scalar beta) are the special
 * cases selected with GDN_ALPHA_SCALAR / GDN_BETA_SCALAR (reading notes, sec. 1
 * table).  It is computed chunkwise: the sequence is cut into chunks of
 * `chunk` tokens, the transitions inside a chunk are accumulated in parallel
 * through the WY/UT representation (cumulative log-decay per chunk, a
 * strictly lower-triangular (I + A)^{-1} solve), and the state is carried from
 * chunk to chunk (reading notes, sec. 2.4).  The result does not depend on
 * `chunk` beyond rounding.
 *
 * Conventions shared by every entry point.
 *   - All tensor arguments are device pointers, row-major and contiguous,
 *     owned by the caller; the library never frees or retains them.
 *   - q, k: [B,T,H,dk]; v, out: [B,T,H,dv]; alpha, beta: [B,T,H,dk], or
 *     [B,T,H] with GDN_ALPHA_SCALAR / GDN_BETA_SCALAR; S0, S_final:
 *     [B,H,dk,dv] float32.
 *   - q, k, v and out share one storage type (gdn_dtype_t).  alpha, beta and
 *     the state are always float32.  Arithmetic is float32 (GDN_F32) or
 *     bf16 inputs with fp16 tensor-core operands and float32 accumulation and
 *     state (GDN_BF16); `out` is rounded to nearest-even on store.
 *   - alpha and beta are post-activation values.  Values outside alpha in
 *     (0,1], beta >= 0, or NaN are not checked (that would cost a pass over
 *     the inputs) and give undefined numbers, not an error.
 *   - S0 == NULL means a zero initial state; S_final == NULL means the final
 *     state is not written.  Feeding S_final back as S0 continues a sequence.
 *   - Every pointer must be 16-byte aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns once it is enqueued.  The caller provides
 *     `workspace` (device memory, 256-byte aligned, at least the size the
 *     matching *_workspace_size function returns); one workspace must not be
 *     used by two calls that can run at the same time.  The library allocates
 *     no device memory.  Unless GDN_SINGLE_STREAM is given, for long sequences
 *     on the tensor-core path it keeps,
 *     per device and created on first use, one high-priority stream and a few
 *     events: a call then forks onto that stream (so part of its work overlaps)
 *     and joins back before returning, so all of its work is still ordered
 *     after earlier and before later work on `stream`, and stream capture
 *     records the fork and the join.  Enqueuing such calls from several host
 *     threads on one device serialises on a lock; capturing one while another
 *     thread enqueues on the same device is not supported.
 *   - Arguments are validated before anything is enqueued; on an error
 *     nothing is enqueued.  Errors found on the device (a bounded wait that
 *     ran out) are recorded in the workspace and read with
 *     gdn_workspace_status().
 *   - The tensor-core path rounds its operands to fp16 (largest finite value
 *     65504).  Normalised q and k and the decay factors are always inside that
 *     range; the value operand sqrt(beta) v, the per-chunk quantities that scale
 *     with v and the fp16 copy of the state are checked, and a call whose values
 *     (or state, for instance from an S0 that large) leave the range, or turn
 *     NaN, records GDN_ERR_RANGE in the workspace status word (read with
 *     gdn_workspace_status): its results are then not valid.  (gdn2_chunk_fwd
 *     checks the state copy only.)  Out-of-range alpha and beta are not detected.
 */
#ifndef GDN_B200_H
#define GDN_B200_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* NULL / misaligned pointer, negative size, dk != dv with channel-wise beta */
    GDN_ERR_UNSUPPORTED = 2,   /* a size the library does not implement (see gdn_chunk_fwd) */
    GDN_ERR_CUDA = 3,          /* a CUDA launch or copy failed (cudaGetLastError is left set) */
    GDN_ERR_TIMEOUT = 4,       /* device side: a bounded wait ran out; outputs are not valid */
    GDN_ERR_WORKSPACE = 5,     /* workspace NULL, misaligned or smaller than required */
    GDN_ERR_RANGE = 6,         /* device side: a value left the fp16 operand range of the tensor-core path */
    GDN_ERR_BOUNDS = 7         /* device side, bounds-checking build only: an index left its buffer
                                  (the access was skipped; outputs are not valid) */
} gdn_status_t;

typedef enum {
    GDN_F32 = 0,               /* q, k, v, out stored as float32 */
    GDN_BF16 = 1               /* q, k, v, out stored as bfloat16 */
} gdn_dtype_t;

enum {
    GDN_ALPHA_SCALAR = 1u,     /* alpha is one value per token and head: [B,T,H] (GDN) */
    GDN_BETA_SCALAR = 2u,      /* beta is one value per token and head: [B,T,H] (KDA, GDN, DeltaNet) */
    GDN_SINGLE_STREAM = 4u     /* keep all of the call's work on `stream`: no fork onto the library's
                                  per-device side stream (no lock, no global state is touched); the
                                  result is the same bit for bit, long sequences take longer */
};

/* Bytes of workspace gdn_chunk_fwd needs for these sizes (0 if the sizes are
 * invalid or unsupported; gdn_chunk_fwd then reports why). */
size_t gdn_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                    gdn_dtype_t dtype, unsigned flags);

/* FG^2-GDN chunkwise forward (eq. (11) above).
 *   q, k [B,T,H,dk], v [B,T,H,dv], out [B,T,H,dv]: dtype storage.
 *   alpha, beta: float32, channel-wise or scalar per `flags`.
 *   S0 (may be NULL), S_final (may be NULL): float32 [B,H,dk,dv].
 * Sizes: B, H, T >= 0 (zero is a no-op that still writes S_final = S0 or 0;
 * with T == 0 the token pointers may be NULL); dk, dv in {32, 64, 128};
 * chunk in {16, 32, 64, 128}; chunk 128 is evaluated as 64-row chunks (the same
 * recurrence, bit for bit the result of chunk 64: the kernels tile at most 64
 * rows).  Channel-wise beta needs dk == dv (sqrt(beta) multiplies v).
 * T need not be a multiple of chunk.  GDN_BF16 with chunk 64 (or 128) and
 * dk == dv == 128 runs on the tensor-core path; other GDN_BF16 shapes and all
 * GDN_F32 shapes run on the float32 CUDA-core path. */
gdn_status_t gdn_chunk_fwd(const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta,
                           const float* S0, void* out, float* S_final,
                           int B, int H, int T, int dk, int dv, int chunk,
                           gdn_dtype_t dtype, unsigned flags,
                           void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* gdn_chunk_fwd for callers that cannot allocate device memory (inside another
 * framework's allocator or memory pool, in runtimes whose device memory is fixed
 * at start-up, or while a stream is being captured): same arguments and result
 * as gdn_chunk_fwd, without the workspace.  The paper has no counterpart; this
 * is a deployment convenience of this library.
 * The scratch is a 64 MiB array inside the library (a file-scope __device__
 * array): every GPU on which the library's device code is loaded holds it until
 * the process exits.  Sizes whose gdn_chunk_fwd_workspace_size exceeds 64 MiB
 * (67108864 bytes) return GDN_ERR_WORKSPACE before anything is enqueued; other
 * argument errors are reported as by gdn_chunk_fwd, also before anything is
 * enqueued.  The first call on a device looks up the array's device address
 * (with that device current) and caches it per device and CUDA context (after a
 * cudaDeviceReset the next call looks it up again); make that first call before
 * any stream capture.  All calls share the array and it keeps the last call's
 * contents (its status word is cleared at the start of each call, device-side
 * errors are not reported back); calls whose work can overlap on the GPU
 * (different streams or threads) race on it. */
gdn_status_t gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta,
                                   const float* S0, void* out, float* S_final,
                                   int B, int H, int T, int dk, int dv, int chunk,
                                   gdn_dtype_t dtype, unsigned flags,
                                   cudaStream_t stream);

/* Bytes of workspace gdn_plus_chunk_fwd needs (0 if invalid/unsupported). */
size_t gdn_plus_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                         gdn_dtype_t dtype, unsigned flags);

/* FG^2-GDN+ chunkwise forward (same paper, "FG2-GDN+ Variant"; reading notes
 * sec. 2.3, eq. (13)).  The write rate is split into a key rate beta^k and a
 * value rate beta^v:
 *     k~_t = sqrt(beta^k_t) (.) k^_t,   v~_t = sqrt(beta^v_t) (.) v_t
 *     S_t  = (I - k~_t k~_t^T) Diag(alpha_t) S_{t-1} + k~_t v~_t^T,   o_t = S_t^T q^_t
 * so the erase acts along beta^k-scaled key directions and the write carries
 * beta^v-scaled values.
 *   beta_k: float32 [B,T,H,dk] ([B,T,H] with GDN_BETA_SCALAR), in [0,1].
 *   beta_v: float32 [B,T,H,dv] ([B,T,H] with GDN_BETA_SCALAR), in [0,1];
 *           GDN_BETA_SCALAR applies to both rates.
 * Everything else (layouts, flags, sizes, workspace, paths, errors) is as for
 * gdn_chunk_fwd, except that channel-wise rates allow dk != dv.  With
 * beta_v == beta_k the result is gdn_chunk_fwd's. */
gdn_status_t gdn_plus_chunk_fwd(const void* q, const void* k, const void* v,
                                const float* alpha, const float* beta_k, const float* beta_v,
                                const float* S0, void* out, float* S_final,
                                int B, int H, int T, int dk, int dv, int chunk,
                                gdn_dtype_t dtype, unsigned flags,
                                void* workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/* Bytes of workspace gdn_deltaproduct_fwd needs (0 if invalid/unsupported). */
size_t gdn_deltaproduct_fwd_workspace_size(int B, int H, int T, int n_h, int dk, int dv,
                                           int chunk, gdn_dtype_t dtype);

/* DeltaProduct n_h forward with a scalar forget gate ("DeltaProduct: Improving
 * State-Tracking in Linear RNNs via Householder Products", "Approach"; the
 * gated variant of its ablation table).  Per token t:
 *     S <- gamma_t S;  for m = 1..n_h:  S <- (I - beta_{t,m} k^_{t,m} k^_{t,m}^T) S
 *                                             + beta_{t,m} k^_{t,m} v_{t,m}^T
 *     o_t = S^T q^_t
 * (gamma is applied once per token, before the first step; k^ and q^ are
 * L2-normalised as above; beta in [0,2] gives eigenvalues in [-1,1]).  It is
 * evaluated as the FG^2-GDN recurrence over the interleaved sequence of n_h*T
 * sub-steps with scalar beta; `chunk` counts sub-steps.
 *   q [B,T,H,dk]; k [B,T,H,n_h,dk]; v [B,T,H,n_h,dv]; gamma [B,T,H];
 *   beta [B,T,H,n_h]; S0, S_final [B,H,dk,dv] float32; out [B,T,H,dv].
 * Sizes as gdn_chunk_fwd, with 1 <= n_h <= 4. */
gdn_status_t gdn_deltaproduct_fwd(const void* q, const void* k, const void* v,
                                  const float* gamma, const float* beta,
                                  const float* S0, void* out, float* S_final,
                                  int B, int H, int T, int n_h, int dk, int dv, int chunk,
                                  gdn_dtype_t dtype,
                                  void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream);

/* Number of kernels one gdn_chunk_fwd / gdn_plus_chunk_fwd / gdn_deltaproduct_fwd
 * call with these sizes enqueues (-1 if the sizes are invalid or unsupported). */
int gdn_chunk_fwd_launches(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                           unsigned flags);
int gdn_plus_chunk_fwd_launches(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                                unsigned flags);
int gdn_deltaproduct_fwd_launches(int B, int H, int T, int n_h, int dk, int dv, int chunk,
                                  gdn_dtype_t dtype);

/* Which path a gdn_chunk_fwd call with these sizes takes: 1 the tensor-core path (tcgen05,
 * fp16 operands, fp32 accumulation), 0 the float32 CUDA-core path (a few tens of times slower
 * at the same size), -1 invalid or unsupported sizes.  The tensor-core path takes GDN_BF16
 * with dk == dv == 128 and chunk 64 (or 128). */
int gdn_chunk_fwd_tensor_cores(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                               unsigned flags);

/* GDN2 transform modes (Su Jianlin's GDN2 stability note): none; clip the decay to
 * min(D, 1/rho) with rho the closed-form spectral norm of I - j' k^T ("Simple
 * Strategy"); or shrink j' toward KDA keeping j'^T k ("Modifying Itself"). */
enum { GDN2_NONE = 0, GDN2_CLIP_DECAY = 1, GDN2_SHRINK_J = 2 };

/* Bytes of workspace gdn2_chunk_fwd needs (0 if invalid/unsupported). */
size_t gdn2_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                     gdn_dtype_t dtype, unsigned flags);

/* GDN2 chunkwise forward: the non-tied update of Su Jianlin's GDN2 stability note
 * ("Problem Description"), written for this library's d_k x d_v state X = S^T:
 *     X_t = (I - k^_t j'_t^T) D_t X_{t-1} + eta_t k^_t v_t^T,    o_t = X_t^T q^_t
 * with q^, k^ L2-normalised as above, j'_t = eta_t k^_t (.) b_t (GDN2's own
 * parameterisation j = k (.) b, b in [0,1]^{dk}, with eta absorbed into j), and D_t =
 * Diag(alpha_t) -- after the token-wise transform `mode` (GDN2_*): GDN2_CLIP_DECAY
 * replaces D by min(D, 1/rho), rho = (||j'|| + sqrt(||j'||^2 - 4 j'^T k^ + 4)) / 2;
 * GDN2_SHRINK_J replaces j' by c k^ + lambda* (j' - c k^), c = j'^T k^,
 * tau = (c - 1) gamma_max + 1/gamma_max (gamma_max = max_i D_ii),
 * lambda* = min(1, sqrt((tau^2 - c^2) / (||j'||^2 - c^2))).  With b = 1 and mode
 * GDN2_NONE this is KDA with write rate eta.  The transforms are fused into the
 * chunk's prep; the chunk form is the non-tied WY form (A pairs erase with write
 * vectors, the state is read along j' and written along k^).
 *   q, k [B,T,H,dk], v, out [B,T,H,dv]: dtype storage; alpha float32 [B,T,H,dk] (or
 *   [B,T,H] with GDN_ALPHA_SCALAR; GDN_SINGLE_STREAM is the only other flag); eta float32 [B,T,H] (>= 0);
 *   b_gate float32 [B,T,H,dk] in [0,1]; S0, S_final float32 [B,H,dk,dv] (may be NULL).
 * GDN_BF16 with chunk 64 and dk == dv == 128 runs on the tensor-core path (fp16
 * operands, as gdn_chunk_fwd); other shapes run on the float32 CUDA-core path with
 * chunk in {16, 32} (64 only where it fits shared memory).  dk, dv in {32, 64, 128}.
 * Workspace and errors as gdn_chunk_fwd. */
gdn_status_t gdn2_chunk_fwd(const void* q, const void* k, const void* v, const float* alpha,
                            const float* eta, const float* b_gate, const float* S0, void* out,
                            float* S_final, int B, int H, int T, int dk, int dv, int chunk,
                            gdn_dtype_t dtype, unsigned flags, int mode,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Number of kernels one gdn2_chunk_fwd call enqueues (-1 if invalid/unsupported). */
int gdn2_chunk_fwd_launches(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                            unsigned flags);

/* Bytes of workspace gdn_chunk_bwd needs (0 if invalid/unsupported). */
size_t gdn_chunk_bwd_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                    gdn_dtype_t dtype, unsigned flags);

/* Chunkwise backward of gdn_chunk_fwd / gdn_plus_chunk_fwd (the training half of
 * the chunkwise algorithm, reading notes sec. 2.4; the forward is eq. (11), or
 * eq. (13) when beta_v != NULL).  Given the forward's inputs and the cotangents
 * dout = dL/dout and dS_final = dL/dS_final, it writes the gradients of L:
 *   dq, dk [B,T,H,dk]; dv [B,T,H,dv]; dalpha and dbeta_k shaped like alpha and
 *   beta_k; dbeta_v shaped like beta_v; dS0 [B,H,dk,dv].  All float32.
 * With beta_v == NULL, dbeta_k is the gradient of the single rate beta (it gets
 * both the key and the value parts) and dbeta_v must be NULL.  Any gradient
 * pointer may be NULL (not written); dS_final == NULL means zero; S0 == NULL
 * means a zero initial state (dS0 is still its gradient).
 *   q, k, v, dout: dtype storage; alpha, beta_k, beta_v, S0, dS_final: float32.
 * The forward is recomputed inside (its chunk quantities and the state at every
 * chunk start are kept in the workspace), in float32 on CUDA cores for both
 * dtypes.  Sizes: as gdn_chunk_fwd, with chunk in {16, 32} (the backward's own
 * chunk; the result does not depend on it beyond rounding).  beta in (0, 1]:
 * the derivative of sqrt(beta) is unbounded at beta = 0.  No device-side waits.
 * Errors as gdn_chunk_fwd. */
gdn_status_t gdn_chunk_bwd(const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta_k, const float* beta_v,
                           const float* S0, const void* dout, const float* dS_final,
                           float* dq, float* dk, float* dv, float* dalpha, float* dbeta_k,
                           float* dbeta_v, float* dS0,
                           int B, int H, int T, int dk_dim, int dv_dim, int chunk,
                           gdn_dtype_t dtype, unsigned flags,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Number of kernels one gdn_chunk_bwd call enqueues (-1 if invalid/unsupported). */
int gdn_chunk_bwd_launches(int B, int H, int T, int dk, int dv, int chunk, gdn_dtype_t dtype,
                           unsigned flags);

/* One recurrent step (single-token decode) for every (b, h): eq. (11) of the
 * reading notes (sec. 2.2) for one token, with the split rates of eq. (13)
 * when beta_v is given:
 *     S_out = (I - k~ k~^T) Diag(alpha) S_in + k~ v~^T,   out = S_out^T q^
 * with q^, k^, k~, v~ as above (v~ = sqrt(beta_v) (.) v, or sqrt(beta_k) (.) v
 * when beta_v == NULL).  This continues a sequence whose state came from
 * gdn_chunk_fwd / gdn_plus_chunk_fwd (their S_final) or from earlier steps.
 *   q, k [B,H,dk]; v, out [B,H,dv]: dtype storage (one token, no T axis).
 *   alpha, beta_k: float32 [B,H,dk] ([B,H] with GDN_ALPHA_SCALAR /
 *   GDN_BETA_SCALAR); beta_v: float32 [B,H,dv] ([B,H] with GDN_BETA_SCALAR) or
 *   NULL (then channel-wise beta_k needs dk == dv).
 *   S_in: float32 [B,H,dk,dv] or NULL (zero state); S_out: float32 [B,H,dk,dv].
 *   S_out may equal S_in (update in place); other overlaps are invalid.
 * Sizes: B, H >= 0 (0 is a no-op); dk, dv in {32, 64, 128}.  Arithmetic is
 * float32 for both dtypes.  No workspace: one kernel, no device-side waits.
 * Errors: GDN_ERR_INVALID_ARG / GDN_ERR_UNSUPPORTED before anything is
 * enqueued, GDN_ERR_CUDA if the launch fails. */
gdn_status_t gdn_recurrent_step(const void* q, const void* k, const void* v,
                                const float* alpha, const float* beta_k, const float* beta_v,
                                const float* S_in, float* S_out, void* out,
                                int B, int H, int dk, int dv, gdn_dtype_t dtype, unsigned flags,
                                cudaStream_t stream);

/* Waits for `stream`, then returns (and clears) the first device-side error
 * recorded in `workspace` by earlier calls: GDN_OK, GDN_ERR_TIMEOUT,
 * GDN_ERR_RANGE or (bounds-checking build) GDN_ERR_BOUNDS; GDN_ERR_CUDA if the
 * wait itself failed.
 *
 * Bounds-checking build: the library compiled with -DGDN_DEBUG_BOUNDS
 * (libgdn_b200_bounds.so; `python -m gated_delta_rule_fg_b200.build
 * --debug-bounds`) checks the global-memory indices its kernels form against
 * the extents of the buffers they address; an index outside records
 * GDN_ERR_BOUNDS and the access is skipped instead of faulting.  Same ABI.
 *
 * Every device-side wait of the library is bounded (2 s); a wait that runs out
 * records GDN_ERR_TIMEOUT and the kernel unwinds (its copies land, its tensor
 * memory is released), leaving the context usable.  Test knob, unset in normal
 * use: with the environment variable GDN_TEST_SCAN_SKIP_CHUNK=<c> set when a
 * forward call is made, the tensor-core scan (bf16, d = 128, chunk 64) leaves
 * chunk c unloaded and bounds its waits by 1 ms, so that call ends with
 * GDN_ERR_TIMEOUT (and invalid outputs). */
gdn_status_t gdn_workspace_status(void* workspace, cudaStream_t stream);

/* Static description of a status code. */
const char* gdn_status_string(gdn_status_t status);

/* Library ABI version (major * 100 + minor). */
int gdn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDN_B200_H */
