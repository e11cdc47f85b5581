// gdn_noalloc.cu -- gdn_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers can't call cudaMalloc (or any allocating routine): code that runs
// inside another framework's memory pool or allocator hooks, embedded runtimes
// whose device memory is fixed at start-up, or code that must not allocate while
// a stream is being captured.  They still own their inputs and outputs but
// cannot provide the workspace gdn_chunk_fwd needs.  For them this file keeps a
// fixed scratch area in a file-scope __device__ array and passes it to the
// unchanged gdn_chunk_fwd.
//
//   - Size: kNoAllocScratchBytes (64 MiB).  Every GPU on which this library's
//     device code is loaded holds the array until the process exits.
//   - Set-up: the first call on a device looks up the array's device address with
//     that device current (cudaGetSymbolAddress) and caches it; in host code the
//     array's name is only a host-side stand-in, never a device address.  Make the
//     first call on each device before any stream capture.  The cache is keyed on
//     the device's current CUDA context (its context id), so after a
//     cudaDeviceReset the next call looks the address up again instead of using
//     an address of the destroyed context.
//   - Arguments are validated before anything is enqueued: a call rejected with an
//     error has queued no work.
//   - Every call shares the array and it keeps the last call's contents; the
//     status word at its start is cleared on each call, and device-side errors
//     recorded there are not reported back (callers of this entry point have no
//     workspace to pass to gdn_workspace_status).  Calls whose kernels can overlap
//     on the GPU (other streams, other threads) race on the array.
#include <mutex>

#include <cuda.h>

#include "gdn.h"
#include "gdn_nvtx.h"

namespace gdn {
gdn_status_t chunk_fwd_check_args(const void* q, const void* k, const void* v, const float* alpha,
                                  const float* beta, const float* S0, const void* out,
                                  const float* S_final, int B, int H, int T, int dk, int dv, int chunk,
                                  gdn_dtype_t dtype, unsigned flags);
}

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchSlot {
    void* addr = nullptr;
    unsigned long long ctx = 0;      // id of the context the address belongs to (0: unknown)
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the calling thread's current context, or 0 if it cannot be read.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        looked_up = true;
        void* f1 = nullptr;
        void* f2 = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, nullptr) == cudaSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, nullptr) == cudaSuccess) {
            get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
            get_id = reinterpret_cast<CtxGetIdFn>(f2);
        }
    }
    if (!get_current || !get_id) return 0;
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

gdn_status_t scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot& s = g_scratch[dev];
    const unsigned long long ctx = current_context_id();
    if (!s.addr || (ctx != 0 && ctx != s.ctx)) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return GDN_ERR_CUDA;
        s.addr = ptr;
        s.ctx = current_context_id();     // the lookup makes the context current if it was not
    }
    *out = s.addr;
    return GDN_OK;
}

}  // namespace

extern "C" gdn_status_t gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                              const float* alpha, const float* beta,
                                              const float* S0, void* out, float* S_final,
                                              int B, int H, int T, int dk, int dv, int chunk,
                                              gdn_dtype_t dtype, unsigned flags,
                                              cudaStream_t stream) {
    gdn::NvtxRange nvtx_range("gdn_chunk_fwd_noalloc");
    // validation first: nothing is enqueued for a call that is rejected
    const gdn_status_t chk = gdn::chunk_fwd_check_args(q, k, v, alpha, beta, S0, out, S_final, B, H, T,
                                                       dk, dv, chunk, dtype, flags);
    if (chk != GDN_OK) return chk;
    const size_t need = gdn_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype, flags);
    if (need == 0) return GDN_ERR_UNSUPPORTED;
    if (need > kNoAllocScratchBytes) return GDN_ERR_WORKSPACE;
    void* scratch = nullptr;
    const gdn_status_t st = scratch_for_current_device(&scratch);
    if (st != GDN_OK) return st;
    if (cudaMemsetAsync(scratch, 0, sizeof(int), stream) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_chunk_fwd(q, k, v, alpha, beta, S0, out, S_final, B, H, T, dk, dv, chunk, dtype, flags,
                         scratch, kNoAllocScratchBytes, stream);
}
