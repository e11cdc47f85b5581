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
//     first call on each device before any stream capture.
//   - Every call shares the array and it keeps the last call's contents; the
//     status word at its start is cleared on each call.  Calls whose kernels can
//     overlap on the GPU (other streams, other threads) race on the array.
#include <mutex>

#include "gdn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

gdn_status_t scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return GDN_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return GDN_OK;
}

}  // namespace

extern "C" gdn_status_t gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                              const float* alpha, const float* beta,
                                              const float* S0, void* out, float* S_final,
                                              int B, int H, int T, int dk, int dv, int chunk,
                                              gdn_dtype_t dtype, unsigned flags,
                                              cudaStream_t stream) {
    const size_t need = gdn_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype, flags);
    if (need == 0)      // invalid or unsupported sizes: let the regular entry point name the error
        return gdn_chunk_fwd(q, k, v, alpha, beta, S0, out, S_final, B, H, T, dk, dv, chunk, dtype,
                             flags, nullptr, 0, stream);
    if (need > kNoAllocScratchBytes) return GDN_ERR_WORKSPACE;
    void* scratch = nullptr;
    const gdn_status_t st = scratch_for_current_device(&scratch);
    if (st != GDN_OK) return st;
    if (cudaMemsetAsync(scratch, 0, sizeof(int), stream) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_chunk_fwd(q, k, v, alpha, beta, S0, out, S_final, B, H, T, dk, dv, chunk, dtype, flags,
                         scratch, kNoAllocScratchBytes, stream);
}
