// gdn_streams.cu -- the per-device side stream that parts of a call fork onto.
#include "gdn_common.cuh"

namespace gdn {
namespace {

constexpr int kMaxDev = 64;

struct Slot {
    bool tried = false, ok = false;
    SideStream ss{};
};
Slot g_slots[kMaxDev];
std::mutex g_mu;

bool create(SideStream& ss) {
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return false;
    if (cudaStreamCreateWithPriority(&ss.stream, cudaStreamNonBlocking, hi) != cudaSuccess) return false;
    bool ok = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < kSideEvents && ok; ++i)
        ok = cudaEventCreateWithFlags(&ss.ready[i], cudaEventDisableTiming) == cudaSuccess;
    return ok;
}

}  // namespace

SideStream* side_stream_lock(std::unique_lock<std::mutex>& lock) {
    lock = std::unique_lock<std::mutex>(g_mu);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
    Slot& s = g_slots[dev];
    if (!s.tried) {
        s.tried = true;
        s.ok = create(s.ss);
    }
    return s.ok ? &s.ss : nullptr;
}

}  // namespace gdn
