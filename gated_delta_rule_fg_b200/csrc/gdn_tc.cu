// gdn_tc.cu -- tensor-core (tcgen05) kernels; filled in by the sm_100a path.
#include "gdn_common.cuh"

namespace gdn {
bool tc_supported(const Problem&, bool) { return false; }
size_t tc_inter_bytes(const Problem&) { return 0; }
cudaError_t launch_tc(const Problem&, cudaStream_t) { return cudaErrorNotSupported; }
int tc_launches(const Problem&) { return 0; }
}  // namespace gdn
