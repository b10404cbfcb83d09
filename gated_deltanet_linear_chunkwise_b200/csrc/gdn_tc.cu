// gdn_tc.cu -- tensor-core path (not yet enabled: every problem runs on the
// CUDA-core kernels).
#include "gdn_tc.h"

namespace gdn {

bool tc_supports(const Problem &) { return false; }
size_t tc_workspace_bytes(const Problem &) { return 0; }
cudaError_t launch_tc(const Problem &, void *, cudaStream_t, cudaEvent_t *) { return cudaErrorNotSupported; }

}  // namespace gdn
