// gdn_tc.h -- tensor-core (tcgen05 / TMEM / TMA) path for bf16 inputs.
#pragma once
#include "gdn_internal.h"

namespace gdn {

// Does the tensor-core path take this problem?  (Otherwise the CUDA-core
// path in gdn_simt.cu runs it.)
bool tc_supports(const Problem &p);
// Does the tensor-core path apply the q/k feature maps inside its kernels (frame-wise
// operator), so no separate prologue pass is needed?
bool tc_fuses_qk_prologue(const Problem &p);
size_t tc_workspace_bytes(const Problem &p);
cudaError_t launch_tc(const Problem &p, void *ws, cudaStream_t s, cudaEvent_t *ev);
// Device word in the workspace where a bounded wait that gave up records it.
int *tc_error_word(const Problem &p, void *ws);

}  // namespace gdn
