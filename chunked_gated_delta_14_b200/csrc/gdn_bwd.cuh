// Host-side declarations of the backward pass (gdn_bwd.cu).
#pragma once

#include <cuda_runtime.h>

#include "gdn_bwd_params.cuh"

namespace gdn {

// Shapes the backward kernels take: chunk 16, 32 or 64; dk 16..128 (a power of
// two); dv a multiple of 32, at most 128.
bool bwd_supports(const BwdParams &p, const char **why);
// Workspace bytes for p (regions 256-byte aligned).
size_t bwd_workspace_bytes(const BwdParams &p);
// Points the ws_* fields of p into `workspace`.
void bwd_carve_workspace(BwdParams &p, void *workspace);
// Enqueues the four launches (five with either truncated series) on `stream`.
cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream);

}  // namespace gdn
