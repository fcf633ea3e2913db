// Tensor-core (tcgen05 / TMEM / TMA) chunk kernel.
#include "gdn_internal.cuh"

namespace gdn {

bool tc_supports(const FwdParams &p, const char **why) {
    (void)p;
    *why = "tensor-core kernel not available in this build";
    return false;
}

int tc_default_slices(const FwdParams &p) { return p.dv >= 128 ? 2 : 1; }

cudaError_t launch_tc(const FwdParams &p, cudaStream_t stream, const char **why) {
    (void)p; (void)stream;
    *why = "tensor-core kernel not available in this build";
    return cudaErrorNotSupported;
}

}  // namespace gdn
