// Tensor-core (tcgen05) path of the bf16 layer.  Filled in after the SIMT path is green.
#include "gdn_internal.cuh"

namespace gdn {

bool tc_supported(const Problem &) { return false; }
size_t tc_workspace_bytes(const Problem &, bool) { return 0; }
cudaError_t launch_tc_fwd(const Params &, const Problem &, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_tc_bwd(const Params &, const Problem &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn
