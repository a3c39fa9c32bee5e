// Small-T projection that streams the weights at HBM bandwidth.
#include "cmp_internal.cuh"

namespace cmp {

bool proj_decode_supported(const Params&) { return false; }
size_t proj_decode_workspace(const Params&) { return 0; }
cudaError_t launch_proj_decode(const Params&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace cmp
