// Prefill projection on the sm_100a tensor cores (tcgen05 / TMEM / TMA).
#include "cmp_internal.cuh"

namespace cmp {

bool proj_tc_supported(const Params&) { return false; }

cudaError_t launch_proj_tc(const Params&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace cmp
