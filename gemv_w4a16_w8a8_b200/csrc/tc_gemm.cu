// tcgen05 tensor-core GEMM family (large M). Not built yet: no configuration reaches it.
#include "common.cuh"

namespace qg {

bool tc_supports(const Problem &, const qgemm_config_t &) { return false; }

cudaError_t launch_tc(const Problem &, const qgemm_config_t &, unsigned int *, cudaStream_t)
{
    return cudaErrorNotSupported;
}

} // namespace qg
