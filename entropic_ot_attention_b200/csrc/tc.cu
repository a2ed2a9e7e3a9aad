// Tensor-core (tcgen05 + TMA) band sweeps for sm_100a.
#include "kernels.cuh"

namespace eot {

bool tc_supported(const Geom&) { return false; }
cudaError_t launch_tc_lse(const LsePass&, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_tc_bwd(const BwdPass&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace eot
