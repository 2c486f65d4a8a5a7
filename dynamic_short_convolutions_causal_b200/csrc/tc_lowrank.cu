// Tensor-core (tcgen05) low-rank kernels: placeholder until the sm_100a kernels land.
#include "internal.h"

namespace dsc {

bool tc_lowrank_supported(int, int, int, int, int, int, bool) { return false; }

cudaError_t launch_tc_lowrank_fwd(const void *, const void *, const void *, void *, int, int, int,
                                  int, int, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

size_t tc_lowrank_bwd_workspace(int, int, int, int, int, int) { return 0; }

cudaError_t launch_tc_lowrank_bwd(const void *, const void *, const void *, const void *, void *,
                                  float *, float *, void *, int, int, int, int, int, int,
                                  cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace dsc
