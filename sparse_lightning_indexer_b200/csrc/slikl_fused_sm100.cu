// Fused per-token kernel on the sm_100a tensor cores (tcgen05 + TMEM). Not yet written:
// every shape goes to the CUDA-core kernel for now.
#include "slikl_common.cuh"

namespace slikl {

cudaError_t launch_fused_sm100(const Params &P, int workers, cudaStream_t s, bool *handled) {
    (void)P; (void)workers; (void)s;
    *handled = false;
    return cudaSuccess;
}

}  // namespace slikl
