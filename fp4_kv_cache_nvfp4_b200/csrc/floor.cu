// Launch-chain floor: a chain of empty dependent kernels with programmatic
// dependent launch, the same launch configuration the decode step uses.  It
// measures the cost of the kernel boundaries alone, so the step time of the
// real chain can be read against it.  No counterpart on the pages.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

__global__ void empty_chain_kernel(int32_t* sink) {
    pdl_wait();
    pdl_trigger();
    if (sink && blockIdx.x == 0 && threadIdx.x == 0) *sink += 1;  // one dependent write per link
}

}  // namespace csa2

extern "C" CSA2_API csa2_status csa2_test_empty_chain(int32_t n_kernels, int32_t ctas, int32_t threads,
                                                      int32_t* sink, void* stream) {
    using namespace csa2;
    if (n_kernels < 0 || ctas < 1 || ctas > 65535 || threads < 32 || threads > 1024 || (threads & 31))
        return CSA2_ERR_INVALID_ARG;
    if (sink && (reinterpret_cast<uintptr_t>(sink) & 3u)) return CSA2_ERR_INVALID_ARG;
    for (int i = 0; i < n_kernels; ++i) {
        LaunchCfg c(dim3((unsigned)ctas), dim3((unsigned)threads), 0, (cudaStream_t)stream);
        if (cudaLaunchKernelEx(&c.cfg, empty_chain_kernel, sink) != cudaSuccess) {
            (void)cudaGetLastError();
            return CSA2_ERR_CUDA;
        }
    }
    return CSA2_OK;
}
