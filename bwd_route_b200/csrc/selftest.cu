// selftest.cu -- exercises the bounded-wait failure path of the pipeline
// kernels on the GPU: one thread waits on an mbarrier that nothing will ever
// arrive on, with a short limit, using the same wait routine as the tcgen05
// kernels. The wait gives up, records MOE_FLAG_WAIT_TIMEOUT in the workspace
// flag word and the kernel returns normally, so the context stays usable.
#include <cstdint>

#include "common.cuh"
#include "internal.h"
#include "moe_top1.h"

namespace moe {
namespace {

__global__ void wait_timeout_kernel(uint32_t* dev_flags, long long limit_cycles) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival; none is ever made
        abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, &abort, dev_flags, limit_cycles);
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_top1_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                                       int64_t limit_cycles, void* stream) {
    if (!workspace) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return MOE_ERR_MISALIGNED;
    if (workspace_bytes < 256) return MOE_ERR_WORKSPACE;
    if (limit_cycles < 1 || limit_cycles > moe::kWaitLimitCycles) return MOE_ERR_INVALID_ARG;
    moe::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(workspace),
                                                                              limit_cycles);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
