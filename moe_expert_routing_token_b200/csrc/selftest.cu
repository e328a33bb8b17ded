// Self-check of the library's bounded waits: every barrier wait in the
// kernels gives up after a time budget (on %globaltimer) instead of hanging,
// records the failure and lets the kernel return.  This kernel waits on an
// mbarrier that nothing completes, with a caller-given budget, and reports
// whether the wait ran out - the failure path exercised without a fault.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_routing.h"
#include "sm100_ptx.cuh"

namespace moe {

int set_error(int status, const char* msg);
int set_cuda_error(cudaError_t err, const char* what);

namespace {

__global__ void bounded_wait_kernel(uint64_t budget_ns, int32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = ptx::globaltimer_ns();
        const bool completed = ptx::mbar_wait(&bar, 0, budget_ns);  // nobody arrives
        const uint64_t waited = ptx::globaltimer_ns() - t0;
        status[0] = completed ? 0 : 1;
        status[1] = (int32_t)(waited / 1000);  // microseconds spent waiting
    }
}

}  // namespace
}  // namespace moe

extern "C" int moe_selftest_bounded_wait(uint64_t budget_ns, int32_t* status, void* stream) {
    if (!status) return moe::set_error(MOE_ERR_INVALID_ARG, "moe_selftest_bounded_wait: null status");
    if (budget_ns == 0 || budget_ns > 1000000000ull)
        return moe::set_error(MOE_ERR_INVALID_ARG, "moe_selftest_bounded_wait: budget outside (0, 1 s]");
    moe::bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(budget_ns, status);
    const cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? MOE_OK : moe::set_cuda_error(err, "moe_selftest_bounded_wait: launch");
}
