// Self-test of the device-side failure path: the bounded mbarrier wait used by
// every pipeline in this library, run on a barrier that nothing arrives on.
// The wait gives up at its deadline, the kernel sets MOE_ERR_TIMEOUT in the
// caller's error word and returns, and the CUDA context stays usable.
#include "common.cuh"

namespace moe {

__global__ void wait_timeout_kernel(uint64_t timeout_ns, int32_t* err_flag) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);           // expects one arrival that never comes
        fence_barrier_init();
    }
    __syncthreads();
    const uint64_t deadline = global_ns() + timeout_ns;
    const bool ok = mbar_wait(&bar, 0, deadline);
    if (!ok && threadIdx.x == 0) raise_error(err_flag, MOE_ERR_TIMEOUT);
}

}  // namespace moe

extern "C" moe_status moe_selftest_wait_timeout(int64_t timeout_ns, int32_t* err_flag,
                                                void* stream) {
    if (timeout_ns <= 0 || timeout_ns > 10000000000ll || !err_flag) return MOE_ERR_INVALID_ARG;
    moe::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(timeout_ns), err_flag);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
