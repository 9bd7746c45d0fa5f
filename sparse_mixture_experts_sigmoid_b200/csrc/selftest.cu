// Self-test of the device failure path: a kernel whose mbarrier wait can never
// complete, run through the same bounded wait (wait_bar) that every producer,
// MMA issuer and epilogue of the tensor-core kernels uses.  When the limit
// runs out the wait raises the library's device flag (MOE_ERR_DEVICE_TIMEOUT
// through moe_device_status) and the kernel returns, leaving the context
// usable.  No GPU fault or hang is involved: the wait is bounded by
// %globaltimer.
#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_probe_kernel(uint32_t *err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);   // one arrival expected; nothing ever arrives
        abort_flag = 0;
        tc::fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        volatile int *abort = &abort_flag;
        tc::wait_bar(&bar, 0, abort, err, limit_ns);   // runs out, raises kErrTimeout
    }
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_selftest_wait_timeout(uint32_t limit_ms, void *stream) {
    if (limit_ms < 1 || limit_ms > 10000) return MOE_ERR_INVALID_ARG;
    uint32_t *err = moe::device_error_word();
    if (!err) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = moe::launch_kernel(moe::wait_timeout_probe_kernel, 1, 32, 0, s, err,
                                             (uint64_t)limit_ms * 1000000ull);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
