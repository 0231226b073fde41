// selftest.cu -- moe_selftest_wait_timeout: exercises the bounded waits that every
// libmoe pipeline uses, against a barrier and a counter that nothing completes, so
// that the timeout path (flag in the status word, orderly exit, usable context) can
// be tested without hanging or faulting a GPU.
#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

// Block 0 waits on an mbarrier phase that never completes (the pipeline wait of the
// GEMM kernels); block 1 waits for a device counter that nothing increments (the
// dependency wait of the fused small-batch FFN).  Both give up after limit_ns.
__global__ void selftest_wait_kernel(uint32_t* status, const uint32_t* never_set,
                                     unsigned long long limit_ns, uint32_t* outcome) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival that never comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bool ok;
        if (blockIdx.x == 0)
            ok = mbar_wait_bounded(&bar, 0, &abort_flag, status, limit_ns);
        else
            ok = flag_wait_bounded(never_set, 1u, &abort_flag, status, limit_ns);
        outcome[blockIdx.x] = ok ? 1u : 2u;  // 2 = gave up, as it must
    }
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t* status, uint32_t* scratch, unsigned long long limit_ns,
                                 cudaStream_t s) {
    // scratch[0] stays zero (the counter nothing sets); scratch[1..2] get the outcomes
    cudaError_t err = cudaMemsetAsync(scratch, 0, 3 * sizeof(uint32_t), s);
    if (err != cudaSuccess) return err;
    selftest_wait_kernel<<<2, 32, 0, s>>>(status, scratch, limit_ns, scratch + 1);
    return cudaGetLastError();
}

}  // namespace moe
