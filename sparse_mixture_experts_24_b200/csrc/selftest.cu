// selftest.cu -- exercises the bounded-wait path of the pipelined kernels
// without breaking anything: one thread waits on an mbarrier that nothing ever
// arrives at, through the same mbar_wait helper the GEMM and router pipelines
// use, with a short budget.  The wait runs out, the kernel sets a status bit
// and returns normally, and the host reads MOE_ERR_TIMEOUT from
// moe_sync_status while the CUDA context stays usable.
#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void __launch_bounds__(32) bounded_wait_probe_kernel(int* status, long long budget_cycles) {
    __shared__ __align__(8) uint64_t bar;
    griddep_wait();
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
        // no thread and no copy ever arrives: the phase never completes
        mbar_wait(smem_u32(&bar), 0, status, kStatusSelfTest, budget_cycles);
    }
    __syncwarp();
}

cudaError_t launch_bounded_wait_probe(int* status, long long budget_cycles, cudaStream_t st) {
    launch_k(bounded_wait_probe_kernel, dim3(1), dim3(32), 0, st, status, budget_cycles);
    return cudaGetLastError();
}

}  // namespace moe
