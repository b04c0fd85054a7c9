// Fault injection for the bounded waits, without a GPU fault: one warp whose
// lane 0 waits, with the same bounded mbarrier wait every kernel of the
// library uses, on a barrier that nothing ever arrives on. The wait gives up
// after its budget (kWaitCycles SM clocks, about 2 s), records the timeout in
// the per-device status word and the kernel returns, so the context stays
// usable and the host reads the timeout through sas_get_error_flag.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace sas {
namespace {

using namespace sm100;

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        volatile int* abort = &abort_flag;
        mbar_wait(&bar, 0, abort, status);   // phase 0 never completes: gives up on the budget
    }
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int* status, cudaStream_t st) {
    bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(status);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace sas
