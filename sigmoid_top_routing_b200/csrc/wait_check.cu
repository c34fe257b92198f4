// moe_wait_bound_check: the failure detection of the grouped GEMM pipelines,
// exercised without a fault.
//
// Every mbarrier wait of the tcgen05 pipelines goes through sm100::mbar_wait
// with a poll limit; when it runs out the kernel writes device error code 2,
// stops issuing work, drains what it issued and returns, so the context stays
// usable and the host learns of it through moe_device_error.  This entry point
// runs that same helper in a one-CTA kernel on an mbarrier nothing ever
// arrives on, with a short limit chosen by the caller: no TMA, no TMEM, no
// tensor-core work, nothing else in flight.  The wait always ends (after at
// most `polls` polls) and reports code 2 exactly as a stalled pipeline would.
#include "../../include/moe.h"
#include "common.cuh"
#include "internal.h"
#include "launch.h"
#include "sm100.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(32) k_wait_bound_check(int* err, uint32_t polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        // phase 0 never completes: no thread arrives and no copy targets it
        if (!sm100::mbar_wait(&bar, 0, nullptr, polls)) report_error(err, kErrWaitExpired);
    }
    __syncwarp();
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_wait_bound_check(uint32_t polls, moe_stream_t stream) {
    if (polls < 1 || polls > (1u << 20)) {
        set_last_error("moe_wait_bound_check: polls must be in [1, 2^20]");
        return MOE_ERR_SHAPE;
    }
    int* err = device_info().err_word;
    if (!err) {
        set_last_error("moe_wait_bound_check: no device error word on this device");
        return MOE_ERR_CUDA;
    }
    cudaError_t e = launch_k(k_wait_bound_check, dim3(1), dim3(32), 0, reinterpret_cast<cudaStream_t>(stream),
                             false, err, polls);
    if (e != cudaSuccess) {
        set_last_error(cudaGetErrorString(e));
        return MOE_ERR_CUDA;
    }
    set_last_launch_count(1);
    return MOE_OK;
}
