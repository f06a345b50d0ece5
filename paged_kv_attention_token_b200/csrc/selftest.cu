// Self-test of the bounded-wait error path that the tensor-core kernels
// share.  Every mbarrier wait in them gives up after a limit, sets
// kStatusWaitTimeout in the caller's status word and lets the kernel run to
// its end, where tensor memory is released.  In normal operation no wait
// runs out, so this kernel makes one run out on purpose, safely: one CTA
// holds tensor memory as the prefill kernel does, waits on an mbarrier that
// nothing ever arrives at (no copy and no MMA is in flight), takes the error
// exit and releases the tensor memory.  The host then reads the status word
// through pa_workspace_status like any other.
#include "common.cuh"
#include "kernels.h"

namespace pa {

namespace {

constexpr uint32_t kSelftestTmemCols = 32;

__global__ void __launch_bounds__(128, 1) wait_selftest_kernel(uint32_t *status, long long limit) {
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&tmem_slot), kSelftestTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    bool err = false;
    // phase 0 of `bar` never completes: its one expected arrival never comes
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit)) err = true;
    if (err) atomicOr(status, kStatusWaitTimeout);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kSelftestTmemCols);
}

}  // namespace

cudaError_t launch_wait_selftest(uint32_t *status, long long limit, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 128, 0, stream>>>(status, limit);
    return cudaGetLastError();
}

}  // namespace pa

extern "C" int pa_selftest_wait_timeout(void *workspace, long long limit_cycles, void *stream) {
    if (!workspace) return PA_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(workspace) % pa::kWorkspaceAlign) return PA_ERR_WORKSPACE;
    if (limit_cycles < 1 || limit_cycles > pa::kWaitLimitCycles) return PA_ERR_SHAPE;
    const cudaError_t e =
        pa::launch_wait_selftest(static_cast<uint32_t *>(workspace), limit_cycles, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : pa::cuda_error();
}
