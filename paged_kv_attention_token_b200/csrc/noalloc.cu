// pa_attention_varlen_noalloc: the varlen paged attention call for callers
// that cannot allocate device memory.
//
// Who needs it: an engine that hands almost all of a GPU's memory to its KV
// pool at start-up and runs its step loop with no allocator left to draw
// scratch from; hosts and plugin interfaces that pass an op only its input
// and output pointers and a stream; and loops where a cudaMalloc/cudaFree
// pair would stall the device (both may synchronize).  Such a caller cannot
// provide the workspace pa_attention_varlen asks for, so this entry point
// takes its scratch from a fixed array that lives in the library's own device
// memory image instead.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes.
// Every GPU that loads the library holds it until the process exits.  Host
// code must not pass the variable's name to a kernel (on the host it is only
// a stand-in symbol, not a device address), so its device address is looked
// up with cudaGetSymbolAddress, with the device current, once per device and
// CUDA context (a context created anew, e.g. after cudaDeviceReset, loads the
// library's device image again, possibly elsewhere), and that address is
// what the kernels receive.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxNoAllocDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchAddr {
    CUcontext ctx = nullptr;  // context the address was looked up in
    void *addr = nullptr;
};
ScratchAddr g_scratch[kMaxNoAllocDevices];
std::mutex g_scratch_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);

// The calling thread's current CUDA context, through the runtime's driver
// entry point (no link-time dependency on the driver library).
bool current_context(CUcontext *ctx) {
    static std::atomic<CtxGetCurrentFn> fn{nullptr};
    CtxGetCurrentFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !ptr) {
            cudaGetLastError();
            return false;
        }
        f = reinterpret_cast<CtxGetCurrentFn>(ptr);
        fn.store(f, std::memory_order_release);
    }
    return f(ctx) == CUDA_SUCCESS && *ctx != nullptr;
}

// Device address of the scratch array on the current device, looked up on
// the first call per device and again whenever the device's current context
// is another one than the lookup's.  Returns nullptr (and sets *status) if
// the lookup fails.
void *scratch_on_current_device(int *status) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxNoAllocDevices) {
        cudaGetLastError();
        *status = PA_ERR_CUDA;
        return nullptr;
    }
    // (before the thread's first runtime call there may be no context yet:
    // the lookup below creates the device's primary context)
    CUcontext ctx = nullptr;
    const bool had_ctx = current_context(&ctx);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchAddr &e = g_scratch[dev];
    if (had_ctx && e.addr && e.ctx == ctx) return e.addr;
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr ||
        (!had_ctx && !current_context(&ctx))) {
        cudaGetLastError();
        *status = PA_ERR_CUDA;
        return nullptr;
    }
    e.ctx = ctx;
    e.addr = addr;
    return addr;
}

}  // namespace
}  // namespace pa

extern "C" size_t pa_noalloc_scratch_bytes(void) { return pa::kNoAllocScratchBytes; }

extern "C" int pa_attention_varlen_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                           const int32_t *block_tables, const int32_t *cu_seqlens_q,
                                           const int32_t *seq_lens, float scale, void *out,
                                           const pa_dims *dims, const pa_plan *plan, void *stream) {
    if (!plan) return PA_ERR_NULL;
    // Reject a plan whose scratch would not fit before touching the device.
    if (pa_plan_workspace_bytes(plan) > pa::kNoAllocScratchBytes) return PA_ERR_TOO_LARGE;
    int status = PA_OK;
    void *scratch = pa::scratch_on_current_device(&status);
    if (!scratch) return status;
    return pa_attention_varlen_ex(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens, scale,
                                  out, dims, plan, scratch, pa::kNoAllocScratchBytes, stream, nullptr);
}

extern "C" int pa_noalloc_status(uint32_t *status, int clear, void *stream_) {
    if (!status) return PA_ERR_NULL;
    int st = PA_OK;
    void *scratch = pa::scratch_on_current_device(&st);
    if (!scratch) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (cudaMemcpyAsync(status, scratch, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return pa::cuda_error();
    if (clear && cudaMemsetAsync(scratch, 0, pa::kHeaderBytes, stream) != cudaSuccess) return pa::cuda_error();
    if (cudaStreamSynchronize(stream) != cudaSuccess) return pa::cuda_error();
    return PA_OK;
}
