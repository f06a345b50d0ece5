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
// up once per device with cudaGetSymbolAddress, with that device current, and
// that address is what the kernels receive.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxNoAllocDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::atomic<void *> g_scratch_addr[kMaxNoAllocDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device (looked up on
// the first call per device).  Returns nullptr if the lookup fails.
void *scratch_on_current_device(int *status) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxNoAllocDevices) {
        cudaGetLastError();
        *status = PA_ERR_CUDA;
        return nullptr;
    }
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (p) return p;
    void *addr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess || !addr) {
        cudaGetLastError();
        *status = PA_ERR_CUDA;
        return nullptr;
    }
    g_scratch_addr[dev].store(addr, std::memory_order_release);
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
