// reshape_and_cache: write each scheduled token's K and V into its cache slot
// ("vLLM 学习笔记 01" §1.6: per token, the slot mapping names the block and
// the row its K/V go to; slot = block_id * 16 + row).
//
// HBM-bound copy (scatter_chunks): one thread per 16-byte chunk of a token's
// K and V.  The grid is a whole number of waves over the SMs.
#include "common.cuh"
#include "kernels.h"
#include "scatter.cuh"

namespace pa {

__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4 *__restrict__ k, const uint4 *__restrict__ v, const int64_t *__restrict__ slots,
    uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache, int64_t num_chunks,
    int chunks_per_token, int64_t num_slots, int wait_at_end) {
    // an attention kernel queued next may set up while the copy runs (not
    // behind the step's attention kernels: what follows then, a merge, waits
    // for all of them, and its CTAs would only hold room early)
    if (!wait_at_end) grid_launch_dependents();
    scatter_chunks(k, v, slots, k_cache, v_cache, num_chunks, chunks_per_token, num_slots,
                   (int64_t)blockIdx.x * blockDim.x + threadIdx.x, (int64_t)gridDim.x * blockDim.x);
    // launched programmatically behind the step's attention kernels: what
    // follows on the stream follows them too
    if (wait_at_end) grid_dependency_wait();
}

cudaError_t launch_reshape_and_cache(const void *k, const void *v, const int64_t *slots,
                                     void *k_cache, void *v_cache, int64_t num_tokens,
                                     int token_elems, int64_t num_slots, int num_sms, bool behind,
                                     cudaStream_t stream) {
    const int chunks_per_token = token_elems / 8;  // 8 bf16 per 16 bytes
    const int64_t num_chunks = num_tokens * chunks_per_token;
    if (num_chunks == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (num_chunks + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms * 8;  // 8 resident CTAs of 256 threads per SM
    if (blocks > cap) blocks = cap;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(threads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = behind ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, reshape_and_cache_kernel, static_cast<const uint4 *>(k),
                                             static_cast<const uint4 *>(v), slots, static_cast<uint4 *>(k_cache),
                                             static_cast<uint4 *>(v_cache), num_chunks, chunks_per_token, num_slots,
                                             behind ? 1 : 0);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace pa
