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
    int chunks_per_token, int64_t num_slots) {
    // an attention kernel queued next may set up while the copy runs
    grid_launch_dependents();
    scatter_chunks(k, v, slots, k_cache, v_cache, num_chunks, chunks_per_token, num_slots,
                   (int64_t)blockIdx.x * blockDim.x + threadIdx.x, (int64_t)gridDim.x * blockDim.x);
}

cudaError_t launch_reshape_and_cache(const void *k, const void *v, const int64_t *slots,
                                     void *k_cache, void *v_cache, int64_t num_tokens,
                                     int token_elems, int64_t num_slots, int num_sms,
                                     cudaStream_t stream) {
    const int chunks_per_token = token_elems / 8;  // 8 bf16 per 16 bytes
    const int64_t num_chunks = num_tokens * chunks_per_token;
    if (num_chunks == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (num_chunks + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms * 8;  // 8 resident CTAs of 256 threads per SM
    if (blocks > cap) blocks = cap;
    reshape_and_cache_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), slots,
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), num_chunks,
        chunks_per_token, num_slots);
    return cudaGetLastError();
}

}  // namespace pa
