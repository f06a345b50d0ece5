// reshape_and_cache: write each scheduled token's K and V into its cache slot
// ("vLLM 学习笔记 01" §1.6: per token, the slot mapping names the block and
// the row its K/V go to; slot = block_id * 16 + row).
//
// HBM-bound copy.  One thread moves one 16-byte chunk of one token's K (and
// the same chunk of its V): a token's Hkv * D values are contiguous both in
// k/v [T][Hkv][D] and in its cache row [NB][16][Hkv][D], so consecutive
// threads read and write consecutive 16-byte chunks (full sectors on both
// sides).  The grid is a whole number of waves over the SMs.
#include "common.cuh"
#include "kernels.h"

namespace pa {

__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4 *__restrict__ k, const uint4 *__restrict__ v, const int64_t *__restrict__ slots,
    uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache, int64_t num_chunks,
    int chunks_per_token, int64_t num_slots) {
    // an attention kernel queued next may set up while the copy runs
    grid_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < num_chunks; c += stride) {
        const int64_t t = c / chunks_per_token;
        const int64_t part = c - t * chunks_per_token;
        // the chunk's K/V do not depend on the slot: all three loads are in
        // flight together, and only the stores wait for the slot
        const int64_t s = __ldg(slots + t);
        const uint4 kv = ld_stream16(k + c);
        const uint4 vv = ld_stream16(v + c);
        if (s < 0 || s >= num_slots) continue;  // negative: skip; past the pool: never written
        const int64_t dst = s * chunks_per_token + part;
        k_cache[dst] = kv;
        v_cache[dst] = vv;
    }
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
