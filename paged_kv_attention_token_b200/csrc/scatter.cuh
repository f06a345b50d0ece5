// The cache write of reshape_and_cache as a device function, shared by the
// scatter kernel and by the kernel that scatters and stages in one launch.
#pragma once
#include "common.cuh"

namespace pa {

// Writes each scheduled token's K and V into its cache slot ("vLLM 学习笔记
// 01" §1.6: per token, the slot mapping names the block and the row its K/V
// go to; slot = block_id * 16 + row).  One thread moves one 16-byte chunk of
// one token's K (and the same chunk of its V), chunks first .. num_chunks - 1
// in steps of `stride`: a token's Hkv * D values are contiguous both in k/v
// [T][Hkv][D] and in its cache row [NB][16][Hkv][D], so consecutive threads
// read and write consecutive 16-byte chunks (full sectors on both sides).
__device__ __forceinline__ void scatter_chunks(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                               const int64_t *__restrict__ slots, uint4 *__restrict__ k_cache,
                                               uint4 *__restrict__ v_cache, int64_t num_chunks,
                                               int chunks_per_token, int64_t num_slots, int64_t first,
                                               int64_t stride) {
    for (int64_t c = first; c < num_chunks; c += stride) {
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

}  // namespace pa
