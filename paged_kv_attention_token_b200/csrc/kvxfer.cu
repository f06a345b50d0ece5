// KV export and import: a request's K/V between the paged cache and a
// contiguous buffer ("vLLM 学习笔记 01" §2.5, prefill/decode disaggregation:
// prefill instances produce a request's full KV cache and a connector moves
// it to the decode instances; §1.5 for the block table that says where each
// of a request's 16-token blocks lives).
//
// Token p of request i (0 <= p < n_i, n_i = cu_tokens[i + 1] - cu_tokens[i])
// is row cu_tokens[i] + p of the contiguous buffers [N][Hkv][D] and row
// p % 16 of cache block block_tables[i][p / 16].  Export copies cache ->
// buffer, import buffer -> cache, bit for bit.
//
// HBM-bound copy, the same shape as the cache scatter: one thread moves one
// 16-byte chunk of one token's K (and the same chunk of its V); a token's
// Hkv * D values are contiguous on both sides, so consecutive threads touch
// consecutive chunks.  A thread finds its request by binary search over
// cu_tokens (a warp's threads share a token row, hence the search path).
// Rows whose block entry is outside the table or the pool are skipped
// (precondition violations; no access is made).
#include "common.cuh"
#include "transfer.h"

namespace pa {

namespace {

template <bool kExport>
__global__ void __launch_bounds__(256) kv_transfer_kernel(
    const uint4 *__restrict__ src_k, const uint4 *__restrict__ src_v, uint4 *__restrict__ dst_k,
    uint4 *__restrict__ dst_v, const int32_t *__restrict__ block_tables, const int32_t *__restrict__ cu_tokens,
    int num_seqs, int max_blocks_per_seq, int64_t num_blocks, int64_t num_chunks, int chunks_per_token) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < num_chunks; c += stride) {
        const int64_t r = c / chunks_per_token;
        const int64_t part = c - r * chunks_per_token;
        // request i: cu_tokens[i] <= r < cu_tokens[i + 1]
        int lo = 0, hi = num_seqs;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(cu_tokens + mid) <= r)
                lo = mid;
            else
                hi = mid;
        }
        const int64_t p = r - __ldg(cu_tokens + lo);
        if (p < 0 || p / kBlockSize >= max_blocks_per_seq) continue;
        const int32_t blk = __ldg(block_tables + (int64_t)lo * max_blocks_per_seq + p / kBlockSize);
        if (blk < 0 || blk >= num_blocks) continue;
        const int64_t slot_chunk = ((int64_t)blk * kBlockSize + p % kBlockSize) * chunks_per_token + part;
        if (kExport) {
            dst_k[c] = ld_stream16(src_k + slot_chunk);
            dst_v[c] = ld_stream16(src_v + slot_chunk);
        } else {
            dst_k[slot_chunk] = ld_stream16(src_k + c);
            dst_v[slot_chunk] = ld_stream16(src_v + c);
        }
    }
}

}  // namespace

cudaError_t launch_kv_transfer(bool do_export, const void *src_k, const void *src_v, void *dst_k, void *dst_v,
                               const int32_t *block_tables, const int32_t *cu_tokens, int num_seqs,
                               int max_blocks_per_seq, int64_t num_blocks, int64_t num_tokens, int token_elems,
                               int num_sms, cudaStream_t stream) {
    const int chunks_per_token = token_elems / 8;  // 8 bf16 per 16 bytes
    const int64_t num_chunks = num_tokens * chunks_per_token;
    if (num_chunks == 0 || num_seqs == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (num_chunks + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms * 8;  // 8 resident CTAs of 256 threads per SM
    if (blocks > cap) blocks = cap;
    const uint4 *sk = static_cast<const uint4 *>(src_k), *sv = static_cast<const uint4 *>(src_v);
    uint4 *dk = static_cast<uint4 *>(dst_k), *dv = static_cast<uint4 *>(dst_v);
    if (do_export)
        kv_transfer_kernel<true><<<(unsigned)blocks, threads, 0, stream>>>(
            sk, sv, dk, dv, block_tables, cu_tokens, num_seqs, max_blocks_per_seq, num_blocks, num_chunks,
            chunks_per_token);
    else
        kv_transfer_kernel<false><<<(unsigned)blocks, threads, 0, stream>>>(
            sk, sv, dk, dv, block_tables, cu_tokens, num_seqs, max_blocks_per_seq, num_blocks, num_chunks,
            chunks_per_token);
    return cudaGetLastError();
}

}  // namespace pa
