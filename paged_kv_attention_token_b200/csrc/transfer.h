// KV export / import launcher of libpa.so (internal).
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

namespace pa {

// KV export (cache -> contiguous [N][Hkv][D] buffers) or import (buffers ->
// cache) of the requests cu_tokens delimits, through their block tables.
cudaError_t launch_kv_transfer(bool do_export, const void *src_k, const void *src_v, void *dst_k, void *dst_v,
                               const int32_t *block_tables, const int32_t *cu_tokens, int num_seqs,
                               int max_blocks_per_seq, int64_t num_blocks, int64_t num_tokens, int token_elems,
                               int num_sms, cudaStream_t stream);

}  // namespace pa
