// Kernel launchers of libpa.so (internal).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "plan.h"

namespace pa {

struct DecodeParams {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_cache;
    const __nv_bfloat16 *v_cache;
    const int32_t *block_tables;
    __nv_bfloat16 *out;
    float *partial_o;       // [pieces][G][D]
    float2 *partial_ml;     // [pieces][G]: (max in log2 units, sum)
    const DecodeUnit *units;
    const DecodeRow *rows;
    const CombineRow *combine;
    uint32_t *arrived;          // per combine row: tickets taken (plan tables; zero between calls)
    uint32_t *status;           // workspace status word (error bits)
    int num_units;
    int num_q_heads;
    int num_kv_heads;
    int group;
    int max_blocks_per_seq;
    float scale_log2;
    int defer_merge;            // nonzero: split rows only write partials (merge_kernel follows)
    // fused step: K/V of this step's tokens ([T][Hkv][D]), read instead of
    // their cache slots (null: every key comes from the cache)
    const __nv_bfloat16 *k_new;
    const __nv_bfloat16 *v_new;
    int wait_first;             // 0 only right behind the step's own scatter (see decode_kernel)
    // nonzero: lets the next launch on the stream (the step's own scatter,
    // queued behind it) go as the kernel starts
    int trigger_dependents;
};

// behind: launched programmatically behind the kernels of its own step (it
// then starts as they let it and waits for them at its end); otherwise a
// plain launch.
cudaError_t launch_reshape_and_cache(const void *k, const void *v, const int64_t *slots,
                                     void *k_cache, void *v_cache, int64_t num_tokens,
                                     int token_elems, int64_t num_slots, int num_sms, bool behind,
                                     cudaStream_t stream);

cudaError_t launch_decode(const DecodeParams &p, int head_dim, cudaStream_t stream);
// Merges all combine rows (after a decode launch with defer_merge).
// programmatic: launched with programmatic stream serialization right behind
// that decode launch on the same stream (its CTAs wait for the decode kernel
// in the kernel); otherwise a plain launch.
cudaError_t launch_merge(const DecodeParams &p, int head_dim, int num_combine, bool programmatic,
                         cudaStream_t stream);

struct PrefillParams {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_cache;
    const __nv_bfloat16 *v_cache;
    const int32_t *block_tables;
    const int32_t *cu_seqlens_q;
    const int32_t *seq_lens;
    __nv_bfloat16 *out;
    const PrefillTile *tiles;  // grouped by CTA
    const int32_t *cta_start;  // CTA c owns tiles [cta_start[c], cta_start[c + 1])
    const StageTile *stages;   // the gather kernel's list
    uint8_t *staged;          // staged K/V tiles (workspace)
    // a fused step's own K/V ([T][Hkv][D]), or null: with them, the pair
    // kernel reads a segment's key tiles whose keys are all this step's
    // tokens from here, and those tiles are not staged
    const __nv_bfloat16 *k_new;
    const __nv_bfloat16 *v_new;
    // shared-prefix tiles write partials of the decode rows they serve
    const DecodeRow *rows;
    const CombineRow *combine;
    float *partial_o;         // [pieces][G][D]
    float2 *partial_ml;       // [pieces][G]: (max in log2 units, sum)
    uint32_t *status;
    int num_tiles;
    int num_ctas;   // persistent CTAs, or with `pair` clusters of two CTAs
    int pair;       // every tile's two heads on a cluster of two CTAs (one head each)
    int num_stages;
    int num_tokens;  // rows of q (extent of its TMA descriptor)
    int num_blocks;  // blocks of the pool (extent of the cache descriptors)
    int num_q_heads;
    int num_kv_heads;
    int group;
    int max_blocks_per_seq;
    float scale_log2;
    long long wait_limit;  // SM cycles an mbarrier wait may take before the kernel gives up
    // pair kernel launched programmatically behind a kernel it reads nothing
    // of (a fused step's plain scatter): it waits for that kernel at its end
    int wait_at_end;
};

// Gathers the staged K/V tiles (must precede launch_prefill in stream order).
cudaError_t launch_stage(const PrefillParams &p, int head_dim, cudaStream_t stream);

// A fused step's cache write: this step's K/V ([T][Hkv][D]) into their slots.
struct ScatterArgs {
    const void *k;
    const void *v;
    const int64_t *slots;
    void *k_cache;
    void *v_cache;
    int64_t num_tokens;
    int token_elems;   // Hkv * D
    int64_t num_slots;  // blocks * 16
    int num_sms;
};
// The cache write and the staging of p's tiles in one launch: the staged
// rows of this step's own keys come from a.k / a.v, so neither part waits
// for the other (every token's slot must be the cache position its segment's
// block table gives it).  Without staged tiles, the plain scatter kernel.
cudaError_t launch_scatter_stage(const ScatterArgs &a, const PrefillParams &p, int head_dim,
                                 cudaStream_t stream);
cudaError_t launch_prefill(const PrefillParams &p, int head_dim, cudaStream_t stream);

// Self-test of the bounded-wait error path: one CTA holds tensor memory,
// waits on an mbarrier that nothing arrives at for `limit` cycles, records
// kStatusWaitTimeout in *status and releases the tensor memory.
cudaError_t launch_wait_selftest(uint32_t *status, long long limit, cudaStream_t stream);

// Data-dependent precondition checks; writes a nonzero flag word on failure.
cudaError_t launch_validate(const int64_t *slots, const int32_t *block_tables,
                            const int32_t *cu_seqlens_q, const int32_t *seq_lens,
                            const pa_dims &d, uint32_t *slot_bitmap, size_t bitmap_words,
                            uint32_t *flag, cudaStream_t stream);

}  // namespace pa
