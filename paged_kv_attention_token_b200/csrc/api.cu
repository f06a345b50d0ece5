// C ABI of libpa.so: argument checks, plan/workspace plumbing and launches.
// The declarations, with the meaning of every argument, are in include/pa.h.
#include <atomic>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "transfer.h"

namespace pa {

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common_dims(const pa_dims *d) {
    if (!d) return PA_ERR_NULL;
    if (d->num_tokens < 0 || d->num_seqs < 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0 ||
        d->head_dim <= 0 || d->num_blocks <= 0 || d->max_blocks_per_seq < 0 || d->block_size <= 0)
        return PA_ERR_SHAPE;
    if (d->num_q_heads % d->num_kv_heads != 0) return PA_ERR_SHAPE;
    if (d->block_size != kBlockSize) return PA_ERR_UNSUPPORTED;
    if (d->head_dim != 64 && d->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (d->num_q_heads / d->num_kv_heads > 16) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

int current_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    return device_sm_count(dev);
}

}  // namespace

int device_sm_count(int device) {
    if (device < 0 || device >= kMaxDevices) return 148;
    int v = g_sm_count[device].load(std::memory_order_relaxed);
    if (v > 0) return v;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) {
        cudaGetLastError();  // clear the sticky-free error so later calls are not blamed
        return 148;
    }
    g_sm_count[device].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace pa

using namespace pa;

extern "C" const char *pa_version(void) { return "0.1.0"; }

extern "C" const char *pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "ok";
        case PA_ERR_NULL: return "a required pointer is NULL";
        case PA_ERR_SHAPE: return "inconsistent or negative sizes";
        case PA_ERR_DTYPE: return "wrong dtype";
        case PA_ERR_ALIGN: return "a base address is not 16-byte aligned";
        case PA_ERR_UNSUPPORTED: return "unsupported shape (block_size 16, head_dim 64/128, group <= 16)";
        case PA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case PA_ERR_BOUNDS: return "input precondition violated (slot, block id or segment bounds)";
        case PA_ERR_CUDA: return "CUDA error";
        case PA_ERR_PLAN: return "plan does not match the call";
        case PA_ERR_TOO_LARGE:
            return "call needs more scratch than the 16 MiB no-alloc array holds; "
                   "use pa_attention_varlen with a workspace";
        default: return "unknown status";
    }
}

extern "C" int pa_reshape_and_cache(const void *k, const void *v, const int64_t *slot_mapping,
                                    void *k_cache, void *v_cache, const pa_dims *dims,
                                    void *stream) {
    if (!dims) return PA_ERR_NULL;
    const pa_dims &d = *dims;
    if (d.num_tokens < 0 || d.num_kv_heads <= 0 || d.head_dim <= 0 || d.num_blocks <= 0 ||
        d.block_size <= 0)
        return PA_ERR_SHAPE;
    if (d.block_size != kBlockSize) return PA_ERR_UNSUPPORTED;
    if (d.head_dim != 64 && d.head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (d.num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_NULL;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PA_ERR_ALIGN;
    const cudaError_t e = launch_reshape_and_cache(
        k, v, slot_mapping, k_cache, v_cache, d.num_tokens, d.num_kv_heads * d.head_dim,
        (int64_t)d.num_blocks * d.block_size, current_sm_count(), false,
        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : cuda_error();
}

namespace {
inline cudaError_t mark(const pa_trace *trace, int i, cudaStream_t stream) {
    if (!trace || !trace->events[i]) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(trace->events[i]), stream);
}
}  // namespace

namespace {
// Per-device stream of the least priority, created on first use, on which
// the decode kernel runs when it shares the GPU with the prefill kernel.
// Never destroyed (it lives as long as the process's context).
cudaStream_t side_stream(int device) {
    static std::mutex mu;
    static cudaStream_t streams[64] = {};
    if (device < 0 || device >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!streams[device]) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return nullptr;
        cudaStream_t s = nullptr;
        if (cudaStreamCreateWithPriority(&s, cudaStreamNonBlocking, least) != cudaSuccess) return nullptr;
        streams[device] = s;
    }
    return streams[device];
}
}  // namespace

extern "C" int pa_attention_varlen(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *block_tables, const int32_t *cu_seqlens_q,
                                   const int32_t *seq_lens, float scale, void *out,
                                   const pa_dims *dims, const pa_plan *plan, void *workspace,
                                   size_t workspace_bytes, void *stream_) {
    return pa_attention_varlen_ex(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens, scale,
                                  out, dims, plan, workspace, workspace_bytes, stream_, nullptr);
}

namespace {
// Host checks of an attention call: PA_OK when it may be queued (or when
// there is nothing to do: T == 0).
int check_attention(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                    const int32_t *cu_seqlens_q, const int32_t *seq_lens, const void *out, const pa_dims *dims,
                    const pa_plan *plan, const void *workspace, size_t workspace_bytes) {
    int st = check_common_dims(dims);
    if (st != PA_OK) return st;
    if (!plan) return PA_ERR_NULL;
    const pa_dims &d = *dims;
    const pa_dims &pd = plan->dims;
    if (pd.num_tokens != d.num_tokens || pd.num_seqs != d.num_seqs ||
        pd.num_q_heads != d.num_q_heads || pd.num_kv_heads != d.num_kv_heads ||
        pd.head_dim != d.head_dim || pd.block_size != d.block_size)
        return PA_ERR_PLAN;
    if (d.num_tokens == 0) return PA_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !cu_seqlens_q || !seq_lens || !out)
        return PA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return PA_ERR_ALIGN;
    const WorkspaceLayout &w = plan->ws;
    if (!workspace || workspace_bytes < w.total) return PA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kWorkspaceAlign) return PA_ERR_WORKSPACE;
    // the plan's tables live on its device
    int cur = -1;
    if (!plan->d_tables || cudaGetDevice(&cur) != cudaSuccess || cur != plan->device) return PA_ERR_PLAN;
    return PA_OK;
}

// Queues the attention kernels of a checked call.  k_new / v_new (a fused
// step, right behind the step's own scatter on `stream_`): the decode kernel
// reads this step's keys from them.
int queue_attention(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                    const int32_t *cu_seqlens_q, const int32_t *seq_lens, float scale, void *out,
                    const pa_dims &d, const pa_plan *plan, void *workspace, void *stream_, const pa_trace *trace,
                    const void *k_new, const void *v_new, const ScatterArgs *scatter) {
    const WorkspaceLayout &w = plan->ws;
    const TableLayout &tl = plan->tl;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const uint8_t *tb = static_cast<const uint8_t *>(plan->d_tables);
    if (mark(trace, 0, stream) != cudaSuccess) return cuda_error();
    // The plan's tables are on the device since its build returned, so
    // nothing sits between the caller's previous kernel and the decode
    // kernel's programmatic launch.  Under stream capture (a CUDA graph) the
    // plan-use event below is not recorded: a graph replay is not tracked by
    // the plan, whose rebuild then must not overlap one.
    cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &capture) != cudaSuccess) return cuda_error();
    const bool track_use = capture == cudaStreamCaptureStatusNone;
    const float scale_log2 = scale * kLog2e;
    DecodeParams p{};
    if (plan->num_units > 0) {
        p.q = static_cast<const __nv_bfloat16 *>(q);
        p.k_cache = static_cast<const __nv_bfloat16 *>(k_cache);
        p.v_cache = static_cast<const __nv_bfloat16 *>(v_cache);
        p.block_tables = block_tables;
        p.out = static_cast<__nv_bfloat16 *>(out);
        p.partial_o = reinterpret_cast<float *>(ws + w.partial_o);
        p.partial_ml = reinterpret_cast<float2 *>(ws + w.partial_ml);
        p.units = reinterpret_cast<const DecodeUnit *>(tb + tl.units);
        p.rows = reinterpret_cast<const DecodeRow *>(tb + tl.rows);
        p.combine = reinterpret_cast<const CombineRow *>(tb + tl.combine);
        p.arrived = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(plan->d_tables) + tl.arrived);
        p.status = reinterpret_cast<uint32_t *>(ws + w.header);
        p.num_units = plan->num_units;
        p.num_q_heads = d.num_q_heads;
        p.num_kv_heads = d.num_kv_heads;
        p.group = plan->group;
        p.max_blocks_per_seq = d.max_blocks_per_seq;
        p.scale_log2 = scale_log2;
        p.defer_merge = 0;
        p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
        p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
        p.wait_first = 1;
    }
    PrefillParams pp{};
    if (plan->num_tiles > 0) {
        pp.q = static_cast<const __nv_bfloat16 *>(q);
        pp.k_cache = static_cast<const __nv_bfloat16 *>(k_cache);
        pp.v_cache = static_cast<const __nv_bfloat16 *>(v_cache);
        pp.block_tables = block_tables;
        pp.cu_seqlens_q = cu_seqlens_q;
        pp.seq_lens = seq_lens;
        pp.out = static_cast<__nv_bfloat16 *>(out);
        pp.tiles = reinterpret_cast<const PrefillTile *>(tb + tl.tiles);
        pp.cta_start = reinterpret_cast<const int32_t *>(tb + tl.cta_start);
        pp.pair = plan->prefill_pair ? 1 : 0;
        pp.num_ctas = plan->prefill_pair ? plan->num_prefill_ctas / 2 : plan->num_prefill_ctas;
        pp.stages = reinterpret_cast<const StageTile *>(tb + tl.stages);
        pp.staged = ws + w.staged;
        pp.num_stages = plan->num_stages;
        pp.rows = reinterpret_cast<const DecodeRow *>(tb + tl.rows);
        pp.combine = reinterpret_cast<const CombineRow *>(tb + tl.combine);
        pp.partial_o = reinterpret_cast<float *>(ws + w.partial_o);
        pp.partial_ml = reinterpret_cast<float2 *>(ws + w.partial_ml);
        pp.status = reinterpret_cast<uint32_t *>(ws + w.header);
        pp.num_tiles = plan->num_tiles;
        pp.num_tokens = d.num_tokens;
        pp.num_blocks = d.num_blocks;
        pp.num_q_heads = d.num_q_heads;
        pp.num_kv_heads = d.num_kv_heads;
        pp.group = plan->group;
        pp.max_blocks_per_seq = d.max_blocks_per_seq;
        pp.scale_log2 = scale_log2;
        pp.wait_limit = kWaitLimitCycles;
    }
    pp.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    pp.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    // A fused step starts with its cache write, and the staging of the
    // prefill segments' keys runs in the same launch (their rows of this
    // step's tokens taken from its K/V input): nothing of the staging is left
    // in the branches below.
    // With the pair kernel and no tile of earlier keys to stage, the prefill
    // kernel reads nothing the scatter writes: it starts behind it by
    // programmatic launch and waits for it only at its end.
    const bool side_by_side = plan->overlap_sms > 0 && plan->num_units > 0 && plan->num_tiles > 0;
    // When neither attention kernel reads what the scatter writes (the pair
    // kernel with no tile of earlier keys to stage: every key it reads is an
    // earlier one from the cache, or this step's from the K/V input, and so
    // are the decode kernel's) and the two run side by side, the scatter is
    // queued last: a scatter queued first holds registers on the SMs the
    // prefill clusters need, and the decode launch waits until every
    // prefill CTA has started.
    const bool scatter_last =
        scatter && side_by_side && !trace && pp.pair && plan->num_stages_fused == 0;
    if (scatter && !scatter_last) {
        pp.wait_at_end = pp.pair && plan->num_stages_fused == 0 ? 1 : 0;
        if (pp.wait_at_end) pp.num_stages = 0;  // the plain scatter kernel
        if (launch_scatter_stage(*scatter, pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
        pp.num_stages = 0;
    }
    if (scatter_last) pp.num_stages = 0;
    if (side_by_side && !trace) {
        // The prefill kernel (persistent, one CTA per SM or SM pair, on
        // overlap_sms SMs) runs as soon as the staging kernel ends, so that
        // its CTAs are placed first; each of them lets the dependent launch
        // go as it starts.  The decode kernel, launched programmatically
        // behind it on the same stream and sized for the other SMs, fills
        // those SMs at once.  It reads nothing the staging or prefill
        // kernels write (its inputs were complete before the staging kernel
        // started), so it does not wait for them before its work, only at
        // its end: what follows on the stream follows both.
        if (launch_stage(pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (launch_prefill(pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
        // shared-prefix partials are not ready while the decode kernel runs:
        // it leaves every merge to the merge kernel behind both (launched
        // programmatically: its CTAs become resident as the decode kernel
        // ends, and wait for it before reading partials)
        p.defer_merge = plan->cascade ? 1 : 0;
        p.wait_first = 0;
        // a scatter queued last starts beside the decode kernel (in the
        // room its CTAs leave on their SMs) and waits for it at its end, so
        // that what follows still follows all three
        p.trigger_dependents = scatter_last ? 1 : 0;
        if (launch_decode(p, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (scatter_last &&
            launch_reshape_and_cache(scatter->k, scatter->v, scatter->slots, scatter->k_cache, scatter->v_cache,
                                     scatter->num_tokens, scatter->token_elems, scatter->num_slots,
                                     scatter->num_sms, true, stream) != cudaSuccess)
            return cuda_error();
        if (p.defer_merge && launch_merge(p, d.head_dim, plan->num_combine, true, stream) != cudaSuccess)
            return cuda_error();
        if (track_use && cudaEventRecord(static_cast<cudaEvent_t>(plan->use_event), stream) != cudaSuccess)
            return cuda_error();
        return PA_OK;
    } else if (side_by_side) {
        // Traced calls: the same two kernels side by side, with the decode
        // kernel on a side stream of the least priority (forked after the
        // staging kernel, joined before the merge), so that caller events
        // can bracket each kernel on its own stream.
        cudaStream_t side = side_stream(plan->device);
        if (!side) return cuda_error();
        cudaEvent_t fork = static_cast<cudaEvent_t>(plan->fork_event);
        cudaEvent_t join = static_cast<cudaEvent_t>(plan->join_event);
        if (launch_stage(pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (mark(trace, 4, stream) != cudaSuccess) return cuda_error();
        if (cudaEventRecord(fork, stream) != cudaSuccess) return cuda_error();
        if (launch_prefill(pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (cudaStreamWaitEvent(side, fork, 0) != cudaSuccess) return cuda_error();
        if (mark(trace, 1, side) != cudaSuccess) return cuda_error();
        // shared-prefix partials are not ready while the decode kernel runs:
        // it leaves every merge to the merge kernel after the join
        p.defer_merge = plan->cascade ? 1 : 0;
        if (launch_decode(p, d.head_dim, side) != cudaSuccess) return cuda_error();
        if (mark(trace, 2, side) != cudaSuccess || mark(trace, 3, side) != cudaSuccess) return cuda_error();
        if (mark(trace, 5, stream) != cudaSuccess) return cuda_error();  // prefill, not the join
        if (cudaEventRecord(join, side) != cudaSuccess || cudaStreamWaitEvent(stream, join, 0) != cudaSuccess)
            return cuda_error();
        if (p.defer_merge && launch_merge(p, d.head_dim, plan->num_combine, false, stream) != cudaSuccess)
            return cuda_error();
        if (track_use && cudaEventRecord(static_cast<cudaEvent_t>(plan->use_event), stream) != cudaSuccess)
            return cuda_error();
        return PA_OK;
    } else if (plan->cascade) {
        // shared-prefix partials first; the decode kernel merges them
        if (launch_stage(pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (mark(trace, 4, stream) != cudaSuccess) return cuda_error();
        if (launch_prefill(pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (mark(trace, 5, stream) != cudaSuccess || mark(trace, 1, stream) != cudaSuccess) return cuda_error();
        if (plan->num_units > 0 && launch_decode(p, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (mark(trace, 2, stream) != cudaSuccess || mark(trace, 3, stream) != cudaSuccess) return cuda_error();
        if (track_use && cudaEventRecord(static_cast<cudaEvent_t>(plan->use_event), stream) != cudaSuccess)
            return cuda_error();
        return PA_OK;
    } else {
        if (mark(trace, 1, stream) != cudaSuccess) return cuda_error();
        // right behind the step's own scatter (fused step, no trace events)
        p.wait_first = k_new != nullptr && !trace ? 0 : 1;
        if (plan->num_units > 0 && launch_decode(p, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (mark(trace, 2, stream) != cudaSuccess || mark(trace, 3, stream) != cudaSuccess) return cuda_error();
        if (plan->num_tiles > 0 && launch_stage(pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
        if (mark(trace, 4, stream) != cudaSuccess) return cuda_error();
        if (plan->num_tiles > 0 && launch_prefill(pp, d.head_dim, stream) != cudaSuccess) return cuda_error();
    }
    if (mark(trace, 5, stream) != cudaSuccess) return cuda_error();
    // the plan's next build waits for this
    if (track_use && cudaEventRecord(static_cast<cudaEvent_t>(plan->use_event), stream) != cudaSuccess)
        return cuda_error();
    return PA_OK;
}
}  // namespace

extern "C" int pa_attention_varlen_ex(const void *q, const void *k_cache, const void *v_cache,
                                      const int32_t *block_tables, const int32_t *cu_seqlens_q,
                                      const int32_t *seq_lens, float scale, void *out,
                                      const pa_dims *dims, const pa_plan *plan, void *workspace,
                                      size_t workspace_bytes, void *stream, const pa_trace *trace) {
    const int st = check_attention(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens, out, dims, plan,
                                   workspace, workspace_bytes);
    if (st != PA_OK || dims->num_tokens == 0) return st;
    return queue_attention(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens, scale, out, *dims, plan,
                           workspace, stream, trace, nullptr, nullptr, nullptr);
}

extern "C" int pa_reshape_and_attention(const void *k, const void *v, const int64_t *slot_mapping,
                                        const void *q, void *k_cache, void *v_cache,
                                        const int32_t *block_tables, const int32_t *cu_seqlens_q,
                                        const int32_t *seq_lens, float scale, void *out, const pa_dims *dims,
                                        const pa_plan *plan, void *workspace, size_t workspace_bytes,
                                        void *stream) {
    if (!dims) return PA_ERR_NULL;
    if (dims->num_tokens > 0) {
        if (!k || !v || !slot_mapping) return PA_ERR_NULL;
        if (!aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u)) return PA_ERR_ALIGN;
    }
    const int st = check_attention(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens, out, dims, plan,
                                   workspace, workspace_bytes);
    if (st != PA_OK || dims->num_tokens == 0) return st;
    const pa_dims &d = *dims;
    ScatterArgs sa{};
    sa.k = k;
    sa.v = v;
    sa.slots = slot_mapping;
    sa.k_cache = k_cache;
    sa.v_cache = v_cache;
    sa.num_tokens = d.num_tokens;
    sa.token_elems = d.num_kv_heads * d.head_dim;
    sa.num_slots = (int64_t)d.num_blocks * d.block_size;
    sa.num_sms = current_sm_count();
    return queue_attention(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens, scale, out, d, plan,
                           workspace, stream, nullptr, k, v, &sa);
}

namespace {
int kv_transfer(bool do_export, const void *src_k, const void *src_v, void *dst_k, void *dst_v,
                const int32_t *block_tables, const int32_t *cu_tokens, const pa_dims *dims, void *stream) {
    if (!dims) return PA_ERR_NULL;
    const pa_dims &d = *dims;
    if (d.num_tokens < 0 || d.num_seqs < 0 || d.num_kv_heads <= 0 || d.head_dim <= 0 || d.num_blocks <= 0 ||
        d.max_blocks_per_seq < 0 || d.block_size <= 0)
        return PA_ERR_SHAPE;
    if (d.block_size != kBlockSize) return PA_ERR_UNSUPPORTED;
    if (d.head_dim != 64 && d.head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (d.num_tokens == 0 || d.num_seqs == 0) return d.num_tokens == 0 ? PA_OK : PA_ERR_SHAPE;
    if (!src_k || !src_v || !dst_k || !dst_v || !block_tables || !cu_tokens) return PA_ERR_NULL;
    if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(cu_tokens) & 3u))
        return PA_ERR_ALIGN;
    const cudaError_t e = launch_kv_transfer(do_export, src_k, src_v, dst_k, dst_v, block_tables, cu_tokens,
                                             d.num_seqs, d.max_blocks_per_seq, d.num_blocks, d.num_tokens,
                                             d.num_kv_heads * d.head_dim, current_sm_count(),
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : cuda_error();
}
}  // namespace

extern "C" int pa_kv_export(const void *k_cache, const void *v_cache, const int32_t *block_tables,
                            const int32_t *cu_tokens, void *k_out, void *v_out, const pa_dims *dims,
                            void *stream) {
    return kv_transfer(true, k_cache, v_cache, k_out, v_out, block_tables, cu_tokens, dims, stream);
}

extern "C" int pa_kv_import(const void *k_in, const void *v_in, const int32_t *block_tables,
                            const int32_t *cu_tokens, void *k_cache, void *v_cache, const pa_dims *dims,
                            void *stream) {
    return kv_transfer(false, k_in, v_in, k_cache, v_cache, block_tables, cu_tokens, dims, stream);
}

extern "C" int pa_workspace_reset(void *workspace, const pa_plan *plan, void *stream_) {
    if (!workspace || !plan) return PA_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(workspace) % kWorkspaceAlign) return PA_ERR_WORKSPACE;
    if (cudaMemsetAsync(workspace, 0, kHeaderBytes, static_cast<cudaStream_t>(stream_)) != cudaSuccess)
        return cuda_error();
    return PA_OK;
}

extern "C" int pa_workspace_status(const void *workspace, void *stream_, uint32_t *status) {
    if (!workspace || !status) return PA_ERR_NULL;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (cudaMemcpyAsync(status, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return cuda_error();
    return PA_OK;
}

// ---------------------------------------------------------------------------
// pa_validate_inputs
// ---------------------------------------------------------------------------

namespace pa {

__global__ void validate_kernel(const int64_t *__restrict__ slots, const int32_t *__restrict__ bt,
                                const int32_t *__restrict__ cu, const int32_t *__restrict__ seq,
                                pa_dims d, uint32_t *__restrict__ bitmap, uint32_t *__restrict__ flag) {
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t num_slots = (int64_t)d.num_blocks * d.block_size;
    if (slots) {
        for (int64_t t = tid; t < d.num_tokens; t += stride) {
            const int64_t s = slots[t];
            if (s < 0) continue;
            if (s >= num_slots) {
                atomicOr(flag, 1u);
                continue;
            }
            const uint32_t bit = 1u << (s & 31);
            if (atomicOr(bitmap + (s >> 5), bit) & bit) atomicOr(flag, 2u);  // duplicate slot
        }
    }
    for (int64_t i = tid; i < d.num_seqs; i += stride) {
        const int32_t L = cu[i + 1] - cu[i];
        if (i == 0 && cu[0] != 0) atomicOr(flag, 4u);
        if (i == d.num_seqs - 1 && cu[d.num_seqs] != d.num_tokens) atomicOr(flag, 4u);
        if (L < 0 || seq[i] < L) {
            atomicOr(flag, 4u);
            continue;
        }
        if (L == 0) continue;
        const int64_t nb = ((int64_t)seq[i] + d.block_size - 1) / d.block_size;
        if (nb > d.max_blocks_per_seq) {
            atomicOr(flag, 8u);
            continue;
        }
        for (int64_t b = 0; b < nb; ++b) {
            const int32_t id = bt[i * (int64_t)d.max_blocks_per_seq + b];
            if (id < 0 || id >= d.num_blocks) {
                atomicOr(flag, 8u);
                break;
            }
        }
    }
}

cudaError_t launch_validate(const int64_t *slots, const int32_t *block_tables,
                            const int32_t *cu_seqlens_q, const int32_t *seq_lens, const pa_dims &d,
                            uint32_t *slot_bitmap, size_t bitmap_words, uint32_t *flag,
                            cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    if (slots && bitmap_words) {
        e = cudaMemsetAsync(slot_bitmap, 0, bitmap_words * sizeof(uint32_t), stream);
        if (e != cudaSuccess) return e;
    }
    const int threads = 256;
    int64_t work = d.num_tokens > d.num_seqs ? d.num_tokens : d.num_seqs;
    int64_t blocks = (work + threads - 1) / threads;
    if (blocks < 1) blocks = 1;
    if (blocks > 4096) blocks = 4096;
    validate_kernel<<<(unsigned)blocks, threads, 0, stream>>>(slots, block_tables, cu_seqlens_q,
                                                              seq_lens, d, slot_bitmap, flag);
    return cudaGetLastError();
}

}  // namespace pa

extern "C" size_t pa_validate_scratch_bytes(const pa_dims *d) {
    if (!d || d->num_blocks <= 0 || d->block_size <= 0) return 0;
    const size_t words = ((size_t)d->num_blocks * d->block_size + 31) / 32;
    return 256 + words * sizeof(uint32_t);
}

extern "C" int pa_validate_inputs(const int64_t *slot_mapping, const int32_t *block_tables,
                                  const int32_t *cu_seqlens_q, const int32_t *seq_lens,
                                  const pa_dims *dims, void *scratch, size_t scratch_bytes,
                                  void *stream_) {
    int st = check_common_dims(dims);
    if (st != PA_OK) return st;
    const pa_dims &d = *dims;
    if (!cu_seqlens_q || !seq_lens || (d.num_seqs > 0 && !block_tables)) return PA_ERR_NULL;
    if (!scratch || scratch_bytes < pa_validate_scratch_bytes(dims) ||
        reinterpret_cast<uintptr_t>(scratch) % kWorkspaceAlign)
        return PA_ERR_WORKSPACE;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    uint32_t *flag = static_cast<uint32_t *>(scratch);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(scratch) + 256);
    const size_t words = ((size_t)d.num_blocks * d.block_size + 31) / 32;
    if (launch_validate(slot_mapping, block_tables, cu_seqlens_q, seq_lens, d, bitmap, words, flag,
                        stream) != cudaSuccess)
        return cuda_error();
    uint32_t h_flag = 0;
    if (cudaMemcpyAsync(&h_flag, flag, sizeof h_flag, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return cuda_error();
    if (cudaStreamSynchronize(stream) != cudaSuccess) return cuda_error();
    return h_flag ? PA_ERR_BOUNDS : PA_OK;
}
