/*
 * pa.h — C ABI of libpa.so: the paged-KV attention step of one
 * continuous-batching forward pass, for NVIDIA B200 (sm_100a).
 *
 * The operation follows "vLLM 学习笔记 01：一个请求在 vLLM 里的一生":
 *   §1.5  the KV cache is cut into fixed 16-token blocks; each request owns a
 *         block table naming the physical block of each of its logical
 *         blocks, and the blocks need not be contiguous;
 *   §1.6  all tokens scheduled in a step are concatenated into one unpadded
 *         stream; the attention op is told where each segment starts and
 *         ends (segments cannot see one another), which slot (block and row)
 *         each new token's K/V is written to, and which blocks hold each
 *         segment's history; prefill chunks and single-token decodes share
 *         one batch;
 *   §1.4  a request tracks computed vs total tokens, so seq_len below counts
 *         the tokens scheduled in this step, and §2.1: a prefill chunk reads
 *         the context earlier chunks cached.
 * The block layout follows "Inside vLLM: Anatomy of a High-Throughput LLM
 * Inference System" (Chinese translation), section "LLM 引擎构造函数": a block
 * of a standard layer holds K and V of block_size tokens for every kv head.
 *
 * Conventions for every call
 *  - Pointers named d_* or described as "device" are CUDA device pointers on
 *    the current device; h_* pointers are host memory.  The caller owns every
 *    buffer and keeps it alive until the work queued on `stream` completes.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    are asynchronous on it unless stated otherwise.
 *  - bf16 tensors are row-major and contiguous, base addresses 16-byte
 *    aligned.  Shapes (T = num_tokens, S = num_seqs, Hq, Hkv, D = head_dim,
 *    NB = num_blocks, MB = max_blocks_per_seq, B = block_size):
 *        q, out        [T][Hq][D]      bf16
 *        k, v          [T][Hkv][D]     bf16
 *        k_cache       [NB][B][Hkv][D] bf16   (v_cache the same, separate)
 *        block_tables  [S][MB]         int32
 *        cu_seqlens_q  [S+1]           int32  (0, non-decreasing, ends at T)
 *        seq_lens      [S]             int32  (q_len <= seq_len)
 *        slot_mapping  [T]             int64
 *  - Supported: B == 16, D in {64, 128}, Hq % Hkv == 0, Hq / Hkv <= 16.
 *  - Every call returns a pa_status and never aborts, throws or traps.
 *    Violations checkable on the host (null pointers, sizes, alignment,
 *    unsupported shapes, workspace too small) are rejected before any work
 *    is queued.  Data-dependent preconditions (slots and block ids inside
 *    the pool, q_len <= seq_len, distinct slots, the device arrays agreeing
 *    with the host arrays the plan was built from) are not checked by the
 *    compute calls; pa_validate_inputs checks them on request.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_NULL = -1,        /* a required pointer is NULL */
    PA_ERR_SHAPE = -2,       /* inconsistent or negative sizes */
    PA_ERR_DTYPE = -3,       /* reserved: the binding reports wrong dtypes with it */
    PA_ERR_ALIGN = -4,       /* a base address is not 16-byte aligned */
    PA_ERR_UNSUPPORTED = -5, /* block_size != 16, head_dim not 64/128, group > 16 */
    PA_ERR_WORKSPACE = -6,   /* workspace NULL or smaller than the plan needs */
    PA_ERR_BOUNDS = -7,      /* pa_validate_inputs found a precondition violated */
    PA_ERR_CUDA = -8,        /* a CUDA runtime call or kernel launch failed */
    PA_ERR_PLAN = -9,        /* the plan does not match the dims of the call */
    PA_ERR_TOO_LARGE = -10   /* the call needs more scratch than the no-alloc
                                entry point's fixed array holds */
} pa_status;

/* Sizes of one call.  block_size must be 16. */
typedef struct {
    int32_t num_tokens;          /* T: scheduled tokens in the flat stream */
    int32_t num_seqs;            /* S: segments (requests) */
    int32_t num_q_heads;         /* Hq */
    int32_t num_kv_heads;        /* Hkv; query head h reads kv head h / (Hq/Hkv) */
    int32_t head_dim;            /* D: 64 or 128 */
    int32_t num_blocks;          /* NB: blocks in the pool */
    int32_t max_blocks_per_seq;  /* MB: columns of block_tables */
    int32_t block_size;          /* B: tokens per block, must be 16 */
} pa_dims;

/*
 * reshape_and_cache — "vLLM 学习笔记 01" §1.6: each new token's K/V is
 * written to the slot its slot mapping names.  For every t in [0, T) with
 * s = slot_mapping[t] >= 0: k_cache[s / 16][s % 16][:][:] = k[t][:][:] and
 * v_cache likewise, bit for bit.  A negative slot skips the token.  Nothing
 * else in the caches changes.
 *   d_k, d_v              device [T][Hkv][D] bf16, read
 *   d_slot_mapping        device [T] int64, read; each s < NB * 16 and no two
 *                         tokens share a slot (precondition)
 *   d_k_cache, d_v_cache  device [NB][16][Hkv][D] bf16, written in place
 *   dims                  host; num_seqs, num_q_heads, max_blocks_per_seq unused
 * T == 0 queues nothing and returns PA_OK.  The kernel lets a
 * programmatically launched kernel queued after it (the attention call's
 * decode kernel) start setting up early; that kernel still reads the caches
 * only after this one has completed.
 */
int pa_reshape_and_cache(const void *d_k, const void *d_v, const int64_t *d_slot_mapping,
                         void *d_k_cache, void *d_v_cache, const pa_dims *dims,
                         void *stream);

/*
 * Work partition for pa_attention_varlen.  From the host copies of cu_seqlens_q and seq_lens (the same values the
 * device arrays will hold) it splits the step into balanced GPU work:
 * segments with q_len <= 16 (decodes, speculative-verification shapes) are
 * cut into equal runs of 16-token KV blocks over all query rows and kv heads
 * (split-KV), one run per CTA and SM, the partials of rows cut between runs
 * being merged by the last CTA to finish them; longer segments are cut into
 * 128-query tiles for pairs of query heads sharing a kv head, for the
 * tensor-core prefill kernel and dealt to at most one CTA per SM.  The
 * resulting tables are uploaded to device memory the plan owns, on a stream
 * of the plan's own (a copy from page-locked memory, the only GPU work a
 * build queues); the call returns once they are on the device.  Build plans
 * outside stream capture.
 *   h_cu_seqlens_q  host [S+1] int32
 *   h_seq_lens      host [S] int32
 *   h_block_tables  host [S][MB] int32 (the values the device array will
 *                   hold), or NULL.  Given, the planner looks for shared
 *                   prefixes ("vLLM 学习笔记 01" §2.2, prefix caching: requests
 *                   whose tables start with the same physical blocks): runs
 *                   of at least 4 consecutive single-token segments whose
 *                   first 16 or more table entries agree.  For such a run the
 *                   prefill kernel attends all its tokens to the shared
 *                   blocks at once (a dense tensor-core pass that reads them
 *                   once per kv head) and leaves partials, and the decode
 *                   kernel reads only each row's later blocks and merges.
 *                   Only the first ceil(seq_len / 16) entries of a row are
 *                   read.
 *   dims            host; T, S, Hq, Hkv, D, B are used
 *   device          CUDA device ordinal the plan is built for (its SM count
 *                   is read once per process and cached; the device tables
 *                   are allocated there).  -1 builds a host-only plan that
 *                   assumes 148 SMs, for inspection with pa_plan_get_info;
 *                   attention calls reject it (PA_ERR_PLAN).
 *   out             in/out.  If *out is NULL a new plan is created and
 *                   stored there; the caller owns it and frees it with
 *                   pa_plan_destroy.  If *out holds a plan from an earlier
 *                   call (same device), that plan is rebuilt in place and its
 *                   buffers are reused (grown when too small), so that a
 *                   caller rebuilding one plan per step allocates nothing
 *                   after the first steps.  Rebuilding or destroying a plan
 *                   first waits (on the host) until its last upload and the
 *                   last attention call that used it have finished on the
 *                   GPU, so an engine that builds step k+1's plan while step
 *                   k runs keeps two plans and alternates.  A plan may serve
 *                   every layer of a step; calls that use the same plan must
 *                   not overlap on the GPU (queue them on one stream, or
 *                   order them with events), because the merge tickets of
 *                   split rows live in the plan's device tables.
 * On error a plan passed in *out is left unusable for attention calls until
 * it is rebuilt successfully; it must still be destroyed.
 * Errors: PA_ERR_NULL, PA_ERR_SHAPE (cu_seqlens not starting at 0, not
 * non-decreasing or not ending at T; q_len > seq_len), PA_ERR_UNSUPPORTED.
 */
typedef struct pa_plan pa_plan;
int pa_plan_build(const int32_t *h_cu_seqlens_q, const int32_t *h_seq_lens,
                  const int32_t *h_block_tables, const pa_dims *dims, int device,
                  pa_plan **out);

/* What a plan holds, for tests, logging and roofline accounting. */
typedef struct {
    int32_t num_sms;              /* SM count the plan was sized for */
    int32_t num_decode_rows;      /* (query token, kv head) rows on the split-KV path */
    int32_t num_decode_units;     /* warps of the split-KV kernel */
    int32_t num_partials;         /* partial results the combine step merges */
    int32_t num_combine_rows;     /* rows cut across more than one warp */
    int32_t num_prefill_tiles;    /* (128-query tile, query-head pair) items */
    int64_t decode_kv_blocks;     /* sum over decode rows of ceil(keys / 16) */
    int64_t prefill_causal_pairs; /* (query, visible key) pairs per query head */
    uint64_t table_bytes;         /* the plan's device tables (uploaded once per build) */
    uint64_t workspace_bytes;     /* = pa_plan_workspace_bytes */
    int32_t num_staged_kv_tiles;  /* 128-key K/V tiles gathered into the workspace
                                     (per kv head): those of the prefill
                                     segments, and of shared prefixes unless the
                                     pair kernel reads those from the cache */
    int32_t num_prefill_ctas;     /* persistent CTAs of the prefill kernel */
    int32_t num_prefix_groups;    /* shared-prefix runs found (h_block_tables given) */
    int32_t attention_launches;   /* kernels one pa_attention_varlen call launches
                                     (decode, staging, prefill, merge) */
    int64_t decode_kv_keys;       /* sum over decode rows of the keys the split-KV
                                     kernel attends (a row's keys, less a shared
                                     prefix the prefill kernel attends); unlike
                                     decode_kv_blocks, no padding of last blocks */
    int32_t prefill_pair;         /* 1: the prefill tiles run on clusters of two
                                     CTAs (num_prefill_ctas / 2 clusters, one
                                     query head per CTA, 2-SM MMAs); 0: one CTA
                                     per SM holds both heads of a tile */
    int32_t overlap_sms;          /* > 0: SMs the prefill kernel runs on beside
                                     the decode kernel; 0: one after the other */
} pa_plan_info;
int pa_plan_get_info(const pa_plan *plan, pa_plan_info *info);

/* Bytes of device workspace pa_attention_varlen needs with this plan
 * (0 for a NULL plan).  256-byte alignment of the workspace is required. */
size_t pa_plan_workspace_bytes(const pa_plan *plan);

/* Frees a plan (NULL is allowed), after waiting until its last upload and
 * the last attention call that used it have finished on the GPU. */
void pa_plan_destroy(pa_plan *plan);

/*
 * Varlen paged attention — "vLLM 学习笔记 01" §1.5-§1.6, §2.1.  For every
 * segment i with q_len L = cu_seqlens_q[i+1] - cu_seqlens_q[i] and seq_len n,
 * query j (0 <= j < L, flat token t = cu_seqlens_q[i] + j) sits at position
 * p = n - L + j (bottom-right causal alignment) and, for every query head h
 * with kv head g = h / (Hq / Hkv):
 *     z_tau  = scale * <q[t][h], K_i[tau][g]>            tau = 0 .. p
 *     out[t][h] = sum_tau softmax(z)_tau * V_i[tau][g]
 * where K_i[tau] = k_cache[block_tables[i][tau / 16]][tau % 16] (V alike).
 * Block-table entries past ceil(n / 16) and cache rows past n are never read.
 * Arithmetic: bf16 operands, fp32 accumulation and online softmax, output
 * rounded to bf16 (round to nearest even).  The new tokens are read from the
 * cache, so pa_reshape_and_cache for this step must be queued first.
 *   d_q             device [T][Hq][D] bf16
 *   d_k_cache/d_v_cache  device [NB][16][Hkv][D] bf16
 *   d_block_tables  device [S][MB] int32
 *   d_cu_seqlens_q  device [S+1] int32, equal to the host copy given to plan
 *   d_seq_lens      device [S] int32, equal to the host copy given to plan
 *   scale           softmax scale (usually 1/sqrt(D))
 *   d_out           device [T][Hq][D] bf16, written
 *   plan            from pa_plan_build with the same dims
 *   d_workspace     device scratch of pa_plan_workspace_bytes(plan) bytes,
 *                   256-byte aligned: a status word (zero-fill it before
 *                   first use), then scratch with no initial value (split
 *                   partials, staged K/V tiles of prefill segments).  Calls
 *                   with different plans may share a workspace.  Two calls
 *                   in flight at once need two workspaces.
 * After a call that reported an error, rebuild the plan (its merge tickets
 * may be left taken) and reset the workspace's status word.
 * The call queues its kernels on `stream` and nothing else (the plan's tables
 * are on the device since its build returned); nothing is copied from the
 * host.  It may be captured into a CUDA graph (stream capture in any mode):
 * a captured call does not record the plan's use, so a plan must not be
 * rebuilt or destroyed while a graph replay that uses it may run, and
 * replays that use one plan must not overlap; the first call on a device
 * (which sets kernel attributes) belongs before the capture, as a warm-up.
 * The decode kernel is launched with programmatic stream serialization: its
 * blocks may start while the kernel queued before it on
 * `stream` is still running, read only the plan's tables until that kernel
 * has completed (griddepcontrol.wait), and then everything else.  Stream
 * order is therefore kept for all caller data.
 * Errors: PA_ERR_NULL, PA_ERR_SHAPE, PA_ERR_ALIGN, PA_ERR_UNSUPPORTED,
 * PA_ERR_PLAN, PA_ERR_WORKSPACE, PA_ERR_CUDA.
 */
int pa_attention_varlen(const void *d_q, const void *d_k_cache, const void *d_v_cache,
                        const int32_t *d_block_tables, const int32_t *d_cu_seqlens_q,
                        const int32_t *d_seq_lens, float scale, void *d_out,
                        const pa_dims *dims, const pa_plan *plan, void *d_workspace,
                        size_t workspace_bytes, void *stream);

/*
 * pa_attention_varlen with optional tracing: when `trace` is not NULL, each
 * non-NULL entry of trace->events (a cudaEvent_t created by the caller) is
 * recorded on `stream` at a fixed point of the call, so that the caller can
 * time every kernel on the stream it runs on:
 *   [0] at the start of the call
 *   [1] before the split-KV decode kernel (which also merges split rows)
 *   [2] after the split-KV kernel      [3] = [2] (no separate combine kernel)
 *   [4] after the K/V staging kernel, before the prefill kernel
 *   [5] after the prefill kernel
 * When the kernels run one after the other, the staging kernel runs between
 * [3] and [4].
 * When the plan runs the two kernels side by side (pa_plan_info
 * num_prefill_ctas below the SM count while decode units exist), [1]-[3]
 * are recorded on the side stream that runs the decode kernel and [4], [5]
 * on `stream`, so both intervals measure their own kernel.
 * Events of stages that do not run are still recorded (adjacent), so every
 * interval is defined.  Results are identical to pa_attention_varlen.
 */
typedef struct {
    void *events[6];
} pa_trace;
int pa_attention_varlen_ex(const void *d_q, const void *d_k_cache, const void *d_v_cache,
                           const int32_t *d_block_tables, const int32_t *d_cu_seqlens_q,
                           const int32_t *d_seq_lens, float scale, void *d_out,
                           const pa_dims *dims, const pa_plan *plan, void *d_workspace,
                           size_t workspace_bytes, void *stream, const pa_trace *trace);

/*
 * One forward step's cache write and attention in one call: the work of
 * pa_reshape_and_cache(d_k, d_v, d_slot_mapping, ...) followed by
 * pa_attention_varlen(...), with the same arguments, outputs and errors
 * (the caches are written exactly as pa_reshape_and_cache writes them; out
 * equals pa_attention_varlen's bit for bit).  Cache write and attention
 * overlap: the decode kernel starts behind the scatter kernel by
 * programmatic launch and reads the keys of this step's own tokens from
 * d_k / d_v instead of their cache slots, and the gather of the long
 * segments' keys for the prefill kernel runs in the scatter's launch, taking
 * those keys from d_k / d_v as well (the two-SM prefill kernel reads key
 * tiles of only this step's tokens from d_k / d_v directly, and starts
 * behind the scatter when nothing else is gathered; when it runs beside the
 * decode kernel with nothing gathered, neither attention kernel reads the
 * slots the scatter writes, and the scatter is queued after them instead,
 * running beside the decode kernel) ("vLLM 学习笔记 01" §1.6: each new
 * token's K/V go to the slot its slot mapping names, and attention reads
 * them there; here attention takes the same values before they land).
 * Everything queued on the stream after the call follows all of its
 * kernels, whichever order they run in.
 * Precondition (besides those of both calls): every token t of segment i at
 * position p = seq_len - q_len + j has slot_mapping[t] ==
 * block_tables[i][p / 16] * 16 + p % 16, i.e. the slot mapping and the block
 * tables describe the same cache positions.
 *   d_k, d_v         device [T][Hkv][D] bf16: this step's K/V, read
 *   d_slot_mapping   device [T] int64
 *   the rest         as pa_attention_varlen; d_k_cache / d_v_cache written
 * Checks of both calls run before anything is queued.
 */
int pa_reshape_and_attention(const void *d_k, const void *d_v, const int64_t *d_slot_mapping,
                             const void *d_q, void *d_k_cache, void *d_v_cache,
                             const int32_t *d_block_tables, const int32_t *d_cu_seqlens_q,
                             const int32_t *d_seq_lens, float scale, void *d_out, const pa_dims *dims,
                             const pa_plan *plan, void *d_workspace, size_t workspace_bytes,
                             void *stream);

/*
 * Status word of a workspace: waits for `stream`, then copies the word to
 * *status.  0 means no error; bit 0 means some wait inside a kernel gave up
 * after about a second (the kernels never block longer, and the affected
 * outputs are undefined).  Error bits accumulate over the calls that used
 * the workspace until pa_workspace_reset clears them.
 */
int pa_workspace_status(const void *d_workspace, void *stream, uint32_t *status);

/*
 * Zeroes the status word of a workspace (a memset queued on `stream`);
 * `plan` is any plan the workspace serves.  Needed only after a call whose
 * status reported an error.
 * Errors: PA_ERR_NULL, PA_ERR_WORKSPACE (not 256-byte aligned), PA_ERR_CUDA.
 */
int pa_workspace_reset(void *d_workspace, const pa_plan *plan, void *stream);

/*
 * KV export and import ("vLLM 学习笔记 01" §2.5, prefill/decode
 * disaggregation: a prefill instance produces a request's full KV cache and
 * a connector carries it to a decode instance, which needs it in its own
 * pool).  Export gathers the K/V of S requests from the paged cache into
 * contiguous buffers; import writes such buffers into a pool through
 * (possibly other) block tables.  Only the local device half: moving the
 * buffers between instances is outside the library.
 * Token p of request i (0 <= p < n_i = cu_tokens[i + 1] - cu_tokens[i]) is
 * row cu_tokens[i] + p of the buffers and row p % 16 of cache block
 * block_tables[i][p / 16].  Bit-for-bit copies; nothing else is touched.
 *   d_k_cache, d_v_cache  device [NB][16][Hkv][D] bf16 (read by export,
 *                         written by import)
 *   d_block_tables        device [S][MB] int32
 *   d_cu_tokens           device [S+1] int32: 0, non-decreasing, ends at N
 *   d_k_out/d_v_out (export), d_k_in/d_v_in (import)  device [N][Hkv][D] bf16
 *   dims                  host; num_tokens = N, num_seqs = S, num_kv_heads,
 *                         head_dim, num_blocks, max_blocks_per_seq,
 *                         block_size (16) are used
 * Preconditions (not checked on the host): n_i <= MB * 16 and every table
 * entry a request's tokens use is inside the pool; rows that break them are
 * skipped without any access.  Import into slots another request also uses
 * is undefined.  N == 0 queues nothing.
 * Errors: PA_ERR_NULL, PA_ERR_SHAPE, PA_ERR_ALIGN, PA_ERR_UNSUPPORTED,
 * PA_ERR_CUDA.
 */
int pa_kv_export(const void *d_k_cache, const void *d_v_cache, const int32_t *d_block_tables,
                 const int32_t *d_cu_tokens, void *d_k_out, void *d_v_out, const pa_dims *dims,
                 void *stream);
int pa_kv_import(const void *d_k_in, const void *d_v_in, const int32_t *d_block_tables,
                 const int32_t *d_cu_tokens, void *d_k_cache, void *d_v_cache, const pa_dims *dims,
                 void *stream);

/*
 * Opt-in check of the data-dependent preconditions, on the device, then a
 * synchronize of `stream`: every slot_mapping entry is negative or inside the
 * pool; no two tokens share a slot; cu_seqlens_q starts at 0, is
 * non-decreasing and ends at T; 0 <= q_len <= seq_len; seq_len <= MB * 16;
 * every block-table entry a segment reads (the first ceil(seq_len / 16)) is
 * inside the pool.  d_slot_mapping may be NULL to skip the slot checks.
 * Returns PA_OK, PA_ERR_BOUNDS, or a host-side error as above.
 *   d_scratch  device, at least pa_validate_scratch_bytes(dims) bytes,
 *              256-byte aligned (overwritten).
 */
size_t pa_validate_scratch_bytes(const pa_dims *dims);
int pa_validate_inputs(const int64_t *d_slot_mapping, const int32_t *d_block_tables,
                       const int32_t *d_cu_seqlens_q, const int32_t *d_seq_lens,
                       const pa_dims *dims, void *d_scratch, size_t scratch_bytes,
                       void *stream);

/*
 * pa_attention_varlen_noalloc — the same computation as pa_attention_varlen,
 * for callers that cannot allocate device memory.  The pages have no
 * counterpart of this call: it exists for callers such as an engine that has
 * given nearly all GPU memory to its KV pool and keeps no allocator in its
 * step loop, a host or plugin interface that hands an op only its inputs,
 * outputs and a stream, or a loop that must avoid the device-wide stalls a
 * cudaMalloc/cudaFree pair can cause.
 *
 * Instead of a caller workspace it uses one fixed array of
 * pa_noalloc_scratch_bytes() (16 MiB) in the library's device memory.  Every
 * GPU that loads libpa.so holds that array until the process exits.  The call
 * allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - Arguments and results are those of pa_attention_varlen, minus
 *     d_workspace / workspace_bytes.
 *   - A plan whose pa_plan_workspace_bytes exceeds the array is rejected with
 *     PA_ERR_TOO_LARGE before any work is queued.
 *   - The first call on each device (with that device current) looks up the
 *     array's device address with cudaGetSymbolAddress and caches it; make
 *     that first call before any stream capture.  A failed lookup returns
 *     PA_ERR_CUDA.
 *   - The address is looked up again when the device's current CUDA context
 *     is another one than at the lookup (after cudaDeviceReset, say, the
 *     library's device image is loaded anew); the first call in a new
 *     context must then also come before any stream capture.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents.  Its first word is a status word like a workspace's (zero
 *     at load; the kernels only ever set error bits in it, which
 *     accumulate until cleared): read and clear it with pa_noalloc_status.
 *     The rest is scratch that every call writes before reading; the plan's
 *     tables live with the plan.  Calls whose GPU work overlaps in time (two
 *     streams, or two threads' streams) race on the array and give
 *     undefined results; order them, or use pa_attention_varlen with
 *     separate workspaces.
 */
size_t pa_noalloc_scratch_bytes(void);
int pa_attention_varlen_noalloc(const void *d_q, const void *d_k_cache, const void *d_v_cache,
                                const int32_t *d_block_tables, const int32_t *d_cu_seqlens_q,
                                const int32_t *d_seq_lens, float scale, void *d_out,
                                const pa_dims *dims, const pa_plan *plan, void *stream);

/*
 * Status word of the no-alloc array on the current device, the counterpart
 * of pa_workspace_status for pa_attention_varlen_noalloc: copies the word to
 * *status after the work queued on `stream` before it (the call waits for
 * `stream`), and with clear != 0 then zeroes it (queued on `stream`, done
 * before the call returns).  0 means no error; bit 0 means some bounded wait
 * inside a kernel of a no-alloc call gave up (that call's output is
 * undefined).  Allocates nothing.  Like the no-alloc call itself, it races
 * with no-alloc work queued on other streams.
 * Errors: PA_ERR_NULL, PA_ERR_CUDA.
 */
int pa_noalloc_status(uint32_t *status, int clear, void *stream);

/*
 * Self-test of the bounded-wait error path.  Every mbarrier wait in the
 * tensor-core kernels gives up after a limit (about a second) and sets bit 0
 * of the status word; this call makes such a wait run out on purpose, with
 * nothing else in flight: it queues on `stream` a one-CTA kernel that holds
 * tensor memory, waits limit_cycles SM cycles on an mbarrier that nothing
 * arrives at, sets bit 0 of the word at d_workspace (a workspace or any
 * 256-byte aligned device word) and releases the tensor memory.  Read the
 * result with pa_workspace_status and clear it with pa_workspace_reset.
 * The pages have no counterpart: it checks the library's failure reporting.
 * Errors: PA_ERR_NULL, PA_ERR_WORKSPACE (misaligned), PA_ERR_SHAPE
 * (limit_cycles outside 1 .. 2e9), PA_ERR_CUDA.
 */
int pa_selftest_wait_timeout(void *d_workspace, long long limit_cycles, void *stream);

/* Static text for a status code. */
const char *pa_status_string(int status);

/* Library version, e.g. "0.1.0". */
const char *pa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PA_H */
