// Host work partitioner: cu_seqlens_q + seq_lens (host copies) -> balanced GPU
// work.  Pure host code; it queues no GPU work.
//
// Decode side (segments with q_len <= kDecodeMaxQLen): every query token of
// such a segment, for every kv head, is a "row" that reads its p + 1 keys
// ("vLLM 学习笔记 01" §1.4/§1.6: the segment's seq_len counts this step's
// tokens, query j sits at position seq_len - q_len + j).  The rows' 16-token
// KV blocks are laid end to end and cut into equal runs, one run per warp
// (split-KV in the flash-decoding manner, balanced like stream-K), so every
// warp moves the same number of KV bytes whatever the length mix.  A row cut
// across several runs leaves one partial (unnormalised O, running max and
// sum) per run; the last run to finish merges them (see CombineRow).
//
// Prefill side (longer segments): 128-query tiles for pairs of query heads
// that share a kv head, dealt to at most one persistent CTA per SM by
// greedy longest-processing-time assignment (each tile, longest first, goes
// to the CTA with the least work so far; a tile costs its 128-key tiles plus
// a fixed start/finish overhead); and, per segment and kv head, the list of
// 128-key tiles of K/V that a gather kernel stages from the paged cache into
// the workspace for them.
#include <algorithm>
#include <cstdlib>
#include <functional>
#include <queue>
#include <utility>
#include <cstring>
#include <new>

#include <cuda_runtime.h>

#include "plan.h"

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Start/finish cost of a prefill tile in units of 128-key steps (Q load,
// first S, output write-back), for the CTA assignment and the side-by-side
// split.  Shared-prefix tiles are short (a few steps) and write fp32
// partials; beside the decode kernel they cost more (B200 sweep of the
// shared-prefix workload: 8 steps beat 2, 16, 24 and running serially).
constexpr int64_t kTileOverheadSteps = 2;
constexpr int64_t kPrefixTileOverheadSteps = 8;

int64_t tile_cost(const pa::PrefillTile &t) {
    return t.n_kv_tiles + (t.row_base >= 0 ? kPrefixTileOverheadSteps : kTileOverheadSteps);
}

// Fewest KV blocks one decode warp is given, so that its fixed costs (loading
// q, the final write or merge) stay small against the streaming.
constexpr int64_t kMinBlocksPerUnit = 4;

// Cost, in blocks, charged at the end of every decode row when runs are cut:
// finishing a row (the output write, or a partial, its ticket and often the
// merge) and starting the next (its q) take about as long as streaming this
// many blocks, so a run that crosses a row boundary gets fewer blocks.
constexpr int64_t kRowCostBlocks = 8;
// The same charge where runs are long (kLongRunBlocks blocks or more on
// average): there a row's finish overlaps more of the run's streaming.
// B200, fused steps: 256 requests of Llama-3-8B shape (~300 blocks per run)
// 425.6-426.7 us with 4 against 429.6-431.2 with 8 (6: 429.0); 64 requests
// of TinyLlama shape (~15 blocks per run) 23.6 us with 8 against 25.6 with
// 4 (12-24: 23.6-24.0).  The threshold lies between the two.
constexpr int64_t kRowCostBlocksLongRuns = 4;
constexpr int64_t kLongRunBlocks = 64;

// Cost model for running the prefill kernel beside the decode kernel on
// disjoint SMs (B200 measurements): one 128-key step of a two-head tile
// takes a CTA (one SM) ~2.9 us when the prefill kernel has a part of the
// GPU (~3.5 us with all SMs); the decode kernel streams ~66 GB/s per SM
// up to ~6.1 TB/s of HBM bandwidth (reached from ~92 SMs on).
constexpr double kPrefillStepUs = 2.9;
// The same step of a two-head tile on a cluster of two SMs (the pair kernel:
// one head per SM, 2-SM MMAs), in microseconds of the cluster.  Measured on
// B200 at ~1.22 on long chunks beside the decode kernel; 1.15 is what the
// split is tuned with: on the 8192-token mixed step it gives the pair kernel
// 36 SMs (499 us per fused step) where 1.05-1.10 / 1.20 / 1.25 / 1.35 give
// 34 / 38 / 40 / 42 SMs (507 / 501 / 503 / 505 us), the decode kernel
// finishing last in every case.
constexpr double kPairStepUs = 1.15;
constexpr double kDecodeBytesPerUsPerSm = 66e3;
constexpr double kHbmBytesPerUs = 6.1e6;
constexpr int kMinSideSms = 8;  // fewest SMs either kernel is given when they share the GPU

// Shared-prefix (cascade) groups: runs of at least kMinGroupSegs consecutive
// single-token segments whose first kMinSharedBlocks or more block-table
// entries are the same physical blocks.
constexpr int kMinGroupSegs = 4;
constexpr int kMinSharedBlocks = 16;

struct PrefixGroup {
    int seg0, nseg;  // segments seg0 .. seg0 + nseg - 1
    int blocks;      // shared leading blocks
};

// Groups of consecutive single-token segments that share their leading
// blocks; each query sits past the shared keys, so all of them see all of
// them.
std::vector<PrefixGroup> find_prefix_groups(const int32_t *h_cu, const int32_t *h_seq, const int32_t *h_bt,
                                            const pa_dims &d) {
    std::vector<PrefixGroup> groups;
    if (!h_bt) return groups;
    const int S = d.num_seqs, MB = d.max_blocks_per_seq;
    auto single = [&](int i) { return h_cu[i + 1] - h_cu[i] == 1; };
    int i = 0;
    while (i < S) {
        if (!single(i) || h_seq[i] < 2) {
            ++i;
            continue;
        }
        const int32_t *bi = h_bt + (size_t)i * MB;
        int c = (h_seq[i] - 1) / pa::kBlockSize;  // blocks wholly before the query's own key
        int j = i + 1;
        while (j < S && single(j) && h_seq[j] >= 2) {
            const int32_t *bj = h_bt + (size_t)j * MB;
            const int cap = std::min(c, (h_seq[j] - 1) / pa::kBlockSize);
            int k = 0;
            while (k < cap && bj[k] == bi[k]) ++k;
            if (k < kMinSharedBlocks) break;
            c = k;
            ++j;
        }
        if (j - i >= kMinGroupSegs && c >= kMinSharedBlocks) {
            groups.push_back({i, j - i, c});
            i = j;
        } else {
            ++i;
        }
    }
    return groups;
}

// SMs for the prefill kernel when it runs beside the decode kernel, or 0 when
// running them one after the other is predicted to be as fast.
int overlap_split(int num_sms, int64_t prefill_steps, int64_t decode_bytes, double step_sm_us) {
    if (prefill_steps <= 0 || decode_bytes <= 0 || num_sms < 2 * kMinSideSms) return 0;
    auto decode_us = [&](int sms) {
        return (double)decode_bytes / std::min(kHbmBytesPerUs, sms * kDecodeBytesPerUsPerSm);
    };
    const double serial = prefill_steps * step_sm_us / num_sms + decode_us(num_sms);
    double best = serial;
    int best_p = 0;
    for (int s = kMinSideSms; s <= num_sms - kMinSideSms; ++s) {
        const double t = std::max(prefill_steps * step_sm_us / s, decode_us(num_sms - s));
        if (t < best) {
            best = t;
            best_p = s;
        }
    }
    return best_p;
}

// Key splits of the shared prefixes and SMs of the prefill kernel beside the
// decode kernel, chosen together for plans with shared-prefix groups.  Each
// group's prefix tiles (chunks x kv heads x head pairs x splits) cost their
// 128-key tiles plus kPrefixTileOverheadSteps each and are nearly uniform, so
// dealt to s persistent CTAs they take ceil(tiles / s) tiles' time; other
// prefill tiles add their average load and one largest tile.  The decode side
// is costed in the blocks its runs stream plus kRowCostBlocks per row (the
// charge the run partition uses).  Picks the fastest (splits, SMs), the
// fewest splits among equals; B200, shared-prefix workload: 2 splits on 64
// SMs beat 4 on 78 (the old choice; 128 tiles left half the CTAs with two),
// 2 on 52 or 58, 3, and 1.
struct CascadeChoice {
    int splits = 1;
    int sms = 0;  // 0: the two kernels run one after the other
};

CascadeChoice choose_cascade(int num_sms, int G, int Hkv, const std::vector<PrefixGroup> &groups,
                             int64_t other_total, int64_t other_max, int64_t decode_cost_bytes, bool pair) {
    CascadeChoice best;
    double best_us = 1e30;
    int nt_min = INT32_MAX;
    for (const PrefixGroup &g : groups) nt_min = std::min<int>(nt_min, (int)cdiv(g.blocks * pa::kBlockSize, pa::kPrefillTileN));
    auto decode_us = [&](int sms) {
        return sms <= 0 ? 1e30 : (double)decode_cost_bytes / std::min(kHbmBytesPerUs, sms * kDecodeBytesPerUsPerSm);
    };
    for (int sp : {1, 2, 3, 4, 6, 8}) {
        if (sp > nt_min) break;
        int64_t tiles = 0, cost = 0;  // prefix tiles and the largest one's cost
        for (const PrefixGroup &g : groups) {
            const int64_t nt = cdiv(g.blocks * pa::kBlockSize, pa::kPrefillTileN);
            tiles += cdiv(g.nseg, pa::kPrefillTileM) * Hkv * cdiv(G, 2) * sp;
            cost = std::max<int64_t>(cost, cdiv(nt, sp) + kPrefixTileOverheadSteps);
        }
        // s SMs hold s persistent CTAs, or s / 2 clusters with the pair kernel
        auto prefill_us = [&](int s) {
            const int slots = pair ? s / 2 : s;
            if (slots < 1) return 1e30;
            double units = (double)cdiv(tiles, slots) * cost;
            if (other_total > 0) units += (double)other_total / slots + (double)other_max;
            return units * (pair ? kPairStepUs : kPrefillStepUs);
        };
        // one after the other, on every SM
        double t = prefill_us(num_sms) + decode_us(num_sms);
        if (t < best_us) {
            best_us = t;
            best = {sp, 0};
        }
        for (int s = kMinSideSms; s <= num_sms - kMinSideSms; s += pair ? 2 : 1) {
            t = std::max(prefill_us(s), decode_us(num_sms - s));
            if (t < best_us) {
                best_us = t;
                best = {sp, s};
            }
        }
    }
    return best;
}

// Scoped switch to the plan's device (plans own device memory, a stream and
// events, which belong to the device they were made on).
struct DeviceScope {
    int prev = -1;
    explicit DeviceScope(int device) {
        if (device < 0) return;
        cudaGetDevice(&prev);
        if (prev != device) cudaSetDevice(device);
    }
    ~DeviceScope() {
        int cur = -1;
        cudaGetDevice(&cur);
        if (prev >= 0 && cur != prev) cudaSetDevice(prev);
    }
};

// Waits until the plan's last upload has executed and the last attention
// call that read its tables has finished.
void wait_idle(const pa_plan *p) {
    if (p->upload_event) cudaEventSynchronize(static_cast<cudaEvent_t>(p->upload_event));
    if (p->use_event) cudaEventSynchronize(static_cast<cudaEvent_t>(p->use_event));
}

void free_tables(pa_plan *p) {
    if (!p->tables) return;
    if (p->tables_pinned)
        cudaFreeHost(p->tables);
    else
        std::free(p->tables);
    p->tables = nullptr;
    p->tables_capacity = 0;
    p->tables_pinned = false;
}

// Host buffer of at least `bytes` for the plan tables: page-locked when the
// plan has a device, ordinary memory otherwise (host-only use, tests).
bool reserve_tables(pa_plan *p, size_t bytes) {
    if (p->tables && p->tables_capacity >= bytes) return true;
    free_tables(p);
    const size_t cap = std::max<size_t>(bytes, 4096);
    if (p->device >= 0) {
        int prev = -1;
        cudaGetDevice(&prev);
        if (prev != p->device) cudaSetDevice(p->device);
        void *h = nullptr;
        if (cudaHostAlloc(&h, cap, cudaHostAllocPortable) == cudaSuccess) {
            p->tables = static_cast<uint8_t *>(h);
            p->tables_pinned = true;
        } else {
            cudaGetLastError();
        }
        if (prev >= 0 && prev != p->device) cudaSetDevice(prev);
    }
    if (!p->tables) {
        p->tables = static_cast<uint8_t *>(std::malloc(cap));
        if (!p->tables) return false;
    }
    p->tables_capacity = cap;
    return true;
}

// Stream and events of a plan with a device (created once).
bool create_sync_objects(pa_plan *p) {
    if (p->device < 0) return true;
    if (p->upload_stream && p->upload_event && p->use_event) return true;
    DeviceScope scope(p->device);
    if (!p->upload_stream) {
        cudaStream_t s = nullptr;
        if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return false;
        p->upload_stream = s;
    }
    for (void **slot : {&p->upload_event, &p->use_event, &p->fork_event, &p->join_event}) {
        if (*slot) continue;
        cudaEvent_t e = nullptr;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
        *slot = e;
    }
    return true;
}

// Copies the host image of the tables to the plan's device buffer on the
// plan's stream and waits for the copy (the caller has waited for the plan
// to be idle).
bool upload_tables(pa_plan *p) {
    if (p->device < 0) return true;
    DeviceScope scope(p->device);
    const size_t bytes = p->tl.bytes;
    if (p->d_capacity < bytes) {
        if (p->d_tables) cudaFree(p->d_tables);
        p->d_tables = nullptr;
        p->d_capacity = 0;
        const size_t cap = std::max<size_t>(bytes, 4096);
        void *d = nullptr;
        if (cudaMalloc(&d, cap) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        p->d_tables = d;
        p->d_capacity = cap;
    }
    cudaStream_t s = static_cast<cudaStream_t>(p->upload_stream);
    if (cudaMemcpyAsync(p->d_tables, p->tables, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return false;
    // the build returns with the tables on the device: attention calls then
    // queue no wait for them (and can be captured into a CUDA graph)
    if (cudaEventRecord(static_cast<cudaEvent_t>(p->upload_event), s) != cudaSuccess) return false;
    return cudaEventSynchronize(static_cast<cudaEvent_t>(p->upload_event)) == cudaSuccess;
}

int check_dims(const pa_dims *d) {
    if (!d) return PA_ERR_NULL;
    if (d->num_tokens < 0 || d->num_seqs < 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0 ||
        d->head_dim <= 0 || d->num_blocks <= 0 || d->max_blocks_per_seq < 0 || d->block_size <= 0)
        return PA_ERR_SHAPE;
    if (d->num_q_heads % d->num_kv_heads != 0) return PA_ERR_SHAPE;
    if (d->block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
    if (d->head_dim != 64 && d->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (d->num_q_heads / d->num_kv_heads > 16) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

}  // namespace

extern "C" int pa_plan_build(const int32_t *h_cu, const int32_t *h_seq, const int32_t *h_bt,
                             const pa_dims *dims, int device, pa_plan **out) {
    if (!out) return PA_ERR_NULL;
    int st = check_dims(dims);
    if (st != PA_OK) return st;
    const pa_dims d = *dims;
    if (d.num_seqs > 0 && (!h_cu || !h_seq)) return PA_ERR_NULL;
    if (d.num_seqs == 0 && d.num_tokens != 0) return PA_ERR_SHAPE;
    if (d.num_seqs > 0) {
        if (h_cu[0] != 0 || h_cu[d.num_seqs] != d.num_tokens) return PA_ERR_SHAPE;
        for (int i = 0; i < d.num_seqs; ++i) {
            const int64_t L = (int64_t)h_cu[i + 1] - h_cu[i];
            if (L < 0 || h_seq[i] < L) return PA_ERR_SHAPE;
            if (L > 0 && cdiv(h_seq[i], pa::kBlockSize) > d.max_blocks_per_seq) return PA_ERR_SHAPE;
        }
    }

    pa_plan *p = *out;
    const bool fresh = (p == nullptr);
    if (fresh) {
        p = new (std::nothrow) pa_plan();
        if (!p) return pa::cuda_error();
        p->device = device;
        if (!create_sync_objects(p)) {
            cudaGetLastError();
            pa_plan_destroy(p);
            return pa::cuda_error();
        }
    } else if (p->device != device) {
        return PA_ERR_PLAN;
    }
    p->dims = d;
    p->group = d.num_q_heads / d.num_kv_heads;
    p->num_sms = device >= 0 ? pa::device_sm_count(device) : 148;
    p->prefill_pairs = 0;
    const int Hkv = d.num_kv_heads;

    const int G = d.num_q_heads / d.num_kv_heads;
    std::vector<pa::DecodeRow> rows;
    std::vector<pa::PrefillTile> tiles;
    std::vector<pa::StageTile> stages;
    // shared prefixes: the prefill kernel attends each group's tokens to the
    // shared blocks (key splits of them, as partials); the decode rows read
    // only the blocks after them
    const std::vector<PrefixGroup> groups =
        pa::prefill_kernel_available() ? find_prefix_groups(h_cu, h_seq, h_bt, d) : std::vector<PrefixGroup>();
    std::vector<int> shared(d.num_seqs, 0), group_of(d.num_seqs, -1), seg_row0(d.num_seqs, -1);
    for (size_t k = 0; k < groups.size(); ++k)
        for (int i = groups[k].seg0; i < groups[k].seg0 + groups[k].nseg; ++i) {
            shared[i] = groups[k].blocks;
            group_of[i] = (int)k;
        }
    std::vector<int> group_splits(groups.size(), 0);
    {
        size_t decode_tokens = 0;  // rows are made for the decode segments only
        for (int i = 0; i < d.num_seqs; ++i) {
            const int L = h_cu[i + 1] - h_cu[i];
            if (L > 0 && (L <= pa::kDecodeMaxQLen || !pa::prefill_kernel_available())) decode_tokens += (size_t)L;
        }
        rows.reserve(decode_tokens * Hkv);
    }
    for (int i = 0; i < d.num_seqs; ++i) {
        const int L = h_cu[i + 1] - h_cu[i];
        const int n = h_seq[i];
        if (L == 0) continue;
        if (L <= pa::kDecodeMaxQLen || !pa::prefill_kernel_available()) {
            seg_row0[i] = (int)rows.size();
            for (int j = 0; j < L; ++j)
                for (int g = 0; g < Hkv; ++g)
                    rows.push_back({h_cu[i] + j, i, n - L + j + 1, pa::kUnsplitRow, -1, shared[i], j + 1, 0});
        } else {
            const int nt = (int)cdiv(n, pa::kPrefillTileN);  // key tiles of the segment
            const int base = (int)stages.size();
            for (int g = 0; g < Hkv; ++g)
                for (int j = 0; j < nt; ++j) stages.push_back({i, g, j, n});
            for (int q0 = 0; q0 < L; q0 += pa::kPrefillTileM) {
                const int last = std::min(L, q0 + pa::kPrefillTileM) - 1;
                const int kv_tiles = (int)cdiv(n - L + last + 1, pa::kPrefillTileN);
                for (int g = 0; g < Hkv; ++g)
                    for (int h = g * G; h < (g + 1) * G; h += 2)
                        tiles.push_back({i, q0, h, kv_tiles, std::min(2, (g + 1) * G - h), base + g * nt, 0, 0,
                                         -1, 0, 0, 0});
            }
            for (int j = 0; j < L; ++j) p->prefill_pairs += n - L + j + 1;
        }
    }
    // Shared-prefix tiles: per group, chunk of up to 128 tokens, kv head,
    // query-head pair and key split, with the splits (and the SMs the
    // prefill kernel gets beside the decode kernel) chosen by
    // choose_cascade.
    // The pair kernel takes a tile's two heads on a cluster of two SMs; it
    // serves plans whose every tile has two heads (an even group size) at
    // head_dim 128.
    bool pair = pa::prefill_kernel_available() && G % 2 == 0 && d.head_dim == 128;
    for (const pa::PrefillTile &t : tiles) pair = pair && t.num_heads == 2;
    CascadeChoice cascade_choice;
    if (!groups.empty()) {
        int64_t other_total = 0, other_max = 0;
        for (const pa::PrefillTile &t : tiles) {
            other_total += tile_cost(t);
            other_max = std::max(other_max, tile_cost(t));
        }
        int64_t decode_cost_blocks = 0;
        for (const pa::DecodeRow &r : rows)
            decode_cost_blocks += cdiv(r.n_keys, pa::kBlockSize) - r.first_block + kRowCostBlocks;
        cascade_choice = choose_cascade(p->num_sms, G, Hkv, groups, other_total, other_max,
                                        decode_cost_blocks * pa::kBlockSize * d.head_dim * 2 * 2, pair);
    }
    // key tiles of the prefill segments: the staging list's head; a shared
    // prefix's tiles follow (the pair kernel reads those from the paged cache)
    const size_t seg_stages = stages.size();
    for (size_t k = 0; k < groups.size(); ++k) {
        const PrefixGroup &gr = groups[k];
        const int keys = gr.blocks * pa::kBlockSize;
        const int nt = (int)cdiv(keys, pa::kPrefillTileN);
        const int chunks = (int)cdiv(gr.nseg, pa::kPrefillTileM);
        const int splits = std::min(cascade_choice.splits, nt);
        group_splits[k] = splits;
        const int base = (int)stages.size();
        for (int g = 0; g < Hkv; ++g)
            for (int j = 0; j < nt; ++j) stages.push_back({gr.seg0, g, j, keys});
        for (int c = 0; c < chunks; ++c) {
            const int s0 = gr.seg0 + c * pa::kPrefillTileM;
            const int q_rows = std::min(pa::kPrefillTileM, gr.seg0 + gr.nseg - s0);
            for (int g = 0; g < Hkv; ++g)
                for (int h = g * G; h < (g + 1) * G; h += 2)
                    for (int sp = 0; sp < splits; ++sp) {
                        const int t0 = (int)((int64_t)nt * sp / splits), t1 = (int)((int64_t)nt * (sp + 1) / splits);
                        tiles.push_back({gr.seg0, h_cu[s0], h, t1 - t0, std::min(2, (g + 1) * G - h), base + g * nt,
                                         t0, keys, seg_row0[s0] + g, sp, q_rows, 0});
                    }
        }
        p->prefill_pairs += (int64_t)gr.nseg * keys;
    }
    std::stable_sort(tiles.begin(), tiles.end(),
                     [](const pa::PrefillTile &a, const pa::PrefillTile &b) { return tile_cost(a) > tile_cost(b); });
    // Deal the tiles to persistent CTAs; each CTA's tiles become contiguous.
    // Decode KV bytes and prefill steps decide whether the two kernels share
    // the GPU side by side, and on how many SMs each runs.
    int64_t decode_blocks_all = 0;
    for (const pa::DecodeRow &r : rows) decode_blocks_all += cdiv(r.n_keys, pa::kBlockSize) - r.first_block;
    int64_t prefill_steps = 0;
    for (const pa::PrefillTile &t : tiles) prefill_steps += tile_cost(t);
    // With shared prefixes the decode rows merge partials of the prefill
    // kernel: the decode kernel follows it, or runs beside it and leaves all
    // merging to a merge kernel after both.
    p->cascade = !groups.empty();
    p->num_prefix_groups = (int32_t)groups.size();
    p->prefill_pair = pair && !tiles.empty();
    p->overlap_sms = groups.empty()
                         ? overlap_split(p->num_sms, prefill_steps, decode_blocks_all * pa::kBlockSize * d.head_dim * 2 * 2,
                                         p->prefill_pair ? 2 * kPairStepUs : kPrefillStepUs)
                         : cascade_choice.sms;
    if (p->prefill_pair) p->overlap_sms &= ~1;  // whole SM pairs
    const int prefill_sms = p->overlap_sms > 0 ? p->overlap_sms : p->num_sms;
    const int decode_sms = p->num_sms - p->overlap_sms;
    // persistent CTAs, or with the pair kernel clusters of two, one per tile slot
    const int grid = (int)std::min<size_t>(tiles.size(), (size_t)(p->prefill_pair ? prefill_sms / 2 : prefill_sms));
    std::vector<int32_t> cta_start(grid + 1, 0);
    if (grid > 0) {
        std::vector<std::vector<int32_t>> per(grid);
        using Load = std::pair<int64_t, int>;
        std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
        for (int c = 0; c < grid; ++c) heap.push({0, c});
        for (size_t t = 0; t < tiles.size(); ++t) {
            Load l = heap.top();
            heap.pop();
            per[l.second].push_back((int32_t)t);
            l.first += tile_cost(tiles[t]);
            heap.push(l);
        }
        std::vector<pa::PrefillTile> dealt;
        dealt.reserve(tiles.size());
        for (int c = 0; c < grid; ++c) {
            cta_start[c] = (int32_t)dealt.size();
            for (int32_t t : per[c]) dealt.push_back(tiles[t]);
        }
        cta_start[grid] = (int32_t)dealt.size();
        tiles.swap(dealt);
    }

    // Cut the decode rows' blocks into equal runs of cost: each row's
    // blocks, then the per-row charge of virtual cost, laid end to end.
    const int64_t R = (int64_t)rows.size();
    std::vector<int64_t> prefix(R + 1, 0), nblocks(R, 0);
    int64_t total = 0;  // real blocks
    for (int64_t r = 0; r < R; ++r) {
        nblocks[r] = cdiv(rows[r].n_keys, pa::kBlockSize) - rows[r].first_block;
        total += nblocks[r];
    }
    int64_t P = 0;
    if (total > 0) {
        const int64_t max_units = (int64_t)decode_sms * pa::decode_units_per_sm(d.head_dim);
        P = std::max<int64_t>(1, std::min(max_units, cdiv(total, kMinBlocksPerUnit)));
    }
    const int64_t row_cost = P > 0 && total / P >= kLongRunBlocks ? kRowCostBlocksLongRuns : kRowCostBlocks;
    for (int64_t r = 0; r < R; ++r) prefix[r + 1] = prefix[r] + nblocks[r] + row_cost;
    const int64_t total_cost = prefix[R];
    std::vector<pa::DecodeUnit> units(P + 1);
    std::vector<int64_t> ustart(P + 1);
    {
        int64_t r = 0;
        // f = floor(total_cost * u / P), stepped without a division per unit
        const int64_t step = P ? total_cost / P : 0, rem = P ? total_cost % P : 0;
        int64_t f = 0, carry = 0;
        for (int64_t u = 0; u <= P; ++u) {
            if (u > 0) {
                f += step;
                carry += rem;
                if (carry >= P) {
                    ++f;
                    carry -= P;
                }
            }
            ustart[u] = f;
            while (r < R && prefix[r + 1] <= f) ++r;  // row whose cost span holds f
            int64_t rr = r, off = r < R ? f - prefix[r] : 0;
            if (rr < R && off >= nblocks[rr]) {  // in the row's virtual cost: start the next row
                ++rr;
                off = 0;
            }
            units[u] = {(int32_t)rr, (int32_t)off + (rr < R ? rows[rr].first_block : 0),
                        rr < R ? rows[rr].seq : 0, rr < R ? rows[rr].n_keys : 0,
                        rr < R ? rows[rr].token : 0, rr < R ? rows[rr].n_new : 0};
        }
        units[P] = {(int32_t)R, 0, 0, 0, 0, 0};
    }
    // Pieces: a row is split if its blocks span more than one unit.
    std::vector<pa::CombineRow> combine;
    combine.reserve((size_t)R);
    int32_t piece_base = 0;
    {
        int64_t u = 0;
        for (int64_t r = 0; r < R; ++r) {
            while (u + 1 < P && ustart[u + 1] <= prefix[r]) ++u;  // unit of the first block
            int64_t v = u;
            while (v + 1 < P && ustart[v + 1] <= prefix[r] + nblocks[r] - 1) ++v;  // unit of the last block
            const int32_t count = (int32_t)(v - u + 1);
            // partials of the row's shared prefix (written by the prefill
            // kernel) come first
            const int sg = group_of[rows[r].seq];
            const int32_t pre = sg >= 0 ? group_splits[sg] : 0;
            if (count > 1 || pre > 0) {
                rows[r].slot_base = piece_base + pre - (int32_t)u;
                rows[r].combine = (int32_t)combine.size();
                combine.push_back({(int32_t)r, piece_base, count + pre, count});
                piece_base += count + pre;
            }
        }
    }

    p->num_units = (int32_t)P;
    p->num_rows = (int32_t)R;
    p->num_pieces = piece_base;
    p->num_combine = (int32_t)combine.size();
    p->decode_blocks = total;
    p->decode_keys = 0;
    for (const pa::DecodeRow &r : rows) p->decode_keys += r.n_keys - (int64_t)r.first_block * pa::kBlockSize;
    p->num_tiles = (int32_t)tiles.size();
    p->num_prefill_ctas = p->prefill_pair ? 2 * grid : grid;
    // tiles the staging kernel gathers into the workspace (the list's head
    // with the pair kernel, all of it otherwise)
    p->num_stages = (int32_t)(p->prefill_pair ? seg_stages : stages.size());
    // a fused step with the pair kernel reads key tiles of the step's own
    // tokens from its K/V input: only tiles with earlier keys are staged
    p->num_stages_fused = 0;
    for (size_t i = 0; i < seg_stages; ++i) {
        const pa::StageTile &st = stages[i];
        const int L = h_cu[st.seq + 1] - h_cu[st.seq];
        if ((int64_t)pa::kPrefillTileN * st.tile < (int64_t)h_seq[st.seq] - L) ++p->num_stages_fused;
    }

    pa::TableLayout &t = p->tl;
    size_t off = 0;
    t.units = off;     off = align_up(off + sizeof(pa::DecodeUnit) * units.size(), pa::kWorkspaceAlign);
    t.rows = off;      off = align_up(off + sizeof(pa::DecodeRow) * rows.size(), pa::kWorkspaceAlign);
    t.combine = off;   off = align_up(off + sizeof(pa::CombineRow) * combine.size(), pa::kWorkspaceAlign);
    t.tiles = off;     off = align_up(off + sizeof(pa::PrefillTile) * tiles.size(), pa::kWorkspaceAlign);
    t.cta_start = off; off = align_up(off + sizeof(int32_t) * cta_start.size(), pa::kWorkspaceAlign);
    t.stages = off;    off = align_up(off + sizeof(pa::StageTile) * stages.size(), pa::kWorkspaceAlign);
    t.arrived = off;   off = align_up(off + sizeof(uint32_t) * combine.size(), pa::kWorkspaceAlign);
    t.bytes = off;

    pa::WorkspaceLayout &w = p->ws;
    off = 0;
    w.header = off;    off = pa::kHeaderBytes;
    w.partial_o = off;
    off = align_up(off + sizeof(float) * (size_t)piece_base * p->group * d.head_dim, pa::kWorkspaceAlign);
    w.partial_ml = off;
    off = align_up(off + sizeof(float) * 2 * (size_t)piece_base * p->group, pa::kWorkspaceAlign);
    off = align_up(off, pa::kStagedAlign);
    w.staged = off;
    off += (size_t)p->num_stages * 2 * (size_t)pa::kPrefillTileN * d.head_dim * 2;
    w.total = align_up(off, pa::kWorkspaceAlign);

    {
        DeviceScope scope(p->device);
        wait_idle(p);  // no queued copy reads the host image, no kernel the device tables
    }
    if (!reserve_tables(p, t.bytes)) {
        if (fresh) pa_plan_destroy(p);
        return pa::cuda_error();
    }
    std::memset(p->tables, 0, t.bytes);
    std::memcpy(p->tables + t.units, units.data(), sizeof(pa::DecodeUnit) * units.size());
    if (!rows.empty())
        std::memcpy(p->tables + t.rows, rows.data(), sizeof(pa::DecodeRow) * rows.size());
    if (!combine.empty())
        std::memcpy(p->tables + t.combine, combine.data(), sizeof(pa::CombineRow) * combine.size());
    if (!tiles.empty())
        std::memcpy(p->tables + t.tiles, tiles.data(), sizeof(pa::PrefillTile) * tiles.size());
    std::memcpy(p->tables + t.cta_start, cta_start.data(), sizeof(int32_t) * cta_start.size());
    if (!stages.empty())
        std::memcpy(p->tables + t.stages, stages.data(), sizeof(pa::StageTile) * stages.size());
    if (!upload_tables(p)) {
        cudaGetLastError();
        if (fresh) pa_plan_destroy(p);
        return pa::cuda_error();
    }
    *out = p;
    return PA_OK;
}

extern "C" int pa_plan_get_info(const pa_plan *p, pa_plan_info *info) {
    if (!p || !info) return PA_ERR_NULL;
    info->num_sms = p->num_sms;
    info->num_decode_rows = p->num_rows;
    info->num_decode_units = p->num_units;
    info->num_partials = p->num_pieces;
    info->num_combine_rows = p->num_combine;
    info->num_prefill_tiles = p->num_tiles;
    info->decode_kv_blocks = p->decode_blocks;
    info->prefill_causal_pairs = p->prefill_pairs;
    info->table_bytes = p->tl.bytes;
    info->workspace_bytes = p->ws.total;
    info->num_staged_kv_tiles = p->num_stages;
    info->num_prefill_ctas = p->num_prefill_ctas;
    info->num_prefix_groups = p->num_prefix_groups;
    // as pa_attention_varlen launches them: the decode kernel; staging and
    // prefill; the merge kernel when shared-prefix tiles run beside decode
    const bool side_by_side = p->overlap_sms > 0 && p->num_units > 0 && p->num_tiles > 0;
    info->decode_kv_keys = p->decode_keys;
    info->prefill_pair = p->prefill_pair ? 1 : 0;
    info->overlap_sms = p->overlap_sms;
    info->attention_launches = (p->num_units > 0 ? 1 : 0) + (p->num_tiles > 0 ? 1 : 0) +
                               (p->num_tiles > 0 && p->num_stages > 0 ? 1 : 0) +
                               (side_by_side && p->cascade && p->num_combine > 0 ? 1 : 0);
    return PA_OK;
}

extern "C" size_t pa_plan_workspace_bytes(const pa_plan *plan) { return plan ? plan->ws.total : 0; }

extern "C" void pa_plan_destroy(pa_plan *plan) {
    if (!plan) return;
    {
        DeviceScope scope(plan->device);
        wait_idle(plan);
        if (plan->d_tables) cudaFree(plan->d_tables);
        if (plan->upload_event) cudaEventDestroy(static_cast<cudaEvent_t>(plan->upload_event));
        for (void *e : {plan->use_event, plan->fork_event, plan->join_event})
            if (e) cudaEventDestroy(static_cast<cudaEvent_t>(e));
        if (plan->upload_stream) cudaStreamDestroy(static_cast<cudaStream_t>(plan->upload_stream));
    }
    free_tables(plan);
    delete plan;
}
