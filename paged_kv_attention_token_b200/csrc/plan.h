// Internal layout of a pa_plan (host) and of the tables it copies into the
// workspace (device).  Shared by plan.cpp and the CUDA sources; not part of
// the public ABI.
#pragma once
#include <cstddef>
#include <climits>
#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/pa.h"

namespace pa {

// PA_ERR_CUDA, after clearing the calling thread's last CUDA error, so that
// the failure is reported once and a later call's launch check does not
// see it again.
inline int cuda_error() {
    cudaGetLastError();
    return PA_ERR_CUDA;
}

constexpr int kBlockSize = 16;
// Segments with q_len above this go to the tensor-core prefill kernel; the
// others are handled as independent query rows by the split-KV decode kernel.
constexpr int kDecodeMaxQLen = 16;
constexpr int kPrefillTileM = 128;  // query rows per prefill tile
constexpr int kPrefillTileN = 128;  // keys per prefill KV tile
constexpr size_t kWorkspaceAlign = 256;
// DecodeRow::slot_base of a row one warp covers entirely.  Split rows hold
// piece_base - first_unit, which may be negative, so the marker lies below
// every value that difference can take.
constexpr int32_t kUnsplitRow = INT32_MIN;

// One decode row: a query token and one kv head (the G query heads of that
// kv head are computed together).  Row id r = token_row * Hkv + kv_head.
struct DecodeRow {
    int32_t token;        // flat token index t
    int32_t seq;          // segment index i (block-table row)
    int32_t n_keys;       // keys this query sees: p + 1
    int32_t slot_base;    // kUnsplitRow: one warp covers the row and writes out
                          // directly; else partial slot of unit u is slot_base + u
    int32_t combine;      // index of the row's CombineRow (split rows only)
    int32_t first_block;  // first block read here: > 0 when the row's leading
                          // blocks are a prefix shared with other rows,
                          // attended by the prefill kernel (cascade)
    int32_t n_new;        // keys of the row written by this step: its segment's
                          // new tokens up to its own (keys n_keys - n_new ..
                          // n_keys - 1 are tokens token - n_new + 1 .. token)
    int32_t pad;
};

// A decode warp's work: flat (row, block) range [start, next unit's start);
// blocks are block-table indices (a row's range starts at its first_block).
// The first row's segment and key count are repeated here so that a warp
// can start its first copies without first reading the row table.
struct DecodeUnit {
    int32_t row;
    int32_t block;
    int32_t seq;     // rows[row].seq (0 for the end marker)
    int32_t n_keys;  // rows[row].n_keys (0 for the end marker)
    int32_t token;   // rows[row].token (0 for the end marker)
    int32_t n_new;   // rows[row].n_new (0 for the end marker)
};

// A row whose result is merged from partials: cut across several decode
// units, and/or with a shared prefix attended by the prefill kernel (whose
// partials come first, written before the decode kernel starts).  Each
// decode unit writes its partial, then takes a ticket from the row's counter
// (in the plan's device tables, zero after every upload); the unit that
// takes the last ticket merges all pieces, writes the row and sets the
// counter back to zero.  Nobody waits.
struct CombineRow {
    int32_t row;
    int32_t piece_base;
    int32_t piece_count;  // all partials: prefix pieces, then the decode units'
    int32_t tickets;      // decode units covering the row
};

// One prefill work item: up to 128 consecutive queries of one segment for one
// or two query heads that share a kv head.
struct PrefillTile {
    int32_t seq;        // segment index (its block table holds the keys)
    int32_t q_start;    // first query: within the segment (j), or for a
                        // shared-prefix tile the flat token index
    int32_t head;       // first query head
    int32_t n_kv_tiles; // 128-key tiles the tile reads
    int32_t num_heads;  // 1 or 2 (head and head + 1)
    int32_t kv_base;    // staged tile index of key tile 0 of (seq, kv head)
    int32_t kv_tile0;   // first key tile read (a key split of a shared prefix)
    int32_t key_limit;  // shared-prefix tile: every query sees keys < key_limit
    int32_t row_base;   // shared-prefix tile: decode row of its first token for
                        // this kv head (row of token k: row_base + k * Hkv);
                        // -1 for a causal tile of a prefill segment
    int32_t piece;      // shared-prefix tile: its piece among the row's partials
    int32_t q_rows;     // shared-prefix tile: query tokens (consecutive)
    int32_t pad;
};

// One staged key tile: keys 128 j .. 128 j + 127 of segment `seq` for one kv
// head, K and V, gathered from the paged cache into the workspace in the
// layout the prefill kernel's shared-memory tiles have (rows past the
// segment's length zeroed).  Staged tile s occupies bytes
// [2 s T, 2 s T + T) (K) and [2 s T + T, 2 (s + 1) T) (V) of the staged
// area, T = 128 * head_dim * 2.
struct StageTile {
    int32_t seq;
    int32_t kv_head;
    int32_t tile;    // j
    int32_t n_keys;  // keys that exist (the segment's length, or a shared
                     // prefix's): rows of the tile at or past it are zeroed
};

constexpr size_t kStagedAlign = 1024;

// The plan's tables, uploaded to a device buffer the plan owns: read-only
// work lists, and one merge ticket counter per split row (zero between
// calls: each call leaves them so).
struct TableLayout {
    size_t units = 0, rows = 0, combine = 0, tiles = 0, cta_start = 0, stages = 0, arrived = 0;  // byte offsets
    size_t bytes = 0;
};

// The caller's workspace: the header (status word first) at offset 0, then
// scratch that needs no initial value (split partials, staged K/V tiles).
struct WorkspaceLayout {
    size_t header = 0, partial_o = 0, partial_ml = 0, staged = 0;
    size_t total = 0;
};

}  // namespace pa

struct pa_plan {
    pa_dims dims{};
    int num_sms = 148;
    int group = 1;                       // Hq / Hkv
    // decode part
    int32_t num_units = 0;
    int32_t num_rows = 0;
    int32_t num_pieces = 0;
    int32_t num_combine = 0;
    int64_t decode_blocks = 0;           // sum over rows of ceil(n_keys / 16) - first_block
    int64_t decode_keys = 0;             // sum over rows of n_keys - 16 first_block
    // prefill part
    int32_t num_tiles = 0;
    int32_t num_prefill_ctas = 0;        // persistent prefill CTAs (one per SM at most)
    bool prefill_pair = false;           // tiles run on clusters of two CTAs (num_prefill_ctas / 2 clusters)
    int32_t overlap_sms = 0;             // > 0: prefill runs on this many SMs beside the decode kernel
    bool cascade = false;                // shared-prefix tiles: the prefill kernel runs first
    int32_t num_prefix_groups = 0;
    int32_t num_stages = 0;              // K/V key tiles staged into the workspace
    int32_t num_stages_fused = 0;        // of them, those holding keys written before the step:
                                         // the ones a fused step stages with the pair kernel
    int64_t prefill_pairs = 0;           // causal (query, key) pairs, per query head
    pa::TableLayout tl;
    pa::WorkspaceLayout ws;
    // Host image of the tables (page-locked when the plan has a device) and
    // its device copy.  A build uploads the image on the plan's own stream,
    // records upload_event and waits for it; every attention call outside
    // stream capture records use_event after its last kernel.  A rebuild or
    // destroy first waits for both, so that neither buffer changes under a
    // queued copy or a running kernel.
    uint8_t *tables = nullptr;
    size_t tables_capacity = 0;
    bool tables_pinned = false;
    void *d_tables = nullptr;            // device buffer (cudaMalloc), d_capacity bytes
    size_t d_capacity = 0;
    void *upload_stream = nullptr;       // cudaStream_t (non-blocking), or null without a device
    void *upload_event = nullptr;        // cudaEvent_t
    void *use_event = nullptr;           // cudaEvent_t
    void *fork_event = nullptr;          // cudaEvent_t: decode and prefill run side by side
    void *join_event = nullptr;          // cudaEvent_t
    int device = -1;
};

namespace pa {
constexpr size_t kHeaderBytes = 256;  // status word and reserved space
// Decode warps resident per SM for a head dim (one planner unit per warp).
int decode_units_per_sm(int head_dim);
// SM count of a device (cached per process; 148 when it cannot be read).
int device_sm_count(int device);
// Whether long segments go to the tensor-core prefill kernel.
bool prefill_kernel_available();
}  // namespace pa
