// Split-KV paged attention for short query segments (decodes).
//
// What is computed ("vLLM 学习笔记 01" §1.5-§1.6): for one query token at
// position p of its segment and one kv head g, the G = Hq / Hkv query heads
// of g attend to keys 0..p of the segment, read through its block table
// (logical block b -> physical block block_tables[seq][b], 16 tokens each).
//
// Design (HBM-bound: every KV byte is read once, ~G flops per byte):
//  * Work: the planner lays every (query row, kv head) row's 16-token blocks
//    end to end and gives each warp an equal run, so every warp moves the
//    same number of KV bytes whatever the length mix.  Warps never wait for
//    one another.
//  * Loads: each warp copies its blocks (the K and V of one kv head, 16
//    tokens) with 16-byte cp.async into its own ring of shared-memory stages
//    and keeps the next two steps in flight while it computes one, so an SM
//    has ~128 KiB of KV requests outstanding without holding them in
//    registers.  The copies write 128-byte rows with the chunk index XORed by
//    the row index (the usual 128-byte swizzle); a 16-token block is too
//    small a unit for TMA boxes to stream at HBM rate here.
//  * Compute: for one block a warp computes S^T[16 keys x 8 heads] = K Q^T
//    and O^T[D x 8 heads] += V^T P^T on warp-level MMA (m16n8k16, bf16 in,
//    fp32 accumulate): the 16 tokens of a block are exactly one M tile, so
//    G = 8 wastes no rows, and S^T turns into the B operand of the second MMA
//    with one movmatrix.trans per half.  The keys of a block are taken in the
//    order 0,4,1,5,2,6,3,7 (+8) and the output dims in the matching chunk
//    order, which makes every fragment read from the swizzled tiles touch 8
//    distinct 16-byte chunks per quarter-warp (no bank conflicts).
//  * Online softmax in fp32, base 2: scores are scaled by scale*log2(e); the
//    running max is shared by the 8 lanes that hold a head (3 xor-shuffles
//    per step), the running sum stays per lane until the end of a row.  A
//    step covers two blocks at D = 64.  The output is rescaled only when a
//    head's max grows by more than kRescaleThreshold, which after the first
//    blocks of a row is rare.
//  * Keys past the row's length in its last block are masked by selection
//    (score -inf, V zeroed), so whatever the cache holds there (NaN
//    included) never reaches the output.
//  * A row a warp covers entirely is normalised and written as bf16; a row
//    cut between warps leaves (O, max, sum) in the workspace and takes a
//    ticket; the warp with the row's last ticket merges the partials.  No
//    warp ever waits for another, and no thread spins.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace pa {

namespace {

// Rescaling of the running output is skipped while a head's running max
// grows by at most this much (log2 units): the probabilities then stay below
// 2^8, which fp32 sums and bf16 operands hold without loss of relative
// precision, and the max used is still an upper bound up to that margin.
constexpr float kRescaleThreshold = 8.f;

template <int D, int NT>
struct DecodeCfg {
    static constexpr int kWarps = 4;  // independent warps per CTA
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kTileBytes = 16 * 128;  // 16 tokens x 64 dims of one head
    static constexpr int kDimTiles = D / 64;
    static constexpr int kBlockBytes = 2 * kDimTiles * kTileBytes;  // K tiles then V tiles
    // blocks per softmax step: two at D = 64, where a block alone carries too
    // little work to pay for a softmax step
    static constexpr int kBlocksPerIter = D == 64 ? 2 : 1;
    static constexpr int kStageBytes = kBlocksPerIter * kBlockBytes;
    static constexpr int kStages = 3;  // per warp: two in flight while one is computed
    static constexpr int kCtasPerSm = 2;
    static constexpr int kSmemBytes = kWarps * kStages * kStageBytes + 1024;  // + alignment slack
    static_assert(kSmemBytes * kCtasPerSm <= 228 * 1024, "shared memory per SM");
};

// Key order inside a block (see the file comment): MMA row m holds token
// pi8(m) = (m >> 1) + 4 * (m & 1) for m < 8, and 8 + pi8(m - 8) above.  The
// same permutation picks each lane's output chunk.
__device__ __forceinline__ int pi8(int m) { return (m >> 1) + 4 * (m & 1); }

__device__ __forceinline__ uint32_t word(const uint4 &x, int i) {
    return i == 0 ? x.x : i == 1 ? x.y : i == 2 ? x.z : x.w;
}

// 2^x with the hardware approximation (ex2.approx.ftz: about 2 ulp); 2^-inf = 0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int D, int NT>
struct RowState {
    uint32_t qf[NT][D / 16][2];
    float o[D / 16][NT][4];
    float m[NT][2];  // max used as the exponent reference (log2 units)
    float l[NT][2];  // per-lane partial sums of 2^(s - m)
};

// One softmax step over NB blocks held in shared memory at `stage` (block nb
// at stage + nb * block_bytes: K tiles, then V tiles).  `valid` = keys of the
// row from the first block on; only the first nb_valid blocks are used.
template <int D, int NT, int NB>
__device__ __forceinline__ void attend_step(RowState<D, NT> &st, uint32_t stage, int valid, int nb_valid,
                                            float scale_log2, int g8, int q4) {
    constexpr int kBlockBytes = 2 * (D / 64) * 2048;
    // keys of unused block slots are masked like keys past the row's end (the
    // row may go on past a step that ends the warp's run)
    valid = min(valid, 16 * nb_valid);
    const int tok0 = pi8(g8), tok1 = 8 + pi8(g8);
    float s[NB][NT][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const uint32_t kt = stage + nb * kBlockBytes;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nb][nt][e] = 0.f;
            if (nb < nb_valid) {
#pragma unroll
                for (int i = 0; i < D / 32; ++i) {
                    const uint32_t tile = kt + (i >> 1) * 2048;
                    const int chunk = 4 * (i & 1) + q4;
                    const uint4 ka = ld_shared16(swz128(tile, tok0, chunk));
                    const uint4 kb = ld_shared16(swz128(tile, tok1, chunk));
                    mma_16816(s[nb][nt], ka.x, kb.x, ka.y, kb.y, st.qf[nt][2 * i][0], st.qf[nt][2 * i][1]);
                    mma_16816(s2, ka.z, kb.z, ka.w, kb.w, st.qf[nt][2 * i + 1][0], st.qf[nt][2 * i + 1][1]);
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nb][nt][e] += s2[e];
        }
    }
    const bool partial = valid < 16 * NB;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 16 * nb + ((e & 2) ? tok1 : tok0);
                float x = s[nb][nt][e] * scale_log2;
                if (partial && tok >= valid) x = -INFINITY;
                s[nb][nt][e] = x;
            }
    // running max per head (the 8 lanes of a head agree after the shuffles)
    float alpha[NT][2];
    bool any_rescale = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float mx = -INFINITY;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) mx = fmaxf(mx, fmaxf(s[nb][nt][e], s[nb][nt][e + 2]));
            mx = warp_max_xor(mx, 4);
            mx = warp_max_xor(mx, 8);
            mx = warp_max_xor(mx, 16);
            alpha[nt][e] = 1.f;
            if (mx > st.m[nt][e] + kRescaleThreshold) {
                alpha[nt][e] = fast_exp2(st.m[nt][e] - mx);
                st.m[nt][e] = mx;
                any_rescale = true;
            }
            float lsum = 0.f;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const float p0 = fast_exp2(s[nb][nt][e] - st.m[nt][e]);
                const float p1 = fast_exp2(s[nb][nt][e + 2] - st.m[nt][e]);
                // the PV product uses these rounded to bf16: sum the same values
                const uint32_t pr = pack_bf16x2(p0, p1);
                s[nb][nt][e] = __uint_as_float(pr << 16);
                s[nb][nt][e + 2] = __uint_as_float(pr & 0xffff0000u);
                lsum += bf16x2_sum(pr);
            }
            st.l[nt][e] = st.l[nt][e] * alpha[nt][e] + lsum;
        }
    if (__any_sync(kFullMask, any_rescale)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int t = 0; t < D / 16; ++t) {
                st.o[t][nt][0] *= alpha[nt][0];
                st.o[t][nt][1] *= alpha[nt][1];
                st.o[t][nt][2] *= alpha[nt][0];
                st.o[t][nt][3] *= alpha[nt][1];
            }
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        if (nb >= nb_valid) break;
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            pb[nt][0] = movmatrix_trans(pack_bf16x2(s[nb][nt][0], s[nb][nt][1]));
            pb[nt][1] = movmatrix_trans(pack_bf16x2(s[nb][nt][2], s[nb][nt][3]));
        }
        // V^T fragments: this lane's keys are tokens q4, q4+4, 8+q4, 12+q4 (the
        // P^T rows 2q4, 2q4+1, 2q4+8, 2q4+9); its dims are chunk pi8(g8) of
        // each 64-dim tile.
        const uint32_t vt = stage + nb * kBlockBytes + (D / 64) * 2048;
        const int vvalid = valid - 16 * nb;
#pragma unroll
        for (int j = 0; j < D / 64; ++j) {
            const uint32_t tile = vt + j * 2048;
            uint4 v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = q4 + 4 * e;
                v[e] = ld_shared16(swz128(tile, tok, pi8(g8)));
                if (partial && tok >= vvalid) v[e] = make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
                const uint32_t v0 = word(v[0], uu), v1 = word(v[1], uu);
                const uint32_t v2 = word(v[2], uu), v3 = word(v[3], uu);
                const uint32_t a0 = __byte_perm(v0, v1, 0x5410);
                const uint32_t a1 = __byte_perm(v0, v1, 0x7632);
                const uint32_t a2 = __byte_perm(v2, v3, 0x5410);
                const uint32_t a3 = __byte_perm(v2, v3, 0x7632);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma_16816(st.o[4 * j + uu][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
        }
    }
}

// Merge the partials of a split row and write it: O = sum_j 2^(m_j - M) O_j /
// sum_j 2^(m_j - M) l_j with M = max_j m_j, in one pass with a running max.
// Run by the warp that took the row's last ticket; the partials are read
// through L2 (ld.cg), where the other warps' released writes are visible,
// kMergeBatch partials at a time so that the loads overlap instead of
// forming a chain.
template <int D>
__device__ __forceinline__ void merge_split_row(const DecodeParams &p, const CombineRow c, int token,
                                             int h0, int tid, int nthreads) {
    constexpr int kMergeBatch = 8;
    const int G = p.group;
    const int n = c.piece_count;
    for (int item = tid; item < G * (D / 8); item += nthreads) {
        const int head = item / (D / 8);
        const int chunk = item % (D / 8);
        // one pass: a batch's (max, sum) and O are loaded together and folded
        // into a running max, sum and accumulator
        float M = -INFINITY, den = 0.f;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < n; j0 += kMergeBatch) {
            float2 ml[kMergeBatch];
            float4 lo[kMergeBatch], hi[kMergeBatch];
#pragma unroll
            for (int k = 0; k < kMergeBatch; ++k) {
                if (j0 + k < n) {
                    const size_t slot = (size_t)(c.piece_base + j0 + k);
                    ml[k] = __ldcg(&p.partial_ml[slot * G + head]);
                    const float4 *po = reinterpret_cast<const float4 *>(p.partial_o + (slot * G + head) * D + 8 * chunk);
                    lo[k] = __ldcg(po);
                    hi[k] = __ldcg(po + 1);
                } else {
                    ml[k] = make_float2(-INFINITY, 0.f);
                    lo[k] = hi[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            float Mn = M;
#pragma unroll
            for (int k = 0; k < kMergeBatch; ++k) Mn = fmaxf(Mn, ml[k].x);
            const float s = M == -INFINITY ? 0.f : exp2f(M - Mn);  // earlier batches, rescaled
            den *= s;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] *= s;
#pragma unroll
            for (int k = 0; k < kMergeBatch; ++k) {
                const float w = exp2f(ml[k].x - Mn);  // 0 for the padding entries
                den += w * ml[k].y;
                acc[0] += w * lo[k].x; acc[1] += w * lo[k].y; acc[2] += w * lo[k].z; acc[3] += w * lo[k].w;
                acc[4] += w * hi[k].x; acc[5] += w * hi[k].y; acc[6] += w * hi[k].z; acc[7] += w * hi[k].w;
            }
            M = Mn;
        }
        const float inv = 1.f / den;
        uint4 o;
        o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
        o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
        st16(p.out + ((size_t)token * p.num_q_heads + h0 + head) * D + 8 * chunk, o);
    }
}

// Takes a ticket: returns the counter's old value and adds one, with release
// semantics for the writes before it and acquire semantics for the reads
// after it (GPU scope), in one round trip to L2.
__device__ __forceinline__ uint32_t ticket_acq_rel(uint32_t *counter) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(counter) : "memory");
    return old;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// A warp's load position in its run: the step that starts at block b of row
// r (a step = up to kBlocksPerIter blocks of one row).  Block ids are fetched
// 32 at a time, one per lane, and broadcast with a shuffle, so a copy does
// not wait on its own block-table load.
struct LoadCursor {
    int r, b, bend, nblk, g;
    const int32_t *bt_row;
    int bt_base, bt_val;
    int n_keys, token, n_new;  // the row's keys, its query token and how many keys are new
    bool done;
};

__device__ __forceinline__ void cursor_set_row(const DecodeParams &p, const DecodeUnit &end, LoadCursor &c,
                                               int seq, int n_keys, int token, int n_new) {
    c.bt_row = p.block_tables + (size_t)seq * p.max_blocks_per_seq;
    c.nblk = (n_keys + 15) >> 4;
    c.n_keys = n_keys;
    c.token = token;
    c.n_new = n_new;
    c.bend = (c.r == end.row) ? end.block : c.nblk;
    c.g = c.r % p.num_kv_heads;
    c.bt_base = -1;
}

// Moves the cursor to the start of row c.r (its first_block), or marks it
// done when the warp's run ends before that.
__device__ __forceinline__ void cursor_enter_row(const DecodeParams &p, const DecodeUnit &end,
                                                 LoadCursor &c) {
    // (the run end of the last unit is row R, block 0: never read)
    if (c.r > end.row || (c.r == end.row && end.block == 0)) {
        c.done = true;
        return;
    }
    const DecodeRow row = p.rows[c.r];
    if (c.r == end.row && end.block <= row.first_block) {
        c.done = true;
        return;
    }
    c.b = row.first_block;
    cursor_set_row(p, end, c, row.seq, row.n_keys, row.token, row.n_new);
}

__device__ __forceinline__ int cursor_block_id(LoadCursor &c, int b, int lane) {
    if ((b & ~31) != c.bt_base) {
        c.bt_base = b & ~31;
        const int idx = c.bt_base + lane;
        c.bt_val = idx < c.nblk ? __ldg(c.bt_row + idx) : 0;
    }
    return __shfl_sync(kFullMask, c.bt_val, b & 31);
}

// Per-lane copy pattern of one block (K or V, one kv head, 16 tokens): chunk
// i of this lane is token row `row`, 16-byte column `col`; it goes to 128-byte
// row `row` of 64-dim tile col / 8, at chunk (col % 8) XOR (row % 8).
template <int D>
struct CopyPattern {
    int src[D / 16];       // element offset from the block's first element of the head
    uint32_t dst[D / 16];  // byte offset in the K (or V) tiles of the block
    __device__ __forceinline__ CopyPattern(int lane, int row_stride) {
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
            const int cidx = lane + 32 * i;
            const int row = cidx / (D / 8), col = cidx % (D / 8);
            src[i] = row * row_stride + 8 * col;
            dst[i] = (col >> 3) * 2048 + row * 128 + (((col & 7) ^ (row & 7)) << 4);
        }
    }
};

// Copies the blocks of the cursor's step into a stage and moves the cursor on.
// With p.k_new (a fused scatter and attention step), the keys this step
// writes are copied from k_new / v_new, the step's own K/V input, instead of
// from cache slots the scatter may not have written yet.
template <int D, int NB>
__device__ __forceinline__ void issue_step(const DecodeParams &p, const DecodeUnit &end, LoadCursor &c,
                                           const CopyPattern<D> &cp, uint32_t stage, int lane) {
    constexpr int kBlockBytes = 2 * (D / 64) * 2048;
    const size_t row_stride = (size_t)p.num_kv_heads * D;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        if (c.b + nb >= c.bend) break;
        const int id = cursor_block_id(c, c.b + nb, lane);
        const size_t base = (size_t)id * 16 * row_stride + (size_t)c.g * D;
        const __nv_bfloat16 *kb = p.k_cache + base;
        const __nv_bfloat16 *vb = p.v_cache + base;
        const uint32_t st = stage + nb * kBlockBytes;
        const int key0 = 16 * (c.b + nb);
        const int first_new = c.n_keys - c.n_new;
        if (p.k_new != nullptr && key0 + 16 > first_new) {
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
                const int cidx = lane + 32 * i;
                const int key = key0 + cidx / (D / 8);
                const __nv_bfloat16 *ks = kb + cp.src[i];
                const __nv_bfloat16 *vs = vb + cp.src[i];
                if (key >= first_new && key < c.n_keys) {
                    // token of key: the row's query token is its last key
                    const size_t o = ((size_t)(c.token - (c.n_keys - 1 - key)) * p.num_kv_heads + c.g) * D +
                                     8 * (cidx % (D / 8));
                    ks = p.k_new + o;
                    vs = p.v_new + o;
                }
                cp_async16(st + cp.dst[i], ks);
                cp_async16(st + (D / 64) * 2048 + cp.dst[i], vs);
            }
        } else {
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
                cp_async16(st + cp.dst[i], kb + cp.src[i]);
                cp_async16(st + (D / 64) * 2048 + cp.dst[i], vb + cp.src[i]);
            }
        }
    }
    c.b += NB;
    if (c.b >= c.bend) {
        ++c.r;
        cursor_enter_row(p, end, c);
    }
}

// Walks a warp's run piece by piece: fn(row_index, row, b0, bend), blocks
// [b0, bend) of the row's block table (a row's range starts at its
// first_block; the run may start inside its first row).
template <typename F>
__device__ __forceinline__ void for_each_piece(const DecodeParams &p, int unit, F &&fn) {
    const DecodeUnit start = p.units[unit];
    const DecodeUnit end = p.units[unit + 1];
    for (int r = start.row; r <= end.row; ++r) {
        if (r == end.row && end.block == 0) break;  // (row R of the last unit's end is never read)
        const DecodeRow row = p.rows[r];
        const int b0 = r == start.row ? start.block : row.first_block;
        const int bend = r == end.row ? end.block : (row.n_keys + 15) >> 4;
        if (b0 >= bend) break;
        fn(r, row, b0, bend);
    }
}

template <int D, int NT>
__global__ void __launch_bounds__(DecodeCfg<D, NT>::kThreads, DecodeCfg<D, NT>::kCtasPerSm)
    decode_kernel(const __grid_constant__ DecodeParams p) {
    using C = DecodeCfg<D, NT>;
    constexpr int S = C::kStages;
    constexpr int NB = C::kBlocksPerIter;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x * C::kWarps + warp;
    if (unit >= p.num_units) return;
    const uint32_t ring = smem_u32(smem) + warp * S * C::kStageBytes;
    const int Hkv = p.num_kv_heads;
    const DecodeUnit run_end = p.units[unit + 1];
    const DecodeUnit first = p.units[unit];
    const CopyPattern<D> cpat(lane, Hkv * D);
    // the plan's tables are ready before the launch; the caller's data may be
    // written by the kernel before this one (programmatic launch).  In a
    // fused step that kernel is the cache scatter, started after everything
    // before it had completed: the new keys come from k_new / v_new, no other
    // data depends on it, and the wait moves to the end (so that what
    // follows on the stream also follows the scatter).
    if (p.wait_first) grid_dependency_wait();
    if (p.trigger_dependents) grid_launch_dependents();

    // Load cursor: this warp's next step to copy; S-1 steps run ahead.
    LoadCursor lc;
    {
        // the unit carries its first row's segment and length: the first
        // copies need no read of the row table
        const DecodeUnit &st = first;
        lc.r = st.row;
        lc.b = st.block;
        lc.done = st.row > run_end.row || (st.row == run_end.row && st.block >= run_end.block);
        if (!lc.done) cursor_set_row(p, run_end, lc, st.seq, st.n_keys, st.token, st.n_new);
    }
#pragma unroll
    for (int j = 0; j < S - 1; ++j) {
        if (!lc.done) issue_step<D, NB>(p, run_end, lc, cpat, ring + j * C::kStageBytes, lane);
        cp_async_commit();
    }

    const int g8 = lane >> 2, q4 = lane & 3;
    const int G = p.group;
    int j = 0;  // this warp's step counter
    for_each_piece(p, unit, [&](int r, const DecodeRow &row, int b0, int bend) {
        const int gkv = r % Hkv;
        const int h0 = gkv * G;
        RowState<D, NT> st;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = 8 * nt + g8;
            const __nv_bfloat16 *qrow = p.q + ((size_t)row.token * p.num_q_heads + h0 + head) * D;
#pragma unroll
            for (int i = 0; i < D / 32; ++i) {
                uint4 w = make_uint4(0, 0, 0, 0);
                if (head < G) w = ld_nc16(qrow + 32 * i + 8 * q4);
                st.qf[nt][2 * i][0] = w.x;
                st.qf[nt][2 * i][1] = w.y;
                st.qf[nt][2 * i + 1][0] = w.z;
                st.qf[nt][2 * i + 1][1] = w.w;
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                st.m[nt][e] = -INFINITY;
                st.l[nt][e] = 0.f;
            }
#pragma unroll
            for (int t = 0; t < D / 16; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) st.o[t][nt][e] = 0.f;
        }
        for (int b = b0; b < bend; b += NB, ++j) {
            // refill the stage consumed last time, then wait for step j
            if (!lc.done) issue_step<D, NB>(p, run_end, lc, cpat, ring + ((j + S - 1) % S) * C::kStageBytes, lane);
            cp_async_commit();
            cp_async_wait<S - 1>();
            __syncwarp();
            attend_step<D, NT, NB>(st, ring + (j % S) * C::kStageBytes, row.n_keys - b * 16,
                                   min(NB, bend - b), p.scale_log2, g8, q4);
            __syncwarp();  // all lanes done with the stage before it is refilled
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float l = st.l[nt][e];
                l += __shfl_xor_sync(kFullMask, l, 4);
                l += __shfl_xor_sync(kFullMask, l, 8);
                l += __shfl_xor_sync(kFullMask, l, 16);
                st.l[nt][e] = l;
            }
        if (row.slot_base == kUnsplitRow) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int head = 8 * nt + 2 * q4 + e;
                    if (head >= G) continue;
                    const float inv = 1.f / st.l[nt][e];
                    __nv_bfloat16 *orow = p.out + ((size_t)row.token * p.num_q_heads + h0 + head) * D;
#pragma unroll
                    for (int jj = 0; jj < D / 64; ++jj) {
                        uint4 w;
                        w.x = pack_bf16x2(st.o[4 * jj + 0][nt][e] * inv, st.o[4 * jj + 0][nt][e + 2] * inv);
                        w.y = pack_bf16x2(st.o[4 * jj + 1][nt][e] * inv, st.o[4 * jj + 1][nt][e + 2] * inv);
                        w.z = pack_bf16x2(st.o[4 * jj + 2][nt][e] * inv, st.o[4 * jj + 2][nt][e + 2] * inv);
                        w.w = pack_bf16x2(st.o[4 * jj + 3][nt][e] * inv, st.o[4 * jj + 3][nt][e + 2] * inv);
                        st16(orow + 8 * (pi8(g8) + 8 * jj), w);
                    }
                }
        } else {
            // the row's merge entry, loaded while the partial is written
            const CombineRow c = p.combine[row.combine];
            const int slot = row.slot_base + unit;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int head = 8 * nt + 2 * q4 + e;
                    if (head >= G) continue;
                    float *po = p.partial_o + ((size_t)slot * G + head) * D;
#pragma unroll
                    for (int jj = 0; jj < D / 64; ++jj) {
                        float4 *dst = reinterpret_cast<float4 *>(po + 8 * (pi8(g8) + 8 * jj));
                        dst[0] = make_float4(st.o[4 * jj + 0][nt][e], st.o[4 * jj + 0][nt][e + 2],
                                             st.o[4 * jj + 1][nt][e], st.o[4 * jj + 1][nt][e + 2]);
                        dst[1] = make_float4(st.o[4 * jj + 2][nt][e], st.o[4 * jj + 2][nt][e + 2],
                                             st.o[4 * jj + 3][nt][e], st.o[4 * jj + 3][nt][e + 2]);
                    }
                    if (g8 == 0) p.partial_ml[(size_t)slot * G + head] = make_float2(st.m[nt][e], st.l[nt][e]);
                }
            // publish the partial, take a ticket; the last warp of the row
            // merges (unless a separate merge kernel follows, which the
            // kernel boundary orders after these writes).  The ticket is one
            // acquire-release atomic of lane 0: the warp barrier before it
            // orders every lane's partial writes before its release, and the
            // one after it orders its acquire before every lane's reads of
            // the other warps' partials.
            __syncwarp();
            if (p.defer_merge) return;
            int last = 0;
            if (lane == 0) last = ticket_acq_rel(&p.arrived[row.combine]) == (uint32_t)c.tickets - 1;
            last = __shfl_sync(kFullMask, last, 0);
            if (last) {
                __syncwarp();
                merge_split_row<D>(p, c, row.token, h0, lane, 32);
                // every ticket of this call is taken: leave the counter at zero
                if (lane == 0) p.arrived[row.combine] = 0u;
            }
        }
    });
    cp_async_wait<0>();  // nothing may still be landing when the warp exits
    if (!p.wait_first) grid_dependency_wait();
}

// Merges every combine row, one CTA per row (G x D / 8 items of one head
// and 8 dims, 128 of them at G = 8, head_dim 128: one round of partial loads
// per thread): used when
// the decode kernel ran beside the kernel that writes a row's shared-prefix
// partials, so that neither can merge.  Launched programmatically behind
// the decode kernel, its CTAs read their plan entries while that kernel
// ends and wait for it (and with it for the prefill kernel, which the
// decode kernel waits for at its end) before reading any partial.
template <int D>
__global__ void __launch_bounds__(128) merge_kernel(const __grid_constant__ DecodeParams p, int num_combine) {
    const int ci = blockIdx.x;
    const CombineRow c = p.combine[ci];
    const DecodeRow row = p.rows[c.row];
    grid_dependency_wait();
    merge_split_row<D>(p, c, row.token, (c.row % p.num_kv_heads) * p.group, threadIdx.x, 128);
}

template <int D, int NT>
cudaError_t launch_decode_t(const DecodeParams &p, cudaStream_t stream) {
    using C = DecodeCfg<D, NT>;
    static std::atomic<uint64_t> configured{0};  // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_relaxed) & bit)) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_relaxed);
    }
    // programmatic launch: the CTAs may become resident and read their work
    // units while the kernel before them (usually the cache scatter) ends
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((p.num_units + C::kWarps - 1) / C::kWarps);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<D, NT>, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

int decode_units_per_sm(int head_dim) {
    return head_dim == 64 ? DecodeCfg<64, 1>::kWarps * DecodeCfg<64, 1>::kCtasPerSm
                          : DecodeCfg<128, 1>::kWarps * DecodeCfg<128, 1>::kCtasPerSm;
}

cudaError_t launch_merge(const DecodeParams &p, int head_dim, int num_combine, bool programmatic,
                         cudaStream_t stream) {
    if (num_combine == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(num_combine);
    cfg.blockDim = dim3(128);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    const cudaError_t e = head_dim == 64 ? cudaLaunchKernelEx(&cfg, merge_kernel<64>, p, num_combine)
                                         : cudaLaunchKernelEx(&cfg, merge_kernel<128>, p, num_combine);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams &p, int head_dim, cudaStream_t stream) {
    if (p.num_units == 0) return cudaSuccess;
    const int nt = p.group > 8 ? 2 : 1;
    if (head_dim == 64) return nt == 1 ? launch_decode_t<64, 1>(p, stream) : launch_decode_t<64, 2>(p, stream);
    return nt == 1 ? launch_decode_t<128, 1>(p, stream) : launch_decode_t<128, 2>(p, stream);
}

}  // namespace pa
