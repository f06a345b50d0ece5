// Paged attention for long query segments (prefill and chunked prefill) on
// the 5th-generation tensor cores.
//
// What is computed ("vLLM 学习笔记 01" §1.5-§1.6 and §2.1): query j of a
// segment with q_len L and seq_len n sits at position n - L + j and attends
// to keys 0 .. n - L + j of its own segment, read through the segment's
// block table; a prefill chunk therefore also reads the context that earlier
// chunks cached.  Here this is heavy, dense work: every query row meets
// hundreds to thousands of keys, so QK^T and PV run on tcgen05 MMAs.
//
// One CTA computes 128 consecutive queries of one segment for two query
// heads A and B that share a kv head (GQA), looping over 128-key tiles of
// the causal range; both heads use every K/V tile the CTA loads.  Tensor
// memory holds, per head, S (128 fp32 columns; P overwrites it as packed
// bf16) and O (head_dim fp32 columns): 512 columns.  Warp roles (384 threads):
//   warp 0      issues the MMAs (one thread) in the order
//                 S_A0 S_B0 | PV_A0 S_A1 | PV_B0 S_B1 | PV_A1 S_A2 | ...
//               where S_Xj = Q_X K_j^T (M 128, N 128, K D, A and B operands
//               in shared memory) and PV_Xj: O_X += P_Xj V_j (M 128, N D, K
//               128, A = P from TMEM).  So while the softmax warps of one
//               head work, the tensor cores work on the other head.
//               tcgen05.mma operations of one thread run in issue order,
//               which is what lets S_X(j+1) reuse the columns P_Xj was read
//               from, and makes "S_Xj complete" imply "PV_X(j-1) complete".
//   warps 1-3   load Q_A, Q_B once and K/V tiles (two stages) with 16-byte
//               cp.async, 16-token blocks dealt out to the warps, through the block
//               table, into 128-byte-swizzled tiles (rows of 64 dims x 2
//               bytes, chunk index XORed by the row: the SWIZZLE_128B layout
//               the MMA descriptors name; Q and K are read K-major, V
//               MN-major).  Rows past the segment's length are written as
//               zeros, so no NaN ever meets the tensor cores.
//   warps 4-7   softmax of head A, warps 8-11 of head B: one query row per
//               thread (warp w holds TMEM lanes 32 (w % 4) ...).  A thread
//               reads its S row twice from TMEM (max, then exponentials),
//               masks the causal edge by selection, works in base 2 with
//               scale*log2(e), moves its running max (and rescales its O row
//               in TMEM) only when it grows by more than
//               kPrefillRescaleThreshold, and writes P into the S columns.
//               At the end it reads its O row, divides by its sum and writes
//               bf16.
// Every wait is on an mbarrier and bounded; on a timeout the kernel sets a
// bit in the workspace status word and runs to the end without waiting,
// after which TMEM is released.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace pa {

namespace {

constexpr float kPrefillRescaleThreshold = 8.f;

template <int D>
struct PrefillCfg {
    static constexpr int kThreads = 384;
    static constexpr int kLoadWarps = 3;  // warps 1-3
    static constexpr int kLoaders = 32 * kLoadWarps;
    static constexpr int kSoftA = 4;      // warps 4-7
    static constexpr int kSoftB = 8;      // warps 8-11
    static constexpr int kTileBytes = 128 * D * 2;  // a Q, K or V tile
    static constexpr int kQAOff = 0;
    static constexpr int kQBOff = kTileBytes;
    static constexpr int kKVOff = 2 * kTileBytes;  // stage s: K at kKVOff + 2 s T, V at + T
    static constexpr int kBarOff = kKVOff + 4 * kTileBytes;
    static constexpr int kNumBars = 13;
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
    static constexpr int kUsed = kTmemSlotOff + 16;
    // At least 120 KiB, so that one CTA (holding 512 TMEM columns) fits per SM.
    static constexpr int kSmemBytes = kUsed + 1024 > 120 * 1024 ? kUsed + 1024 : 120 * 1024;
    static constexpr uint32_t kTmemCols = 512;
    // TMEM columns: S_A, O_A, S_B, O_B
    static constexpr uint32_t kSA = 0, kOA = 128, kSB = 256, kOB = 384;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ void st_shared_zero16(uint32_t addr) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic).
__device__ __forceinline__ uint64_t f2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Row max over 32 S columns; keys > pos excluded when `masked`.
__device__ __forceinline__ float chunk_max(const uint32_t (&r)[32], float mx, bool masked, int key0, int pos) {
    if (!masked) {
#pragma unroll
        for (int c = 0; c < 32; c += 2) mx = max3f(mx, __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
    } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) mx = fmaxf(mx, key0 + c <= pos ? __uint_as_float(r[c]) : -INFINITY);
    }
    return mx;
}

// P for 32 S columns: 2^(s*scale - m) as 16 packed bf16 pairs; adds the
// rounded values to lsum (as a packed pair of partial sums).
__device__ __forceinline__ void chunk_exp(const uint32_t (&r)[32], uint32_t (&pk)[16], uint64_t &lsum,
                                          uint64_t scale2, uint64_t nm2, bool masked, int key0, int pos) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        float x0, x1;
        f2_split(f2_fma(f2(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), scale2, nm2), x0, x1);
        if (masked) {
            if (key0 + 2 * c > pos) x0 = -INFINITY;
            if (key0 + 2 * c + 1 > pos) x1 = -INFINITY;
        }
        pk[c] = pack_bf16x2(fast_exp2(x0), fast_exp2(x1));
        lsum = f2_add(lsum, f2(__uint_as_float(pk[c] << 16), __uint_as_float(pk[c] & 0xffff0000u)));
    }
}

// Softmax of one head, one query row per thread (128 threads); the same code
// serves both heads of the CTA.
template <int D>
__device__ __noinline__ void softmax_head(const PrefillParams &p, uint32_t trow, uint32_t s_col, uint32_t o_col,
                                          uint64_t *s_full, uint64_t *p_full, uint64_t *o_done, int nkv, int t,
                                          int q_rows, int pos, int first_pos, int tok0, int head, bool &err) {
    float m = -INFINITY, l = 0.f;
    const uint64_t scale2 = f2(p.scale_log2, p.scale_log2);
    for (int j = 0; j < nkv; ++j) {
        if (!err && !mbar_wait(s_full, j & 1)) err = true;
        tc_fence_after();
        const int kbase = 128 * j;
        // only tiles that reach past the first query's position need the
        // causal mask (pos < n also covers the segment's length)
        const bool masked = kbase + 127 > first_pos;
        // pass 1: row max of the raw scores (scale > 0 commutes with max);
        // each TMEM load is in flight while the previous chunk is reduced
        float mx = -INFINITY;
        {
            uint32_t ra[32], rb[32];
            tmem_ld32(trow + s_col, ra);
            tmem_ld_wait();
            tmem_ld32(trow + s_col + 32, rb);
            mx = chunk_max(ra, mx, masked, kbase, pos);
            tmem_ld_wait();
            tmem_ld32(trow + s_col + 64, ra);
            mx = chunk_max(rb, mx, masked, kbase + 32, pos);
            tmem_ld_wait();
            tmem_ld32(trow + s_col + 96, rb);
            mx = chunk_max(ra, mx, masked, kbase + 64, pos);
            tmem_ld_wait();
            mx = chunk_max(rb, mx, masked, kbase + 96, pos);
        }
        mx *= p.scale_log2;
        float alpha = 1.f;
        const bool rescale = mx > m + kPrefillRescaleThreshold;
        if (rescale) {
            alpha = fast_exp2(m - mx);
            m = mx;
        }
        // O_X is stable: S_Xj completing implies PV_X(j-1) completed.  TMEM
        // loads and stores are warp-collective, so the warp rescales if any
        // lane needs it (alpha = 1 for the others).
        if (j > 0 && __any_sync(kFullMask, rescale)) {
#pragma unroll
            for (int i = 0; i < D / 32; ++i) {
                uint32_t o[32];
                tmem_ld32(trow + o_col + 32 * i, o);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                tmem_st32(trow + o_col + 32 * i, o);
            }
        }
        // pass 2: P = 2^(s*scale - m) as bf16, written over the S columns
        // already read (P chunk i goes to columns 16 i .. 16 i + 15)
        const uint64_t nm2 = f2(-m, -m);
        uint64_t lsum = f2(0.f, 0.f);
        {
            uint32_t ra[32], rb[32], pk[16];
            tmem_ld32(trow + s_col, ra);
            tmem_ld_wait();
            tmem_ld32(trow + s_col + 32, rb);
            chunk_exp(ra, pk, lsum, scale2, nm2, masked, kbase, pos);
            tmem_st16(trow + s_col, pk);
            tmem_ld_wait();
            tmem_ld32(trow + s_col + 64, ra);
            chunk_exp(rb, pk, lsum, scale2, nm2, masked, kbase + 32, pos);
            tmem_st16(trow + s_col + 16, pk);
            tmem_ld_wait();
            tmem_ld32(trow + s_col + 96, rb);
            chunk_exp(ra, pk, lsum, scale2, nm2, masked, kbase + 64, pos);
            tmem_st16(trow + s_col + 32, pk);
            tmem_ld_wait();
            chunk_exp(rb, pk, lsum, scale2, nm2, masked, kbase + 96, pos);
            tmem_st16(trow + s_col + 48, pk);
        }
        float l0, l1;
        f2_split(lsum, l0, l1);
        l = l * alpha + (l0 + l1);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
    }
    if (!err && !mbar_wait(o_done, 0)) err = true;
    tc_fence_after();
    const float inv = 1.f / l;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
        uint32_t o[32];
        tmem_ld32(trow + o_col + 32 * i, o);
        tmem_ld_wait();
        if (t < q_rows) {
            __nv_bfloat16 *orow = p.out + ((size_t)(tok0 + t) * p.num_q_heads + head) * D + 32 * i;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
                st16(orow + 8 * c, w);
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(384, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
    using C = PrefillCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQA = smem_u32(smem + C::kQAOff);
    const uint32_t sQB = smem_u32(smem + C::kQBOff);
    const uint32_t sKV = smem_u32(smem + C::kKVOff);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *q_full = bars + 0;
    uint64_t *kv_full = bars + 1;   // [2]
    uint64_t *kv_empty = bars + 3;  // [2]: both heads' PV of the stage's tile are complete
    uint64_t *sA_full = bars + 5, *sB_full = bars + 6;
    uint64_t *pA_full = bars + 7, *pB_full = bars + 8;
    uint64_t *oA_done = bars + 9, *oB_done = bars + 10;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kTmemSlotOff);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (blockIdx.x >= p.num_tiles) return;
    const PrefillTile tile = p.tiles[blockIdx.x];
    const int seq = tile.seq, q0 = tile.q_start;
    const int hA = tile.head;
    const bool two = tile.num_heads == 2;
    const int hB = hA + 1;
    const int tok0 = p.cu_seqlens_q[seq] + q0;
    const int L = p.cu_seqlens_q[seq + 1] - p.cu_seqlens_q[seq];
    const int n = p.seq_lens[seq];
    const int q_rows = min(128, L - q0);
    const int nkv = tile.n_kv_tiles;  // 128-key tiles covering keys 0 .. n - L + q0 + q_rows - 1
    const int g = hA / p.group;

    if (tid == 0) {
        mbar_init(q_full, C::kLoaders);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&kv_full[s], C::kLoaders);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(sA_full, 1);
        mbar_init(sB_full, 1);
        mbar_init(pA_full, 128);
        mbar_init(pB_full, 128);
        mbar_init(oA_done, 1);
        mbar_init(oB_done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool err = false;

    if (warp == 0) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, D, false, true);
            auto mma_s = [&](uint32_t sQ, int j, uint32_t col) {
                const uint32_t sK = sKV + (j & 1) * 2 * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {  // 16 dims per MMA
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_bf16_ss(tmem + col, umma_desc_sw128(sQ + off, 16, 1024),
                                 umma_desc_sw128(sK + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            auto mma_pv = [&](uint32_t p_col, int j, uint32_t o_col) {
                const uint32_t sV = sKV + (j & 1) * 2 * C::kTileBytes + C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // 16 keys per MMA; P: 8 columns of bf16 pairs
                    umma_bf16_ts(tmem + o_col, tmem + p_col + 8 * kk, umma_desc_sw128(sV + kk * 2048, 16384, 1024),
                                 idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
            };
            if (!err && !mbar_wait(q_full, 0)) err = true;
            if (!err && !mbar_wait(&kv_full[0], 0)) err = true;
            tc_fence_after();
            mma_s(sQA, 0, C::kSA);
            umma_commit(sA_full);
            if (two) {
                mma_s(sQB, 0, C::kSB);
                umma_commit(sB_full);
            }
            for (int j = 0; j < nkv; ++j) {
                const bool next = j + 1 < nkv;
                if (!err && !mbar_wait(pA_full, j & 1)) err = true;
                tc_fence_after();
                mma_pv(C::kSA, j, C::kOA);
                if (!next) umma_commit(oA_done);
                if (next) {
                    if (!err && !mbar_wait(&kv_full[(j + 1) & 1], ((j + 1) >> 1) & 1)) err = true;
                    tc_fence_after();
                    mma_s(sQA, j + 1, C::kSA);
                    umma_commit(sA_full);
                }
                if (two) {
                    if (!err && !mbar_wait(pB_full, j & 1)) err = true;
                    tc_fence_after();
                    mma_pv(C::kSB, j, C::kOB);
                    if (!next) umma_commit(oB_done);
                }
                umma_commit(&kv_empty[j & 1]);
                if (two && next) {
                    mma_s(sQB, j + 1, C::kSB);
                    umma_commit(sB_full);
                }
            }
            // nothing of ours may be in flight when TMEM is released
            if (!err && !mbar_wait(&kv_empty[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1)) err = true;
        }
    } else if (warp < C::kSoftA) {
        // ------------------------------------------------ loaders
        // A warp copies whole 16-token blocks: its lanes' (row, chunk) pairs
        // and their swizzled destinations are the same for every block.
        constexpr int kPerLane = 16 * (D / 8) / 32;  // chunks per lane per block
        const int lw = warp - 1;                     // loader warp 0..2
        const int kv_stride = p.num_kv_heads * D;    // elements between tokens of a block
        int src_col[kPerLane], row_of[kPerLane];
        uint32_t dst_off[kPerLane];
#pragma unroll
        for (int k = 0; k < kPerLane; ++k) {
            const int cidx = lane + 32 * k;
            const int row = cidx / (D / 8), ch = cidx % (D / 8);
            row_of[k] = row;
            src_col[k] = 8 * ch;
            dst_off[k] = (ch >> 3) * 16384 + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
        }
        const int32_t *bt_row = p.block_tables + (size_t)seq * p.max_blocks_per_seq;
        // Q tiles: 16-row groups of both heads dealt out to the loader warps
        {
            const size_t q_stride = (size_t)p.num_q_heads * D;
            for (int grp = lw; grp < (two ? 16 : 8); grp += C::kLoadWarps) {
                const int hh = grp >> 3, r0 = 16 * (grp & 7);
                const uint32_t sQ = hh ? sQB : sQA;
                const __nv_bfloat16 *qh = p.q + (size_t)tok0 * q_stride + (size_t)(hh ? hB : hA) * D;
#pragma unroll
                for (int k = 0; k < kPerLane; ++k) {
                    const int row = r0 + row_of[k];
                    const uint32_t dst = sQ + r0 * 128 + dst_off[k];
                    if (row < q_rows)
                        cp_async16(dst, qh + (size_t)row * q_stride + src_col[k]);
                    else
                        st_shared_zero16(dst);
                }
            }
        }
        cp_async_commit();
        // Tiles 0 and 1 go out at once; tile j >= 2 reuses the stage of tile
        // j - 2 once both heads' PV of that tile is complete.  A tile's
        // arrival is signalled before any wait on a stage, since the MMAs
        // that free the stage depend on it.  The tile's 8 blocks (K and V)
        // are dealt out to the loader warps.
        auto issue_tile = [&](int j) {
            const uint32_t sK = sKV + (j & 1) * 2 * C::kTileBytes, sV = sK + C::kTileBytes;
            for (int b = lw; b < 8; b += C::kLoadWarps) {  // block within the tile
                const int key0 = 128 * j + 16 * b;  // its first key
                const uint32_t tile_off = 16 * b * 128;
                if (key0 < n) {
                    const int blk = __ldg(bt_row + (key0 >> 4));
                    const size_t base = (size_t)blk * 16 * kv_stride + (size_t)g * D;
                    const __nv_bfloat16 *kb = p.k_cache + base, *vb = p.v_cache + base;
#pragma unroll
                    for (int k = 0; k < kPerLane; ++k) {
                        const int off = row_of[k] * kv_stride + src_col[k];
                        if (key0 + row_of[k] < n) {
                            cp_async16(sK + tile_off + dst_off[k], kb + off);
                            cp_async16(sV + tile_off + dst_off[k], vb + off);
                        } else {
                            st_shared_zero16(sK + tile_off + dst_off[k]);
                            st_shared_zero16(sV + tile_off + dst_off[k]);
                        }
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < kPerLane; ++k) {
                        st_shared_zero16(sK + tile_off + dst_off[k]);
                        st_shared_zero16(sV + tile_off + dst_off[k]);
                    }
                }
            }
            cp_async_commit();
        };
        issue_tile(0);
        if (nkv >= 2) {
            issue_tile(1);
            cp_async_wait<2>();  // Q has landed
        } else {
            cp_async_wait<1>();
        }
        fence_proxy_async_smem();
        mbar_arrive(q_full);
        if (nkv >= 2)
            cp_async_wait<1>();  // tile 0 has landed
        else
            cp_async_wait<0>();
        fence_proxy_async_smem();
        mbar_arrive(&kv_full[0]);
        for (int j = 2; j < nkv; ++j) {
            cp_async_wait<0>();  // tile j - 1 has landed
            fence_proxy_async_smem();
            mbar_arrive(&kv_full[(j - 1) & 1]);
            if (!err && !mbar_wait(&kv_empty[j & 1], ((j - 2) >> 1) & 1)) err = true;
            issue_tile(j);
        }
        if (nkv >= 2) {
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&kv_full[(nkv - 1) & 1]);
        }
    } else {
        // ------------------------------------------------ softmax warps
        const bool headA = warp < C::kSoftB;
        if (headA || two) {
            const int quarter = warp & 3;  // TMEM lane quarter this warp may access
            const int t = quarter * 32 + lane;
            const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
            const int first_pos = n - L + q0;
            const int pos = t < q_rows ? first_pos + t : 0;  // padding rows see key 0 only
            softmax_head<D>(p, trow, headA ? C::kSA : C::kSB, headA ? C::kOA : C::kOB, headA ? sA_full : sB_full,
                            headA ? pA_full : pB_full, headA ? oA_done : oB_done, nkv, t, q_rows, pos, first_pos,
                            tok0, headA ? hA : hB, err);
        }
    }
    if (err) atomicOr(p.status, kStatusWaitTimeout);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
}

template <int D>
cudaError_t launch_prefill_t(const PrefillParams &p, cudaStream_t stream) {
    using C = PrefillCfg<D>;
    static std::atomic<uint64_t> configured{0};  // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_relaxed) & bit)) {
        cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_relaxed);
    }
    prefill_kernel<D><<<p.num_tiles, C::kThreads, C::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool prefill_kernel_available() { return true; }

cudaError_t launch_prefill(const PrefillParams &p, int head_dim, cudaStream_t stream) {
    if (p.num_tiles == 0) return cudaSuccess;
    return head_dim == 64 ? launch_prefill_t<64>(p, stream) : launch_prefill_t<128>(p, stream);
}

}  // namespace pa
