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
//   warp 1      loads: Q of both heads once with TMA (no multicast), then
//               K tiles into a ring of kKStages and V tiles into a ring of
//               kVStages, K running ahead of V (K_(j+1) is issued before
//               V_j), each tile with one bulk copy from the staged tiles.
//               Tiles are 128-byte rows with the 128-byte swizzle the MMA
//               descriptors name (Q and K read K-major, V MN-major).
//
// Staging (stage_kernel, launched first): the K/V of a prefill segment are
// gathered once per kv head from the paged cache, through the block table,
// into the workspace as 128-key tiles laid out exactly like the shared-memory
// tiles, rows past the segment's length zeroed (so that P = 0 meets zeros,
// never unused or NaN slots).  Measured on B200, TMA boxes of one 16-token
// block fill shared memory at ~20 B per SM clock and cp.async at ~24, while
// two 128-query heads of this kernel consume ~32 B per clock at tensor-core
// rate; contiguous bulk copies from L2 run at ~50.  The gather moves each
// K/V byte of a segment once more, which next to the segment's
// (q_len x keys) work is a small fraction for any q_len above 16.
//   warps 2-3   idle (they only give their registers to the softmax warps).
//   warps 4-7   softmax of head A, warps 8-11 of head B: one query row per
//               thread (warp w holds TMEM lanes 32 (w % 4) ...).  A thread
//               reads its S row once from TMEM into registers, masks the
//               causal edge by selection, works in base 2 with
//               scale*log2(e), moves its running max (and rescales its O row
//               in TMEM) only when it grows by more than
//               kPrefillRescaleThreshold, and writes P into the S columns.
//               At the end it reads its O row, divides by its sum and
//               writes bf16.
// Every wait is on an mbarrier and bounded; on a timeout the kernel sets a
// bit in the workspace status word and runs to the end without waiting for
// its partners, but still waits (bounded) for its own MMAs and copies in
// flight before TMEM is released and the CTA ends.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace pa {

namespace {

constexpr float kPrefillRescaleThreshold = 8.f;

// The softmax evaluates 2^x on two pipes: the MUFU unit (ex2.approx) and, for
// the pairs k (0..15) of a 32-column chunk with bit k % 4 set in
// kPolyPairMask, a polynomial on the FMA and integer pipes.  The MUFU unit
// does 16 results per SM clock, so 128 x 128 exponentials per head and
// 128-key step take as long as that step's MMAs; moving part of them to the
// FMA pipe shortens each softmax chain.
constexpr uint32_t kPolyPairMask = 0x0;
// P is packed to bf16 pairs either with cvt.rn.bf16x2.f32 or with integer
// adds and a byte permute (rounding half up; it differs from round-to-even
// only on exact ties).
constexpr bool kPackOnAlu = false;

template <int D>
struct PrefillCfg {
    static constexpr int kThreads = 384;
    static constexpr int kSoftB = 8;  // softmax of head A: warps 4-7, of head B: warps 8-11
    static constexpr int kSlabs = D / 64;           // 64-dim slabs of a tile
    static constexpr int kTileBytes = 128 * D * 2;  // a Q, K or V tile
    static constexpr int kKStages = D == 128 ? 3 : 4;
    static constexpr int kVStages = D == 128 ? 2 : 4;
    static constexpr int kQAOff = 0;
    static constexpr int kQBOff = kTileBytes;
    static constexpr int kKOff = 2 * kTileBytes;
    static constexpr int kVOff = kKOff + kKStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
    // mbarriers
    static constexpr int kBarQ = 0, kBarQEmpty = 1;
    static constexpr int kBarKFull = 2;
    static constexpr int kBarKEmpty = kBarKFull + kKStages;
    static constexpr int kBarVFull = kBarKEmpty + kKStages;
    static constexpr int kBarVEmpty = kBarVFull + kVStages;
    static constexpr int kBarSA = kBarVEmpty + kVStages, kBarSB = kBarSA + 1;
    static constexpr int kBarPA = kBarSB + 1, kBarPB = kBarPA + 1;
    static constexpr int kBarOA = kBarPB + 1, kBarOB = kBarOA + 1;
    static constexpr int kBarOAFree = kBarOB + 1, kBarOBFree = kBarOAFree + 1;
    static constexpr int kBarDrain = kBarOBFree + 1;  // every MMA issued has completed
    static constexpr int kNumBars = kBarDrain + 1;
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
    static constexpr int kUsed = kTmemSlotOff + 16;
    // + 1024 to align the base; well above half an SM's shared memory, so
    // one CTA (holding all 512 TMEM columns) runs per SM.
    static constexpr int kSmemBytes = kUsed + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kSmemBytes > 116 * 1024, "one CTA per SM");
    static constexpr uint32_t kTmemCols = 512;
    // TMEM columns: S_A, O_A, S_B, O_B
    static constexpr uint32_t kSA = 0, kOA = 128, kSB = 256, kOB = 384;
    // Register split: the kernel starts with kLaunchRegs per thread (the
    // launch bound's cap, checked against ptxas output at build time);
    // warpgroup 0 (MMA, TMA, idle warps) gives registers up to the two
    // softmax warpgroups.
    static constexpr int kLaunchRegs = 168;
    static constexpr int kRegsLow = 104;
    static constexpr int kRegsHigh = 200;
    static_assert(128 * kRegsLow + 256 * kRegsHigh <= 384 * kLaunchRegs, "register split");
};

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
__device__ __forceinline__ uint64_t f2_add_rm(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rm.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 2^x of a pair without the MUFU unit.  With x clamped to >= -127,
// 2^x = 2^n * 2^f for n = floor(x) and f = x - n in [0, 1): adding 1.5 * 2^23
// with rounding toward -inf leaves n in the low mantissa bits of the sum (so
// n is exact and f = x - n exact), 2^f is a cubic in f, and 2^n enters by
// adding n to the exponent field of the cubic's value (the low bits of the
// sum, shifted up 23 places, are n mod 2^9).  The cubic's coefficients were
// fitted here to 2^f on [0, 1) by least squares reweighted towards the
// smallest maximum relative error: 8.6e-5, against 2^-9 for the bf16 P the
// value becomes.  At x = -127 the result is about 2^-127 (masked keys are
// zeroed by selection).
__device__ __forceinline__ uint64_t exp2_poly(uint64_t x) {
    constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
    constexpr float kC1 = 0.6951165795326233f, kC2 = 0.22764593362808228f, kC3 = 0.07706617563962936f;
    float x0, x1;
    f2_split(x, x0, x1);
    x = f2(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
    const uint64_t magic = f2(kMagic, kMagic);
    const uint64_t t = f2_add_rm(x, magic);
    const uint64_t fr = f2_sub(x, f2_sub(t, magic));
    uint64_t p = f2_fma(fr, f2(kC3, kC3), f2(kC2, kC2));
    p = f2_fma(fr, p, f2(kC1, kC1));
    p = f2_fma(fr, p, f2(1.f, 1.f));
    float p0, p1, t0, t1;
    f2_split(p, p0, p1);
    f2_split(t, t0, t1);
    return f2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
              __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

// bf16 pair of two probabilities (>= 0): e0 in the low half.
__device__ __forceinline__ uint32_t pack_p(float e0, float e1) {
    if constexpr (kPackOnAlu) {
        return __byte_perm(__float_as_uint(e0) + 0x8000u, __float_as_uint(e1) + 0x8000u, 0x7632);
    } else {
        return pack_bf16x2(e0, e1);
    }
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Max over 32 S columns; keys > pos excluded when `masked`.  Two
// independent chains, so that the reduction's latency is half its length.
__device__ __forceinline__ float chunk_max(const uint32_t (&r)[32], bool masked, int key0, int pos) {
    float a = -INFINITY, b = -INFINITY;
    if (!masked) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
            a = max3f(a, __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
            b = max3f(b, __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
        }
    } else {
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
            a = fmaxf(a, key0 + c <= pos ? __uint_as_float(r[c]) : -INFINITY);
            b = fmaxf(b, key0 + c + 1 <= pos ? __uint_as_float(r[c + 1]) : -INFINITY);
        }
    }
    return fmaxf(a, b);
}

// P for 32 S columns: 2^(s*scale - m) as 16 packed bf16 pairs; keys past
// `pos` (when `masked`) get P = 0 by selection.
__device__ __forceinline__ void chunk_exp(const uint32_t (&r)[32], uint32_t (&pk)[16], uint64_t scale2,
                                          uint64_t nm2, bool masked, int key0, int pos) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint64_t x = f2_fma(f2(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), scale2, nm2);
        float e0, e1;
        if ((kPolyPairMask >> (c & 3)) & 1u) {
            f2_split(exp2_poly(x), e0, e1);
            if (masked) {
                if (key0 + 2 * c > pos) e0 = 0.f;
                if (key0 + 2 * c + 1 > pos) e1 = 0.f;
            }
        } else {
            float x0, x1;
            f2_split(x, x0, x1);
            if (masked) {
                if (key0 + 2 * c > pos) x0 = -INFINITY;
                if (key0 + 2 * c + 1 > pos) x1 = -INFINITY;
            }
            e0 = fast_exp2(x0);
            e1 = fast_exp2(x1);
        }
        pk[c] = pack_p(e0, e1);
    }
}

// Sum of the 32 rounded values of a P chunk (as a packed pair of partial
// sums), so that the row sum matches the P the PV product uses.  Two
// independent chains.
__device__ __forceinline__ uint64_t chunk_sum(const uint32_t (&pk)[16]) {
    uint64_t sum[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < 16; ++c)
        sum[c & 1] = f2_add(sum[c & 1], f2(__uint_as_float(pk[c] << 16), __uint_as_float(pk[c] & 0xffff0000u)));
    return f2_add(sum[0], sum[1]);
}

// Ties 16 registers to this point of the program (volatile asm keeps its
// order), so that work on them is not scheduled before it.
__device__ __forceinline__ void regs_after(uint32_t (&r)[16]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]));
}

// Softmax of one head for one tile, one query row per thread (128 threads);
// the same code serves both heads.  `it` counts this head's 128-key steps
// over the CTA's tiles (the parity of s_full / p_full), `k` its tiles (the
// parity of o_done).  After the last step the thread reads its O row from
// TMEM, releases O (o_free) for the next tile's first PV, then divides by
// its sum and writes bf16.
template <int D>
__device__ __forceinline__ void softmax_tile(const PrefillParams &p, int nkv, int kv_tile0, int row_base, int piece,
                                             uint32_t trow, uint32_t s_col, uint32_t o_col, uint64_t *s_full,
                                             uint64_t *p_full, uint64_t *o_done, uint64_t *o_free, uint32_t &it,
                                             uint32_t k, int t, int q_rows, int pos, int first_pos, int tok0, int head,
                                             int hl, bool &err) {
    float m = -INFINITY, l = 0.f;
    const uint64_t scale2 = f2(p.scale_log2, p.scale_log2);
    for (int j = 0; j < nkv; ++j, ++it) {
        if (!err && !mbar_wait(s_full, it & 1, p.wait_limit)) err = true;
        tc_fence_after();
        const int kbase = 128 * (kv_tile0 + j);  // first key of this step
        // only tiles that reach past the first query's position need the
        // causal mask (pos < n also covers the segment's length)
        const bool masked = kbase + 127 > first_pos;
        uint32_t s0[32], s1[32], s2[32], s3[32];
        tmem_ld32(trow + s_col, s0);
        tmem_ld32(trow + s_col + 32, s1);
        tmem_ld32(trow + s_col + 64, s2);
        tmem_ld32(trow + s_col + 96, s3);
        tmem_ld_wait();
        // row max of the raw scores (scale > 0 commutes with max)
        float mx = fmaxf(fmaxf(chunk_max(s0, masked, kbase, pos), chunk_max(s1, masked, kbase + 32, pos)),
                         fmaxf(chunk_max(s2, masked, kbase + 64, pos), chunk_max(s3, masked, kbase + 96, pos)));
        mx *= p.scale_log2;
        float alpha = 1.f;
        const bool rescale = mx > m + kPrefillRescaleThreshold;
        if (rescale) {
            alpha = fast_exp2(m - mx);
            m = mx;
        }
        // P = 2^(s*scale - m) as bf16, written over the S columns (P chunk
        // i goes to columns 16 i .. 16 i + 15)
        const uint64_t nm2 = f2(-m, -m);
        uint32_t pk0[16], pk1[16], pk2[16], pk3[16];
        chunk_exp(s0, pk0, scale2, nm2, masked, kbase, pos);
        tmem_st16(trow + s_col, pk0);
        chunk_exp(s1, pk1, scale2, nm2, masked, kbase + 32, pos);
        tmem_st16(trow + s_col + 16, pk1);
        chunk_exp(s2, pk2, scale2, nm2, masked, kbase + 64, pos);
        tmem_st16(trow + s_col + 32, pk2);
        chunk_exp(s3, pk3, scale2, nm2, masked, kbase + 96, pos);
        tmem_st16(trow + s_col + 48, pk3);
        // O_X is stable: S_Xj completing implies PV_X(j-1) completed; PV_Xj
        // waits for p_full.  TMEM loads and stores are warp-collective, so
        // the warp rescales if any lane needs it (alpha = 1 for the others).
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
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(p_full);
        // the row sum, off the path that hands P to the tensor cores
        regs_after(pk0);
        regs_after(pk1);
        regs_after(pk2);
        regs_after(pk3);
        const uint64_t lsum = f2_add(f2_add(chunk_sum(pk0), chunk_sum(pk1)), f2_add(chunk_sum(pk2), chunk_sum(pk3)));
        float l0, l1;
        f2_split(lsum, l0, l1);
        l = l * alpha + (l0 + l1);
    }
    if (!err && !mbar_wait(o_done, k & 1, p.wait_limit)) err = true;
    tc_fence_after();
    // the whole O row at once (one wait: TMEM loads queue behind the MMAs of
    // the other head), then O is free for the next tile
    uint32_t o[D / 32][32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) tmem_ld32(trow + o_col + 32 * i, o[i]);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(o_free);
    if (row_base >= 0) {
        // shared-prefix tile: unnormalised O and (max, sum) become one
        // partial of the decode row of this token and kv head (hl: the
        // head's index within its kv group)
        if (t < q_rows) {
            const int G = p.group;
            const int r = row_base + t * p.num_kv_heads;
            const int slot = p.combine[p.rows[r].combine].piece_base + piece;
            float *po = p.partial_o + ((size_t)slot * G + hl) * D;
#pragma unroll
            for (int i = 0; i < D / 32; ++i)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    reinterpret_cast<float4 *>(po + 32 * i)[c] =
                        make_float4(__uint_as_float(o[i][4 * c]), __uint_as_float(o[i][4 * c + 1]),
                                    __uint_as_float(o[i][4 * c + 2]), __uint_as_float(o[i][4 * c + 3]));
            p.partial_ml[(size_t)slot * G + hl] = make_float2(m, l);
        }
        return;
    }
    const float inv = 1.f / l;
    if (t < q_rows) {
        __nv_bfloat16 *orow = p.out + ((size_t)(tok0 + t) * p.num_q_heads + head) * D;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(o[i][8 * c + 0]) * inv, __uint_as_float(o[i][8 * c + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(o[i][8 * c + 2]) * inv, __uint_as_float(o[i][8 * c + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(o[i][8 * c + 4]) * inv, __uint_as_float(o[i][8 * c + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(o[i][8 * c + 6]) * inv, __uint_as_float(o[i][8 * c + 7]) * inv);
                st16(orow + 32 * i + 8 * c, w);
            }
        }
    }
}

// TMA descriptor of q as {D, Hq, T} (innermost first), boxes of
// {64, 1, 128}: one 64-dim slab of 128 tokens of one head, 128-byte swizzle.
struct PrefillMaps {
    CUtensorMap q;
};

// Gathers staged tile blockIdx.x (K for blockIdx.y = 0, V for 1) from the
// paged cache: 16-byte chunks, rows of one kv head's keys, swizzled as the
// prefill kernel's shared-memory tiles.
template <int D>
__global__ void __launch_bounds__(256) stage_kernel(const __grid_constant__ PrefillParams p) {
    constexpr int kRowChunks = D / 8;
    const int kv = blockIdx.y;
    const StageTile st = p.stages[blockIdx.x];
    const int n = st.n_keys;
    const int32_t *bt_row = p.block_tables + (size_t)st.seq * p.max_blocks_per_seq;
    const __nv_bfloat16 *cache = kv ? p.v_cache : p.k_cache;
    uint8_t *tile = p.staged + ((size_t)blockIdx.x * 2 + kv) * (128 * D * 2);
    for (int c = threadIdx.x; c < 128 * kRowChunks; c += 256) {
        const int row = c / kRowChunks, ch = c % kRowChunks;
        const int key = 128 * st.tile + row;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (key < n) {
            const int blk = __ldg(bt_row + (key >> 4));
            v = ld_stream16(cache + (((size_t)blk * kBlockSize + (key & 15)) * p.num_kv_heads + st.kv_head) * D + ch * 8);
        }
        st16(tile + (ch >> 3) * 16384 + row * 128 + (((ch & 7) ^ (row & 7)) << 4), v);
    }
}

// One persistent CTA per SM works through its tiles [cta_start[c],
// cta_start[c + 1]).  Barrier phases run on across tiles: the rings of K and
// V stages, the per-step handshakes (S ready, P ready) and the per-tile ones
// (Q loaded, Q free, O ready, O free).
template <int D>
__global__ void __launch_bounds__(384, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps maps) {
    using C = PrefillCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQA = smem_u32(smem + C::kQAOff);
    const uint32_t sQB = smem_u32(smem + C::kQBOff);
    const uint32_t sK = smem_u32(smem + C::kKOff);
    const uint32_t sV = smem_u32(smem + C::kVOff);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *q_full = bars + C::kBarQ, *q_empty = bars + C::kBarQEmpty;
    uint64_t *k_full = bars + C::kBarKFull, *k_empty = bars + C::kBarKEmpty;
    uint64_t *v_full = bars + C::kBarVFull, *v_empty = bars + C::kBarVEmpty;
    uint64_t *sA_full = bars + C::kBarSA, *sB_full = bars + C::kBarSB;
    uint64_t *pA_full = bars + C::kBarPA, *pB_full = bars + C::kBarPB;
    uint64_t *oA_done = bars + C::kBarOA, *oB_done = bars + C::kBarOB;
    uint64_t *oA_free = bars + C::kBarOAFree, *oB_free = bars + C::kBarOBFree;
    uint64_t *drain = bars + C::kBarDrain;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kTmemSlotOff);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (blockIdx.x >= p.num_ctas) return;
    const int t_begin = p.cta_start[blockIdx.x], t_end = p.cta_start[blockIdx.x + 1];
    if (t_begin >= t_end) return;

    if (tid == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::kKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::kVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(sA_full, 1);
        mbar_init(sB_full, 1);
        mbar_init(pA_full, 4);  // one arrive per softmax warp
        mbar_init(pB_full, 4);
        mbar_init(oA_done, 1);
        mbar_init(oB_done, 1);
        mbar_init(oA_free, 4);
        mbar_init(oB_free, 4);
        mbar_init(drain, 1);
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

    if (warp < 4) {
        warpgroup_reg_dealloc<C::kRegsLow>();
        if (warp == 0 && lane == 0) {
            // ------------------------------------------------ MMA issuer
            // The tensor pipe runs dry unless this thread issues an MMA
            // every few dozen cycles while it shares its SM sub-partition
            // with two softmax warps, so all descriptors are formed once:
            // the start-address field holds address >> 4 in the low bits,
            // so a byte offset o within shared memory adds o >> 4.
            constexpr uint32_t idesc_s = umma_idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, D, false, true);
            constexpr uint32_t kTileStep = C::kTileBytes >> 4;
            const uint64_t dQA = umma_desc_sw128(sQA, 16, 1024), dQB = umma_desc_sw128(sQB, 16, 1024);
            const uint64_t dK = umma_desc_sw128(sK, 16, 1024), dV = umma_desc_sw128(sV, 16384, 1024);
            auto mma_s = [&](uint64_t dq, uint64_t dk, uint32_t col) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {  // 16 dims per MMA
                    const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                    umma_bf16_ss(tmem + col, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            auto mma_pv = [&](uint64_t dv, uint32_t p_col, uint32_t o_col, uint32_t acc0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // 16 keys per MMA; P: 8 columns of bf16 pairs
                    umma_bf16_ts(tmem + o_col, tmem + p_col + 8 * kk, dv + ((kk * 2048) >> 4), idesc_pv,
                                 kk > 0 ? 1u : acc0);
            };
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                if (!err && !mbar_wait(bar, parity, p.wait_limit)) err = true;
            };
            int vs = 0, ks = 0;          // ring slots of the next V and K tiles
            uint32_t vph = 0, kph = 0;   // and their phases
            uint32_t itA = 0, itB = 0;   // 128-key steps of head A / head B so far
            uint32_t kA = 0, kB = 0;     // tiles of head A / head B so far
            for (int ti = t_begin; ti < t_end; ++ti) {
                const PrefillTile tile = p.tiles[ti];
                const bool two = tile.num_heads == 2;
                const int nkv = tile.n_kv_tiles;
                wait(q_full, (uint32_t)(ti - t_begin) & 1);
                wait(&k_full[ks], kph);
                tc_fence_after();
                uint64_t dk = dK + ks * kTileStep;
                mma_s(dQA, dk, C::kSA);
                umma_commit(sA_full);
                if (two) {
                    mma_s(dQB, dk, C::kSB);
                    umma_commit(sB_full);
                }
                umma_commit(&k_empty[ks]);
                if (nkv == 1) umma_commit(q_empty);
                if (++ks == C::kKStages) { ks = 0; kph ^= 1u; }
                for (int j = 0; j < nkv; ++j) {
                    const bool next = j + 1 < nkv;
                    const uint64_t dv = dV + vs * kTileStep;
                    const uint32_t acc0 = j > 0 ? 1u : 0u;
                    wait(pA_full, itA & 1);
                    if (j == 0 && kA > 0) wait(oA_free, (kA - 1) & 1);  // previous tile's O_A read out
                    wait(&v_full[vs], vph);
                    tc_fence_after();
                    mma_pv(dv, C::kSA, C::kOA, acc0);
                    if (!next) umma_commit(oA_done);
                    if (next) {
                        wait(&k_full[ks], kph);
                        tc_fence_after();
                        dk = dK + ks * kTileStep;
                        mma_s(dQA, dk, C::kSA);
                        umma_commit(sA_full);
                    }
                    if (two) {
                        wait(pB_full, itB & 1);
                        if (j == 0 && kB > 0) wait(oB_free, (kB - 1) & 1);
                        tc_fence_after();
                        mma_pv(dv, C::kSB, C::kOB, acc0);
                        if (!next) umma_commit(oB_done);
                    }
                    umma_commit(&v_empty[vs]);
                    if (next) {
                        if (two) {
                            mma_s(dQB, dk, C::kSB);
                            umma_commit(sB_full);
                        }
                        umma_commit(&k_empty[ks]);
                        if (j + 2 == nkv) umma_commit(q_empty);  // last S of the tile issued
                        if (++ks == C::kKStages) { ks = 0; kph ^= 1u; }
                    }
                    if (++vs == C::kVStages) { vs = 0; vph ^= 1u; }
                    ++itA;
                    if (two) ++itB;
                }
                ++kA;
                if (two) ++kB;
            }
            // nothing of ours may be in flight when TMEM is released: one
            // more commit covers every MMA issued, and it is waited for even
            // after a timeout (bounded), so that an error never frees TMEM
            // under a running MMA
            umma_commit(drain);
            if (!mbar_wait(drain, 0, p.wait_limit)) err = true;
        } else if (warp == 1 && lane == 0) {
            // ------------------------------------------------ loads
            int vs = 0, ks = 0;
            uint32_t vuse = 0, kuse = 0;  // K / V tiles loaded so far
            for (int ti = t_begin; ti < t_end; ++ti) {
                const PrefillTile tile = p.tiles[ti];
                const bool two = tile.num_heads == 2;
                const int nkv = tile.n_kv_tiles;
                const int hA = tile.head;
                const int tok0 = tile.row_base >= 0 ? tile.q_start : p.cu_seqlens_q[tile.seq] + tile.q_start;
                if (ti > t_begin && !err && !mbar_wait(q_empty, (uint32_t)(ti - t_begin - 1) & 1, p.wait_limit)) err = true;
                mbar_arrive_expect_tx(q_full, (two ? 2 : 1) * C::kTileBytes);
#pragma unroll
                for (int s = 0; s < C::kSlabs; ++s) {
                    tma_load_3d(sQA + s * 16384, &maps.q, q_full, 64 * s, hA, tok0);
                    if (two) tma_load_3d(sQB + s * 16384, &maps.q, q_full, 64 * s, hA + 1, tok0);
                }
                // staged tile kv_base + j: K then V, kTileBytes each
                const uint8_t *kv_tiles = p.staged + (size_t)(tile.kv_base + tile.kv_tile0) * 2 * C::kTileBytes;
                auto load_k = [&](int j) {
                    if (kuse >= (uint32_t)C::kKStages && !err &&
                        !mbar_wait(&k_empty[ks], (kuse / C::kKStages - 1) & 1, p.wait_limit))
                        err = true;
                    mbar_arrive_expect_tx(&k_full[ks], C::kTileBytes);
                    bulk_load(sK + ks * C::kTileBytes, kv_tiles + (size_t)j * 2 * C::kTileBytes, C::kTileBytes,
                              &k_full[ks]);
                    ++kuse;
                    if (++ks == C::kKStages) ks = 0;
                };
                auto load_v = [&](int j) {
                    if (vuse >= (uint32_t)C::kVStages && !err &&
                        !mbar_wait(&v_empty[vs], (vuse / C::kVStages - 1) & 1, p.wait_limit))
                        err = true;
                    mbar_arrive_expect_tx(&v_full[vs], C::kTileBytes);
                    bulk_load(sV + vs * C::kTileBytes, kv_tiles + ((size_t)j * 2 + 1) * C::kTileBytes, C::kTileBytes,
                              &v_full[vs]);
                    ++vuse;
                    if (++vs == C::kVStages) vs = 0;
                };
                load_k(0);
                for (int j = 0; j < nkv; ++j) {
                    if (j + 1 < nkv) load_k(j + 1);
                    load_v(j);
                }
            }
            // every copy has landed before the CTA ends, even after a
            // timeout (bounded waits): the last load of each stage, the last Q
            for (int s = 0; s < C::kKStages; ++s) {
                const uint32_t uses = kuse / C::kKStages + ((uint32_t)s < kuse % C::kKStages ? 1u : 0u);
                if (uses && !mbar_wait(&k_full[s], (uses - 1) & 1u, p.wait_limit)) err = true;
            }
            for (int s = 0; s < C::kVStages; ++s) {
                const uint32_t uses = vuse / C::kVStages + ((uint32_t)s < vuse % C::kVStages ? 1u : 0u);
                if (uses && !mbar_wait(&v_full[s], (uses - 1) & 1u, p.wait_limit)) err = true;
            }
            if (!mbar_wait(q_full, (uint32_t)(t_end - t_begin - 1) & 1u, p.wait_limit)) err = true;
        }
    } else {
        // ------------------------------------------------ softmax warps
        warpgroup_reg_alloc<C::kRegsHigh>();
        const bool headA = warp < C::kSoftB;
        const int quarter = warp & 3;  // TMEM lane quarter this warp may access
        const int t = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        uint32_t it = 0, k = 0;
        for (int ti = t_begin; ti < t_end; ++ti) {
            const PrefillTile tile = p.tiles[ti];
            if (!headA && tile.num_heads != 2) continue;
            int tok0, q_rows, first_pos, pos;
            if (tile.row_base >= 0) {
                // shared prefix: every query sees all keys < key_limit
                tok0 = tile.q_start;
                q_rows = tile.q_rows;
                first_pos = tile.key_limit - 1;
                pos = t < q_rows ? first_pos : 0;
            } else {
                const int seq = tile.seq, q0 = tile.q_start;
                tok0 = p.cu_seqlens_q[seq] + q0;
                const int L = p.cu_seqlens_q[seq + 1] - p.cu_seqlens_q[seq];
                const int n = p.seq_lens[seq];
                q_rows = min(128, L - q0);
                first_pos = n - L + q0;
                pos = t < q_rows ? first_pos + t : 0;  // padding rows see key 0 only
            }
            const int head = tile.head + (headA ? 0 : 1);
            softmax_tile<D>(p, tile.n_kv_tiles, tile.kv_tile0, tile.row_base, tile.piece, trow,
                            headA ? C::kSA : C::kSB, headA ? C::kOA : C::kOB, headA ? sA_full : sB_full,
                            headA ? pA_full : pB_full, headA ? oA_done : oB_done, headA ? oA_free : oB_free, it, k, t,
                            q_rows, pos, first_pos, tok0, head, head % p.group, err);
            ++k;
        }
    }
    if (err) atomicOr(p.status, kStatusWaitTimeout);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on the driver library).
using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn tensor_map_encoder() {
    static std::atomic<EncodeFn> fn{nullptr};
    EncodeFn f = fn.load(std::memory_order_acquire);
    if (f) return f;
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !ptr) {
        cudaGetLastError();
        return nullptr;
    }
    f = reinterpret_cast<EncodeFn>(ptr);
    fn.store(f, std::memory_order_release);
    return f;
}

// bf16 tensor of `rank` dims (innermost first), 128-byte swizzle.
bool encode_bf16(EncodeFn enc, CUtensorMap *map, const void *base, int rank, const cuuint64_t *dims,
                 const cuuint64_t *strides_bytes, const cuuint32_t *box) {
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides_bytes, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_prefill_t(const PrefillParams &p, cudaStream_t stream) {
    using C = PrefillCfg<D>;
    EncodeFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    PrefillMaps maps;
    const cuuint64_t dims[3] = {D, (cuuint64_t)p.num_q_heads, (cuuint64_t)p.num_tokens};
    const cuuint64_t strides[2] = {D * 2ull, (cuuint64_t)p.num_q_heads * D * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    if (!encode_bf16(enc, &maps.q, p.q, 3, dims, strides, box)) return cudaErrorInvalidValue;
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
    prefill_kernel<D><<<p.num_ctas, C::kThreads, C::kSmemBytes, stream>>>(p, maps);
    return cudaGetLastError();
}

}  // namespace

bool prefill_kernel_available() { return true; }

cudaError_t launch_stage(const PrefillParams &p, int head_dim, cudaStream_t stream) {
    if (p.num_stages == 0) return cudaSuccess;
    if (head_dim == 64)
        stage_kernel<64><<<dim3(p.num_stages, 2), 256, 0, stream>>>(p);
    else
        stage_kernel<128><<<dim3(p.num_stages, 2), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillParams &p, int head_dim, cudaStream_t stream) {
    if (p.num_tiles == 0) return cudaSuccess;
    return head_dim == 64 ? launch_prefill_t<64>(p, stream) : launch_prefill_t<128>(p, stream);
}

}  // namespace pa
