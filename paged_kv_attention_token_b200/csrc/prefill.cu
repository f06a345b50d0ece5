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
#include "scatter.cuh"

namespace pa {

namespace {

constexpr float kPrefillRescaleThreshold = 8.f;

// The softmax evaluates 2^x on two pipes: the MUFU unit (ex2.approx) and, for
// the pairs k (0..15) of a 32-column chunk with bit k % 4 set in
// kPolyPairMask, a polynomial on the FMA and integer pipes.  The MUFU unit
// does 16 results per SM clock, so 128 x 128 exponentials per head and
// 128-key step take as long as that step's MMAs; moving part of them to the
// FMA pipe shortens each softmax chain.  Measured on B200: the two-head
// kernel is fastest with the MUFU unit alone; the pair kernel gains ~2 %
// with a quarter of the pairs on the polynomial (half of them: slower).
constexpr uint32_t kPolyPairMask = 0x0;
constexpr uint32_t kPairPolyPairMask = 0x1;
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
template <uint32_t PolyMask = kPolyPairMask>
__device__ __forceinline__ void chunk_exp(const uint32_t (&r)[32], uint32_t (&pk)[16], uint64_t scale2,
                                          uint64_t nm2, bool masked, int key0, int pos) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint64_t x = f2_fma(f2(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), scale2, nm2);
        float e0, e1;
        if ((PolyMask >> (c & 3)) & 1u) {
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
    CUtensorMap out;  // the same shape over the output (pair kernel's stores)
    // pair kernel: the K and V caches as [blocks * 16][Hkv][D], box {64, 1, 16}
    // (one 16-token block of one kv head, one 64-dim slab), 128-byte swizzle
    CUtensorMap k, v;
    // pair kernel, fused step: this step's K and V as [T][Hkv][D], box
    // {64, 1, 64} (64 tokens of one kv head, one 64-dim slab), 128-byte
    // swizzle: the layout of a staged tile's rows
    CUtensorMap kn, vn;
};

// Gathers staged tile `tile` (K for kv = 0, V for 1) from the paged cache:
// 16-byte chunks, rows of one kv head's keys, swizzled as the prefill
// kernel's shared-memory tiles; rows past the keys are zeroed.  With `fresh`
// (a fused step's own K or V, [T][Hkv][D]), keys written by this step come
// from it instead of their cache slots: key k of segment i is token
// cu_seqlens_q[i] + k - (seq_lens[i] - q_len) when it is one of the last
// q_len keys.
template <int D>
__device__ __forceinline__ void stage_tile(const PrefillParams &p, int tile, int kv, const __nv_bfloat16 *fresh,
                                           int tid, int nthreads) {
    constexpr int kRowChunks = D / 8;
    const StageTile st = p.stages[tile];
    const int n = st.n_keys;
    const int32_t *bt_row = p.block_tables + (size_t)st.seq * p.max_blocks_per_seq;
    const __nv_bfloat16 *cache = kv ? p.v_cache : p.k_cache;
    uint8_t *dst = p.staged + ((size_t)tile * 2 + kv) * (128 * D * 2);
    int first_new = INT32_MAX, tok_base = 0;  // keys from first_new on are this step's tokens
    if (fresh != nullptr) {
        const int c0 = __ldg(p.cu_seqlens_q + st.seq), c1 = __ldg(p.cu_seqlens_q + st.seq + 1);
        first_new = __ldg(p.seq_lens + st.seq) - (c1 - c0);
        tok_base = c0 - first_new;
        // the pair kernel reads a tile of this step's keys only from the input
        if (p.pair && 128 * st.tile >= first_new) return;
    }
    for (int c = tid; c < 128 * kRowChunks; c += nthreads) {
        const int row = c / kRowChunks, ch = c % kRowChunks;
        const int key = 128 * st.tile + row;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (key < n) {
            if (key >= first_new) {
                v = ld_stream16(fresh + ((size_t)(tok_base + key) * p.num_kv_heads + st.kv_head) * D + ch * 8);
            } else {
                const int blk = __ldg(bt_row + (key >> 4));
                v = ld_stream16(cache + (((size_t)blk * kBlockSize + (key & 15)) * p.num_kv_heads + st.kv_head) * D +
                                ch * 8);
            }
        }
        st16(dst + (ch >> 3) * 16384 + row * 128 + (((ch & 7) ^ (row & 7)) << 4), v);
    }
}

// Gathers staged tile blockIdx.x (K for blockIdx.y = 0, V for 1).
template <int D>
__global__ void __launch_bounds__(256) stage_kernel(const __grid_constant__ PrefillParams p) {
    stage_tile<D>(p, blockIdx.x, blockIdx.y, nullptr, threadIdx.x, 256);
}

// A fused step's cache write and staging in one launch: blocks below
// scatter_blocks write this step's K/V into their slots, each block above
// gathers one staged tile's K or V (its own keys from k / v).
template <int D>
__global__ void __launch_bounds__(256)
    scatter_stage_kernel(const __grid_constant__ ScatterArgs a, const __grid_constant__ PrefillParams p,
                         int scatter_blocks) {
    // a decode kernel queued next may set up while this runs
    grid_launch_dependents();
    const int cpt = a.token_elems / 8;
    if ((int)blockIdx.x < scatter_blocks) {
        scatter_chunks(static_cast<const uint4 *>(a.k), static_cast<const uint4 *>(a.v), a.slots,
                       static_cast<uint4 *>(a.k_cache), static_cast<uint4 *>(a.v_cache), a.num_tokens * cpt, cpt,
                       a.num_slots, (int64_t)blockIdx.x * 256 + threadIdx.x, (int64_t)scatter_blocks * 256);
        return;
    }
    const int i = blockIdx.x - scatter_blocks;
    stage_tile<D>(p, i >> 1, i & 1, static_cast<const __nv_bfloat16 *>((i & 1) ? a.v : a.k), threadIdx.x, 256);
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

    // a decode kernel launched programmatically behind this one may place its
    // CTAs on the other SMs now (it reads nothing this kernel writes)
    grid_launch_dependents();
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
    PrefillMaps maps{};
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

// ---------------------------------------------------------------------------
// Pair kernel (head_dim 128): one tile per cluster of two CTAs on two SMs.
// The CTA of cluster rank r holds head A + r of the tile, and every product
// runs as one MMA over both SMs (tcgen05 with cta_group::2, M = 256).
//
// The two-head kernel above keeps both heads of a tile in one SM's 512 TMEM
// columns, so each head has a single S buffer and its loop S(j) -> softmax
// -> PV(j) -> S(j + 1) is serial.  Here each SM holds one head: two S
// buffers (256 columns) and two accumulators (below).  S(j + 2) is computed
// into the buffer P(j) occupied, right after PV(j), so the softmax finds the
// next S ready.
//
// A 2-SM MMA takes the 256 rows of A from both CTAs (rows 0-127 from rank 0,
// 128-255 from rank 1: the two heads' Q in shared memory, or their P in
// TMEM), splits B by its N columns (rank r holds columns N/2 r ..
// N/2 r + N/2 - 1) and writes each CTA's 128 rows of D into that CTA's TMEM.
// So for S = Q K^T rank r loads keys 64 r .. 64 r + 63 of a K tile, and for
// O += P V dims 64 r .. 64 r + 63 of a V tile: each K/V byte crosses from L2
// into shared memory once per pair, and each SM's MMAs read half of B.  Per
// 128-key step and SM that is 32 KB of loads and 64 KB of operand reads
// beside the 1024 tensor cycles of the step's two products; a single SM
// holding both heads moves 256 KB per two such steps.
//
// Rank 0 issues every MMA (one warp, one elected lane) and owns the barriers
// that gate them: a K/V stage or Q is ready once a forwarding warp in each
// CTA has seen that CTA's copy land and arrived on rank 0's barrier; P and
// the release of O wait for the softmax warps of both CTAs (remote
// arrivals).  Every commit
// arrives in both CTAs (tcgen05.commit cta_group::2 with cluster multicast),
// so each CTA's loader, softmax warps and epilogue wait on barriers of their
// own.  No TMA or bulk load uses cluster multicast.
//
// Eight softmax warps per CTA split every query row into two halves of 64
// keys (warps 4-7 and 8-11 share TMEM lanes).  Each half is an online
// softmax of its own, with its own running max and sum and its own
// accumulator in TMEM (O_0 for keys 0-63 of every step, O_1 for 64-127), so
// the two warps on an SM sub-partition never wait for each other within a
// tile; the halves combine once per tile.
//
// A prefill segment's K/V come from staged tiles; a shared prefix's straight
// from the paged cache (TMA boxes of one 16-token block), see the loader.
// ---------------------------------------------------------------------------
struct PairCfg {
    static constexpr int D = 128;
    static constexpr int kThreads = 384;
    static constexpr int kSoftHi = 8;                      // warps 4-7: keys 0-63 of a step, warps 8-11: 64-127
    static constexpr int kTileBytes = 128 * D * 2;         // a staged K or V tile (two 64-dim slabs of 16 KB)
    static constexpr int kQBytes = 128 * D * 2;            // Q of this CTA's head
    static constexpr int kKBytes = 64 * D * 2;             // this CTA's 64 keys of a K tile (8 KB of each slab)
    static constexpr int kVBytes = 128 * 64 * 2;           // this CTA's 64 dims of a V tile (one slab)
    static constexpr int kKStages = 5;
    static constexpr int kVStages = 4;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQBytes;
    static constexpr int kVOff = kKOff + kKStages * kKBytes;
    static constexpr int kXchOff = kVOff + kVStages * kVBytes;  // float [2 slots][2 halves][128 rows]
    static constexpr int kOutOff = kXchOff + 2 * 2 * 128 * 4;   // bf16 output tile: two 64-dim slabs, 128-byte swizzle
    static constexpr int kBarOff = kOutOff + 128 * D * 2;
    // mbarriers.  "land": this CTA's copy arrived (its own loads' bytes);
    // "ready": both CTAs' copies arrived (used in rank 0, one arrival per
    // CTA); "empty": the MMAs reading a stage completed (multicast commit).
    static constexpr int kBarQLand = 0, kBarQReady = 1, kBarQEmpty = 2;
    static constexpr int kBarKLand = 3;
    static constexpr int kBarKReady = kBarKLand + kKStages;
    static constexpr int kBarKEmpty = kBarKReady + kKStages;
    static constexpr int kBarVLand = kBarKEmpty + kKStages;
    static constexpr int kBarVReady = kBarVLand + kVStages;
    static constexpr int kBarVEmpty = kBarVReady + kVStages;
    static constexpr int kSBufs = 2;                       // S buffers in TMEM
    static constexpr int kBarS = kBarVEmpty + kVStages;    // [kSBufs]: S of the step in TMEM buffer b
    static constexpr int kBarP = kBarS + kSBufs;           // [kSBufs][2]: P of half h in buffer b, both CTAs (rank 0)
    static constexpr int kBarPV = kBarP + 2 * kSBufs;      // [2]: the PV product of half h completed
    static constexpr int kBarO = kBarPV + 2;               // the tile's last PV products completed
    static constexpr int kBarOFree = kBarO + 1;            // both CTAs read O (rank 0)
    static constexpr int kBarDrain = kBarOFree + 1;        // every MMA issued completed
    static constexpr int kNumBars = kBarDrain + 1;
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
    static constexpr int kUsed = kTmemSlotOff + 16;
    static constexpr int kSmemBytes = kUsed + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kSmemBytes > 116 * 1024, "one CTA per SM");
    static constexpr uint32_t kTmemCols = 512;
    // S buffers at 0 and 128; the accumulators O_0 (keys 0-63 of every
    // step) at 256 and O_1 (keys 64-127) at 384
    static constexpr uint32_t kS = 0, kO = 256;
    static constexpr int kLaunchRegs = 168;
    static constexpr int kRegsLow = 104;
    static constexpr int kRegsHigh = 200;
    static_assert(128 * kRegsLow + 256 * kRegsHigh <= 384 * kLaunchRegs, "register split");
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrival on an mbarrier of any CTA of the cluster (shared::cluster address),
// with the default semantics (release at CTA scope).  Measured on B200, an
// arrival with .release.cluster costs its thread ~1000 cycles; the data it
// hands over is TMEM (completed by tcgen05.wait::st and ordered by
// tcgen05.fence::before_thread_sync) or the other CTA's own copies, whose
// completion the arriving thread observed on its mbarrier.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// TMEM allocation shared by the two CTAs (one warp of each executes it).
__device__ __forceinline__ void tmem_alloc_pair(uint32_t smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_dst), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// One lane of the (converged) warp: 1 there, 0 elsewhere.
__device__ __forceinline__ uint32_t elect_one() {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b32 l;\n\t"
        "elect.sync l|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r));
    return r;
}
// The MMA helpers below are executed by a whole warp with the operands
// warp-uniform; only the lane with `issue` != 0 issues the instruction.
// 2-SM MMA, A and B in shared memory (same offsets in both CTAs).
__device__ __forceinline__ void umma_pair_ss(uint32_t issue, uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %6, 0;\n\t"
        "@q tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(issue));
}
// 2-SM MMA, A in TMEM (each CTA's 128 rows), B in shared memory.
__device__ __forceinline__ void umma_pair_ts(uint32_t issue, uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %6, 0;\n\t"
        "@q tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n\t}" ::"r"(
            d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(issue));
}
// Arrives once on `bar` in both CTAs when every MMA issued so far is
// complete (issued by the lane with `issue` != 0).
__device__ __forceinline__ void umma_commit_pair(uint32_t issue, uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred q;\n\t"
        "setp.ne.b32 q, %2, 0;\n\t"
        "@q tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::"r"(
            smem_u32(bar)),
        "h"((uint16_t)3), "r"(issue)
        : "memory");
}
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// 3-D tiled TMA store (no multicast) of a shared-memory box, tracked in this
// thread's bulk async-group; c0 must be a multiple of 8 bf16 elements.
__device__ __forceinline__ void tma_store_3d(const void *map, uint32_t src, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until the shared memory of this thread's bulk stores has been read.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Softmax of one tile for this thread's half row: keys 64 half .. + 63 of
// every step, as an online softmax of its own (running max m, sum l and the
// accumulator O_half in TMEM), so that the two warps on an SM sub-partition
// never wait for each other within a tile.  The halves combine at the end:
// with M = max(m0, m1), O = (O_0 2^(m0 - M) + O_1 2^(m1 - M)) / (l0 2^(m0 - M)
// + l1 2^(m1 - M)).  g counts the steps over the CTA's tiles, (sb, sph) the
// TMEM buffer of the next step and the phase of its barriers, k the tiles,
// e the end-of-tile exchanges with the partner thread (same row, other half).
// p_full0 and o_free0 are rank 0's barriers (shared::cluster addresses);
// out_stage is the shared-memory staging of the output tile, stored through
// out_map.
__device__ __forceinline__ void pair_softmax_tile(const PrefillParams &p, const PrefillTile &tile, uint32_t trow,
                                                  int half, float *xch, uint64_t *s_full, uint32_t p_full0,
                                                  uint64_t *pv_done, uint64_t *o_done, uint32_t o_free0, uint32_t &g,
                                                  uint32_t &sb, uint32_t &sph, uint32_t k, const CUtensorMap *out_map,
                                                  uint32_t out_stage, uint32_t &e, int t, int quarter, int q_rows,
                                                  int pos, int first_pos, int tok0, int head, int hl, bool &err) {
    using C = PairCfg;
    constexpr int D = C::D;
    constexpr int kHalfO = D / 2;  // output columns of this thread
    const uint32_t o_mine = C::kO + 128 * half;
    float m = -INFINITY, l = 0.f;
    const uint64_t scale2 = f2(p.scale_log2, p.scale_log2);
    auto exchange = [&](float v) {  // the partner thread's value of v
        float *slot = xch + (e & 1u) * 256;
        slot[half * 128 + t] = v;
        named_sync(1 + quarter, 64);
        const float o = slot[(half ^ 1) * 128 + t];
        ++e;
        return o;
    };
    for (int j = 0; j < tile.n_kv_tiles; ++j, ++g) {
        const uint32_t b = sb;
        if (!err && !mbar_wait(&s_full[b], sph, p.wait_limit)) err = true;
        if (++sb == C::kSBufs) { sb = 0; sph ^= 1u; }
        tc_fence_after();
        const int kbase = 128 * (tile.kv_tile0 + j) + 64 * half;  // first key of this half step
        const bool masked = kbase + 63 > first_pos;
        // S of this half in columns 64 half .. + 63; its P (bf16 pairs) goes
        // to columns 64 half .. + 31, which no other thread reads
        const uint32_t s_col = C::kS + 128 * b + 64 * half;
        uint32_t s0[32], s1[32];
        tmem_ld32(trow + s_col, s0);
        tmem_ld32(trow + s_col + 32, s1);
        tmem_ld_wait();
        const float mx =
            fmaxf(chunk_max(s0, masked, kbase, pos), chunk_max(s1, masked, kbase + 32, pos)) * p.scale_log2;
        float alpha = 1.f;
        const bool rescale = mx > m + kPrefillRescaleThreshold;
        if (rescale) {
            alpha = fast_exp2(m - mx);
            m = mx;
        }
        const uint64_t nm2 = f2(-m, -m);
        uint32_t pk0[16], pk1[16];
        chunk_exp<kPairPolyPairMask>(s0, pk0, scale2, nm2, masked, kbase, pos);
        tmem_st16(trow + s_col, pk0);
        chunk_exp<kPairPolyPairMask>(s1, pk1, scale2, nm2, masked, kbase + 32, pos);
        tmem_st16(trow + s_col + 16, pk1);
        // O_half is rescaled after the previous step's PV product for this
        // half completed and before this step's P is handed over
        if (j > 0 && __any_sync(kFullMask, rescale)) {
            if (!err && !mbar_wait(&pv_done[half], (g - 1) & 1u, p.wait_limit)) err = true;
            tc_fence_after();
#pragma unroll
            for (int i = 0; i < D / 32; ++i) {
                uint32_t o[32];
                tmem_ld32(trow + o_mine + 32 * i, o);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                tmem_st32(trow + o_mine + 32 * i, o);
            }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive_remote(p_full0 + 8 * (2 * b + half));
        // the sum of the rounded P values the PV product uses
        regs_after(pk0);
        regs_after(pk1);
        float l0, l1;
        f2_split(f2_add(chunk_sum(pk0), chunk_sum(pk1)), l0, l1);
        l = l * alpha + (l0 + l1);
    }
    if (!err && !mbar_wait(o_done, k & 1u, p.wait_limit)) err = true;
    tc_fence_after();
    // both halves of the row: the same maximum M and sum L in both threads
    const float m_o = exchange(m), l_o = exchange(l);
    const float mm = fmaxf(m, m_o);
    const float c_me = fast_exp2(m - mm), c_o = fast_exp2(m_o - mm);
    const float lsum = l * c_me + l_o * c_o;
    // output columns kHalfO half .. + kHalfO - 1 from both accumulators
    const uint32_t o_other = C::kO + 128 * (half ^ 1);
    uint32_t o[kHalfO / 32][32];
#pragma unroll
    for (int i = 0; i < kHalfO / 32; ++i) {
        uint32_t x[32];
        tmem_ld32(trow + o_mine + kHalfO * half + 32 * i, o[i]);
        tmem_ld32(trow + o_other + kHalfO * half + 32 * i, x);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c)
            o[i][c] = __float_as_uint(__uint_as_float(o[i][c]) * c_me + __uint_as_float(x[c]) * c_o);
    }
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive_remote(o_free0);
    if (tile.row_base >= 0) {
        // Partials of decode rows, one row per thread, each row's 64 values at
        // its own slot: they go out through a 4 KB region of the output
        // staging per warp, 32 dims at a time, so that each store instruction
        // writes four rows' whole 128-byte pieces instead of 32 scattered
        // 16-byte ones.
        const int G = p.group;
        float *po = nullptr;
        if (t < q_rows) {
            const int r = tile.row_base + t * p.num_kv_heads;
            const int slot = p.combine[p.rows[r].combine].piece_base + tile.piece;
            po = p.partial_o + ((size_t)slot * G + hl) * D + kHalfO * half;
            if (half == 0) p.partial_ml[(size_t)slot * G + hl] = make_float2(mm, lsum);
        }
        const bool issuer = (threadIdx.x & 127) == 0;
        if (issuer) bulk_wait_read();  // a previous tile's output store has read the staging
        named_sync(5 + half, 128);
        const int lane = threadIdx.x & 31;
        const uint32_t region = out_stage + ((threadIdx.x >> 5) - 4) * 4096;
#pragma unroll
        for (int i = 0; i < kHalfO / 32; ++i) {
            // row `lane` of the warp: 32 floats, 16-byte chunk c at c ^ (lane % 8)
#pragma unroll
            for (int c = 0; c < 8; ++c)
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(region + lane * 128 + ((c ^ (lane & 7)) << 4)),
                             "r"(o[i][4 * c]), "r"(o[i][4 * c + 1]), "r"(o[i][4 * c + 2]), "r"(o[i][4 * c + 3])
                             : "memory");
            __syncwarp();
#pragma unroll
            for (int s4 = 0; s4 < 8; ++s4) {
                const int row = 4 * s4 + (lane >> 3), c = lane & 7;
                float *dst = reinterpret_cast<float *>(
                    __shfl_sync(kFullMask, reinterpret_cast<unsigned long long>(po), row));
                const uint4 v = ld_shared16(region + row * 128 + ((c ^ (row & 7)) << 4));
                if (dst != nullptr) st16(dst + 32 * i + 4 * c, v);
            }
            __syncwarp();
        }
        return;
    }
    const float inv = 1.f / lsum;
    if (q_rows == 128) {
        // A full tile: the half rows go through shared memory (the 128-byte
        // swizzled box of the output's tensor map) and leave as one TMA
        // store per half, so that the rows' scattered 16-byte pieces become
        // whole lines and the warps need not wait for them.
        const uint32_t slab = out_stage + half * 16384;
        const bool issuer = (threadIdx.x & 127) == 0;
        if (issuer) bulk_wait_read();  // the previous tile's store has read the slab
        named_sync(5 + half, 128);
#pragma unroll
        for (int i = 0; i < kHalfO / 32; ++i) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(o[i][8 * c + 0]) * inv, __uint_as_float(o[i][8 * c + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(o[i][8 * c + 2]) * inv, __uint_as_float(o[i][8 * c + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(o[i][8 * c + 4]) * inv, __uint_as_float(o[i][8 * c + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(o[i][8 * c + 6]) * inv, __uint_as_float(o[i][8 * c + 7]) * inv);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(swz128(slab, t, 4 * i + c)), "r"(w.x),
                             "r"(w.y), "r"(w.z), "r"(w.w)
                             : "memory");
            }
        }
        fence_proxy_async_smem();
        named_sync(5 + half, 128);
        if (issuer) tma_store_3d(out_map, slab, 64 * half, head, tok0);
        return;
    }
    if (t < q_rows) {
        __nv_bfloat16 *orow = p.out + ((size_t)(tok0 + t) * p.num_q_heads + head) * D + kHalfO * half;
#pragma unroll
        for (int i = 0; i < kHalfO / 32; ++i) {
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

// Cluster c (CTAs 2c and 2c + 1) works through tiles [cta_start[c],
// cta_start[c + 1]); every tile has two heads.  Both CTAs run the same tile
// list, so they take the same K/V stages in the same order and both reach
// every cluster barrier.
__global__ void __launch_bounds__(384, 1)
    prefill_pair_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps maps) {
    using C = PairCfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    // the same 1024-aligned offset in both CTAs: the 2-SM MMAs read both
    // CTAs' operands through one descriptor
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(smem + C::kQOff);
    const uint32_t sK = smem_u32(smem + C::kKOff);
    const uint32_t sV = smem_u32(smem + C::kVOff);
    float *xch = reinterpret_cast<float *>(smem + C::kXchOff);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *q_land = bars + C::kBarQLand, *q_ready = bars + C::kBarQReady, *q_empty = bars + C::kBarQEmpty;
    uint64_t *k_land = bars + C::kBarKLand, *k_ready = bars + C::kBarKReady, *k_empty = bars + C::kBarKEmpty;
    uint64_t *v_land = bars + C::kBarVLand, *v_ready = bars + C::kBarVReady, *v_empty = bars + C::kBarVEmpty;
    uint64_t *s_full = bars + C::kBarS, *p_full = bars + C::kBarP, *pv_done = bars + C::kBarPV;
    uint64_t *o_done = bars + C::kBarO, *o_free = bars + C::kBarOFree, *drain = bars + C::kBarDrain;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kTmemSlotOff);

    // a decode kernel launched programmatically behind this one may place its
    // CTAs on the other SMs now (it reads nothing this kernel writes)
    grid_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const int cl = blockIdx.x >> 1;
    // (the launch has exactly num_ctas clusters; a cluster with no tiles
    // still takes every cluster barrier below)
    const int t_begin = p.cta_start[cl], t_end = p.cta_start[cl + 1];

    if (tid == 0) {
        mbar_init(q_land, 1);
        mbar_init(q_ready, 2);  // one forwarder per CTA
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::kKStages; ++s) {
            mbar_init(&k_land[s], 1);
            mbar_init(&k_ready[s], 2);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::kVStages; ++s) {
            mbar_init(&v_land[s], 1);
            mbar_init(&v_ready[s], 2);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < C::kSBufs; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[2 * b], 8);  // one arrival per softmax warp of the half, both CTAs
            mbar_init(&p_full[2 * b + 1], 8);
        }
        mbar_init(&pv_done[0], 1);
        mbar_init(&pv_done[1], 1);
        mbar_init(o_done, 1);
        mbar_init(o_free, 16);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // both CTAs' barriers are initialised before either touches the other's
    cluster_sync();
    const uint32_t tmem = *tmem_slot;
    bool err = false;
    // rank 0's copy of a barrier of this CTA's layout
    auto at_rank0 = [](uint64_t *bar) { return peer_addr(smem_u32(bar), 0); };

    if (warp < 4) {
        warpgroup_reg_dealloc<C::kRegsLow>();
        if (warp == 0 && rank == 0) {
            // ------------------------------------------------ MMA issuer (rank 0, warp 0; one lane issues)
            //   S(j) = Q K_j^T (M 256, N 128, K D) into TMEM buffer j % 2,
            //   PV_h(j): O_h += P_h(j) V_h,j (M 256, N D, K 64: keys
            //   64 h .. 64 h + 63 of the step, A = P from TMEM),
            // issued S(0) S(1) | PV_0(0) PV_1(0) S(2) | PV_0(1) PV_1(1) S(3)
            // | ...: each half's PV goes as soon as that half's P is there,
            // and S(j + 2) reuses the buffer both PV(j) have just read
            // (tcgen05 MMAs of one thread run in issue order).
            const uint32_t me = elect_one();
            constexpr uint32_t idesc_s = umma_idesc_bf16_f32(256, 128, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(256, D, false, true);
            const uint64_t dQ = umma_desc_sw128(sQ, 16, 1024);
            const uint64_t dK = umma_desc_sw128(sK, 16, 1024), dV = umma_desc_sw128(sV, 16384, 1024);
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                if (!err && !mbar_wait(bar, parity, p.wait_limit)) err = true;
            };
            int vs = 0, ks = 0;
            uint32_t vph = 0, kph = 0;
            uint32_t k = 0;                           // tiles so far
            uint32_t sb = 0, pb = 0, pph = 0;         // buffer of the next S, of the next P and its phase
            for (int ti = t_begin; ti < t_end; ++ti) {
                const PrefillTile tile = p.tiles[ti];
                const int n = tile.n_kv_tiles;
                int s_issued = 0;
                auto issue_s = [&]() {
                    wait(&k_ready[ks], kph);
                    tc_fence_after();
                    const uint64_t dk = dK + ks * (uint32_t)(C::kKBytes >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        // 16 dims = 32 bytes along a 128-byte row; 64-dim slabs
                        // 16 KB apart in Q, 8 KB apart in this CTA's K half
                        const uint32_t q_off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                        const uint32_t k_off = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
                        umma_pair_ss(me, tmem + C::kS + 128 * sb, dQ + q_off, dk + k_off, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit_pair(me, &s_full[sb]);
                    umma_commit_pair(me, &k_empty[ks]);
                    if (++ks == C::kKStages) { ks = 0; kph ^= 1u; }
                    if (++sb == C::kSBufs) sb = 0;
                    // the tile's last S product releases Q
                    if (++s_issued == n) umma_commit_pair(me, q_empty);
                };
                wait(q_ready, (uint32_t)(ti - t_begin) & 1u);
                for (int j = 0; j < C::kSBufs && j < n; ++j) issue_s();
                for (int j = 0; j < n; ++j) {
                    const uint64_t dv = dV + vs * (uint32_t)(C::kVBytes >> 4);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        wait(&p_full[2 * pb + h], pph);
                        if (h == 0) {
                            if (j == 0 && k > 0) wait(o_free, (k - 1) & 1u);
                            wait(&v_ready[vs], vph);
                        }
                        tc_fence_after();
                        // P_h: bf16 pairs in columns 64 h .. + 31 of the buffer;
                        // V rows (keys) 64 h + 16 kk .. + 15, 128 bytes each
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_pair_ts(me, tmem + C::kO + 128 * h, tmem + C::kS + 128 * pb + 64 * h + 8 * kk,
                                         dv + (((64 * h + 16 * kk) * 128) >> 4), idesc_pv, kk > 0 || j > 0 ? 1u : 0u);
                        umma_commit_pair(me, &pv_done[h]);
                    }
                    if (j + 1 == n) umma_commit_pair(me, o_done);
                    umma_commit_pair(me, &v_empty[vs]);
                    if (++vs == C::kVStages) { vs = 0; vph ^= 1u; }
                    if (++pb == C::kSBufs) { pb = 0; pph ^= 1u; }
                    if (j + C::kSBufs < n) issue_s();
                }
                ++k;
            }
            umma_commit_pair(me, drain);
            if (!mbar_wait(drain, 0, p.wait_limit)) err = true;
        } else if (warp == 0 && lane == 0) {
            // rank 1: the last commit (and with it every earlier one) has
            // arrived here before the CTA may end
            if (!mbar_wait(drain, 0, p.wait_limit)) err = true;
        } else if (warp == 1 && lane == 0) {
            // ------------------------------------------------ loads (both CTAs)
            // In the order the MMAs consume them, per tile: Q, K0 K1, V0 K2,
            // V1 K3 ...  A stage is reloaded once the MMAs that read it (in both
            // CTAs) completed.  A prefill segment's K/V come from its staged
            // tiles (bulk copies of this CTA's halves); a shared prefix's
            // straight from the paged cache, one TMA box per 16-token block
            // and 64-dim slab at the block's id from the block table, blocks
            // past the keys not loaded (the forwarder zeroes what the V tile
            // needs zeroed).  Staging pays where many query tiles read the
            // same keys (a segment's); a prefix's tiles read each key tile
            // once per head pair.
            int vs = 0, ks = 0;
            uint32_t vuse = 0, kuse = 0;
            for (int ti = t_begin; ti < t_end; ++ti) {
                const PrefillTile tile = p.tiles[ti];
                const int n = tile.n_kv_tiles;
                const int tok0 = tile.row_base >= 0 ? tile.q_start : p.cu_seqlens_q[tile.seq] + tile.q_start;
                if (ti > t_begin && !err &&
                    !mbar_wait(q_empty, (uint32_t)(ti - t_begin - 1) & 1u, p.wait_limit))
                    err = true;
                mbar_arrive_expect_tx(q_land, C::kQBytes);
#pragma unroll
                for (int s = 0; s < D / 64; ++s)
                    tma_load_3d(sQ + s * 16384, &maps.q, q_land, 64 * s, tile.head + (int)rank, tok0);
                // the keys' segment (or shared prefix), kv head and length
                const bool gather = tile.row_base >= 0;
                const StageTile src = p.stages[tile.kv_base];
                const int32_t *bt = p.block_tables + (size_t)src.seq * p.max_blocks_per_seq;
                const int nblk = (src.n_keys + kBlockSize - 1) / kBlockSize;
                const uint8_t *kv = p.staged + (size_t)tile.kv_base * 2 * C::kTileBytes;  // segments only
                // a fused step: the segment's key tiles from first_new / 128 on
                // hold only this step's tokens and come straight from its K/V
                // input (key k is token key_tok + k), as 64-row boxes
                int first_new = INT32_MAX, key_tok = 0;
                if (!gather && p.k_new != nullptr) {
                    const int c0 = p.cu_seqlens_q[tile.seq], c1 = p.cu_seqlens_q[tile.seq + 1];
                    first_new = p.seq_lens[tile.seq] - (c1 - c0);
                    key_tok = c0 - first_new;
                }
                const int kv_head = tile.head / p.group;
                auto load_k = [&](int t) {  // key tile t: this CTA's keys 64 rank .. + 63
                    if (kuse >= (uint32_t)C::kKStages && !err &&
                        !mbar_wait(&k_empty[ks], (kuse / C::kKStages - 1) & 1u, p.wait_limit))
                        err = true;
                    if (!gather && 128 * t >= first_new) {
                        mbar_arrive_expect_tx(&k_land[ks], C::kKBytes);
#pragma unroll
                        for (int s = 0; s < D / 64; ++s)
                            tma_load_3d(sK + ks * C::kKBytes + s * 8192, &maps.kn, &k_land[ks], 64 * s, kv_head,
                                        key_tok + 128 * t + 64 * (int)rank);
                        ++kuse;
                        if (++ks == C::kKStages) ks = 0;
                        return;
                    }
                    if (!gather) {
                        const uint8_t *kt = kv + (size_t)t * 2 * C::kTileBytes;
                        mbar_arrive_expect_tx(&k_land[ks], C::kKBytes);
#pragma unroll
                        for (int s = 0; s < D / 64; ++s)
                            bulk_load(sK + ks * C::kKBytes + s * 8192, kt + s * 16384 + rank * 8192, 8192,
                                      &k_land[ks]);
                        ++kuse;
                        if (++ks == C::kKStages) ks = 0;
                        return;
                    }
                    const int b0 = 8 * t + 4 * (int)rank;
                    int id[4];
                    uint32_t bytes = 0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        id[i] = b0 + i < nblk ? __ldg(bt + b0 + i) : 0;
                        bytes += b0 + i < nblk ? 2 * 2048 : 0;
                    }
                    mbar_arrive_expect_tx(&k_land[ks], bytes);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (b0 + i < nblk)
#pragma unroll
                            for (int s = 0; s < D / 64; ++s)
                                tma_load_3d(sK + ks * C::kKBytes + s * 8192 + i * 2048, &maps.k, &k_land[ks], 64 * s,
                                            src.kv_head, id[i] * kBlockSize);
                    ++kuse;
                    if (++ks == C::kKStages) ks = 0;
                };
                auto load_v = [&](int t) {  // key tile t: dims 64 rank .. + 63 of its 128 keys
                    if (vuse >= (uint32_t)C::kVStages && !err &&
                        !mbar_wait(&v_empty[vs], (vuse / C::kVStages - 1) & 1u, p.wait_limit))
                        err = true;
                    if (!gather && 128 * t >= first_new) {
                        mbar_arrive_expect_tx(&v_land[vs], C::kVBytes);
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tma_load_3d(sV + vs * C::kVBytes + h * 8192, &maps.vn, &v_land[vs], 64 * (int)rank,
                                        kv_head, key_tok + 128 * t + 64 * h);
                        ++vuse;
                        if (++vs == C::kVStages) vs = 0;
                        return;
                    }
                    if (!gather) {
                        const uint8_t *vt = kv + ((size_t)t * 2 + 1) * C::kTileBytes;
                        mbar_arrive_expect_tx(&v_land[vs], C::kVBytes);
                        bulk_load(sV + vs * C::kVBytes, vt + rank * 16384, C::kVBytes, &v_land[vs]);
                        ++vuse;
                        if (++vs == C::kVStages) vs = 0;
                        return;
                    }
                    const int b0 = 8 * t;
                    int id[8];
                    uint32_t bytes = 0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        id[i] = b0 + i < nblk ? __ldg(bt + b0 + i) : 0;
                        bytes += b0 + i < nblk ? 2048 : 0;
                    }
                    mbar_arrive_expect_tx(&v_land[vs], bytes);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (b0 + i < nblk)
                            tma_load_3d(sV + vs * C::kVBytes + i * 2048, &maps.v, &v_land[vs], 64 * (int)rank,
                                        src.kv_head, id[i] * kBlockSize);
                    ++vuse;
                    if (++vs == C::kVStages) vs = 0;
                };
                for (int j = 0; j < C::kSBufs && j < n; ++j) load_k(tile.kv_tile0 + j);
                for (int j = 0; j < n; ++j) {
                    load_v(tile.kv_tile0 + j);
                    if (j + C::kSBufs < n) load_k(tile.kv_tile0 + j + C::kSBufs);
                }
            }
        } else if (warp == 2) {
            // ------------------------------------------------ forwarder (both CTAs, one warp)
            // Walks the loads in the loader's order; once this CTA's copy has
            // landed it arrives on rank 0's ready barrier.  A V tile that
            // reaches past the keys first gets its rows from the last key on
            // zeroed (the blocks past the keys were not loaded, and the last
            // block's slots past the keys may hold anything, NaN included,
            // which P = 0 would not cancel).  Having waited for every landing,
            // the warp also guarantees that no copy into this CTA is in
            // flight when the CTA ends.
            int vs = 0, ks = 0;
            uint32_t vuse = 0, kuse = 0;
            auto fwd = [&](uint64_t *land, uint64_t *ready, uint32_t parity) {
                if (!mbar_wait(land, parity, p.wait_limit)) err = true;
                if (lane == 0) mbar_arrive_remote(at_rank0(ready));
            };
            auto fwd_k = [&]() {
                fwd(&k_land[ks], &k_ready[ks], (kuse / C::kKStages) & 1u);
                ++kuse;
                if (++ks == C::kKStages) ks = 0;
            };
            auto fwd_v = [&](int keys) {  // keys of the tile that exist (<= 128)
                if (!mbar_wait(&v_land[vs], (vuse / C::kVStages) & 1u, p.wait_limit)) err = true;
                if (keys < 128) {
                    const uint32_t stage = sV + vs * C::kVBytes;
                    for (int c = keys * 8 + lane; c < 128 * 8; c += 32)  // 16-byte chunks of 128-byte rows
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(stage + 16 * c), "r"(0u)
                                     : "memory");
                    fence_proxy_async_smem();  // the zeros, before the tensor cores read the tile
                    __syncwarp();
                }
                if (lane == 0) mbar_arrive_remote(at_rank0(&v_ready[vs]));
                ++vuse;
                if (++vs == C::kVStages) vs = 0;
            };
            for (int ti = t_begin; ti < t_end; ++ti) {
                const PrefillTile tile = p.tiles[ti];
                const int n = tile.n_kv_tiles;
                // (staged tiles have their rows past the keys zeroed already;
                // a tile read from the step's input has the next tokens' rows
                // there, or zeros past the input's end)
                const int n_keys = tile.row_base >= 0 ? p.stages[tile.kv_base].n_keys
                                   : p.k_new != nullptr ? p.seq_lens[tile.seq]
                                                        : 1 << 30;
                fwd(q_land, q_ready, (uint32_t)(ti - t_begin) & 1u);
                for (int j = 0; j < C::kSBufs && j < n; ++j) fwd_k();
                for (int j = 0; j < n; ++j) {
                    fwd_v(min(128, n_keys - 128 * (tile.kv_tile0 + j)));
                    if (j + C::kSBufs < n) fwd_k();
                }
            }
        }
    } else {
        // ------------------------------------------------ softmax warps (both CTAs)
        warpgroup_reg_alloc<C::kRegsHigh>();
        const int half = warp < C::kSoftHi ? 0 : 1;
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t p_full0 = at_rank0(p_full), o_free0 = at_rank0(o_free);
        uint32_t g = 0, sb = 0, sph = 0, k = 0, e = 0;
        // a tile's rows; the next tile's are read from global memory while
        // the current one is worked on
        struct Rows {
            PrefillTile tile;
            int tok0, q_rows, first_pos, pos;
        };
        auto rows_of = [&](int ti) {
            Rows r;
            r.tile = p.tiles[ti];
            if (r.tile.row_base >= 0) {
                r.tok0 = r.tile.q_start;
                r.q_rows = r.tile.q_rows;
                r.first_pos = r.tile.key_limit - 1;
                r.pos = t < r.q_rows ? r.first_pos : 0;
            } else {
                const int seq = r.tile.seq, q0 = r.tile.q_start;
                const int c0 = p.cu_seqlens_q[seq], c1 = p.cu_seqlens_q[seq + 1];
                const int n = p.seq_lens[seq];
                r.tok0 = c0 + q0;
                r.q_rows = min(128, c1 - c0 - q0);
                r.first_pos = n - (c1 - c0) + q0;
                r.pos = t < r.q_rows ? r.first_pos + t : 0;
            }
            return r;
        };
        Rows cur = rows_of(t_begin < t_end ? t_begin : 0);
        for (int ti = t_begin; ti < t_end; ++ti) {
            const Rows nxt = rows_of(ti + 1 < t_end ? ti + 1 : ti);
            const int head = cur.tile.head + (int)rank;
            pair_softmax_tile(p, cur.tile, trow, half, xch, s_full, p_full0, pv_done, o_done, o_free0, g, sb, sph, k,
                              &maps.out, smem_u32(smem + C::kOutOff), e, t, quarter, cur.q_rows, cur.pos,
                              cur.first_pos, cur.tok0, head, head % p.group, err);
            ++k;
            cur = nxt;
        }
        // the output stores have read their shared memory before the CTA ends
        if ((threadIdx.x & 127) == 0) bulk_wait_all();
    }
    if (err) atomicOr(p.status, kStatusWaitTimeout);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // rank 0 saw its last MMA complete, and each CTA its own copies land,
    // before getting here: neither CTA frees TMEM or ends while the other's
    // MMAs, copies or arrivals may still touch it
    cluster_sync();
    if (warp == 0) tmem_dealloc_pair(tmem, C::kTmemCols);
    // launched programmatically behind the step's scatter: what follows on
    // the stream follows both
    if (p.wait_at_end) grid_dependency_wait();
}

cudaError_t launch_prefill_pair(const PrefillParams &p, cudaStream_t stream) {
    using C = PairCfg;
    constexpr int D = C::D;
    EncodeFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    PrefillMaps maps{};
    const cuuint64_t dims[3] = {D, (cuuint64_t)p.num_q_heads, (cuuint64_t)p.num_tokens};
    const cuuint64_t strides[2] = {D * 2ull, (cuuint64_t)p.num_q_heads * D * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    if (!encode_bf16(enc, &maps.q, p.q, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!encode_bf16(enc, &maps.out, p.out, 3, dims, strides, box)) return cudaErrorInvalidValue;
    const cuuint64_t kv_dims[3] = {D, (cuuint64_t)p.num_kv_heads, (cuuint64_t)p.num_blocks * kBlockSize};
    const cuuint64_t kv_strides[2] = {D * 2ull, (cuuint64_t)p.num_kv_heads * D * 2};
    const cuuint32_t kv_box[3] = {64, 1, kBlockSize};
    if (!encode_bf16(enc, &maps.k, p.k_cache, 3, kv_dims, kv_strides, kv_box) ||
        !encode_bf16(enc, &maps.v, p.v_cache, 3, kv_dims, kv_strides, kv_box))
        return cudaErrorInvalidValue;
    if (p.k_new != nullptr) {
        const cuuint64_t new_dims[3] = {D, (cuuint64_t)p.num_kv_heads, (cuuint64_t)p.num_tokens};
        const cuuint32_t new_box[3] = {64, 1, 64};
        if (!encode_bf16(enc, &maps.kn, p.k_new, 3, new_dims, kv_strides, new_box) ||
            !encode_bf16(enc, &maps.vn, p.v_new, 3, new_dims, kv_strides, new_box))
            return cudaErrorInvalidValue;
    }
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_relaxed) & bit)) {
        cudaError_t e =
            cudaFuncSetAttribute(prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_relaxed);
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * p.num_ctas);  // num_ctas counts clusters here
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.wait_at_end ? 2 : 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_pair_kernel, p, maps);
    return e != cudaSuccess ? e : cudaGetLastError();
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

cudaError_t launch_scatter_stage(const ScatterArgs &a, const PrefillParams &p, int head_dim,
                                 cudaStream_t stream) {
    if (p.num_stages == 0)
        return launch_reshape_and_cache(a.k, a.v, a.slots, a.k_cache, a.v_cache, a.num_tokens, a.token_elems,
                                        a.num_slots, a.num_sms, false, stream);
    const int64_t chunks = a.num_tokens * (a.token_elems / 8);
    // the scatter's share: as many blocks as the plain scatter kernel takes
    const int scatter_blocks = (int)std::min<int64_t>((chunks + 255) / 256, (int64_t)a.num_sms * 8);
    const dim3 grid(scatter_blocks + 2 * p.num_stages);
    if (head_dim == 64)
        scatter_stage_kernel<64><<<grid, 256, 0, stream>>>(a, p, scatter_blocks);
    else
        scatter_stage_kernel<128><<<grid, 256, 0, stream>>>(a, p, scatter_blocks);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillParams &p, int head_dim, cudaStream_t stream) {
    if (p.num_tiles == 0) return cudaSuccess;
    if (p.pair) return head_dim == 128 ? launch_prefill_pair(p, stream) : cudaErrorInvalidValue;
    return head_dim == 64 ? launch_prefill_t<64>(p, stream) : launch_prefill_t<128>(p, stream);
}

}  // namespace pa
