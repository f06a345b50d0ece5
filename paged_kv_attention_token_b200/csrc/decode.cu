// Split-KV paged attention for short query segments (decodes), and the
// combine step that merges split rows.
//
// What is computed ("vLLM 学习笔记 01" §1.5-§1.6): for one query token at
// position p of its segment and one kv head g, the G = Hq / Hkv query heads
// of g attend to keys 0..p of the segment, read through its block table
// (logical block b -> physical block block_tables[seq][b], 16 tokens each).
//
// Design (HBM-bound: every KV byte is read once, ~G flops per byte):
//  * Work: the planner lays every row's 16-token blocks end to end and gives
//    each warp an equal run (see plan.cpp).  A warp walks its run block by
//    block; a row it covers entirely is normalised and written as bf16, a
//    row it covers in part leaves (unnormalised O, max, sum) for the combine.
//  * Arithmetic on the tensor cores with warp-level MMA (m16n8k16, bf16 in,
//    fp32 accumulate), with the keys as the M dimension and the G query heads
//    as N (8 columns; G <= 8 uses one n-tile, G <= 16 two):
//        S^T[16 keys x 8 heads]  = K_blk[16 x D] * Q^T[D x 8]
//        O^T[D x 8 heads]       += V_blk^T[D x 16 keys] * P^T[16 keys x 8]
//    A block of 16 tokens is exactly one M tile, so no padding is wasted for
//    G = 8.  The S^T accumulator becomes the B operand of the second MMA
//    through one movmatrix.trans per 8x8 half.
//  * Loads go straight from HBM into MMA fragments with 16-byte loads, no
//    shared memory: the contraction order over head_dim is free, so each
//    thread's 16-byte chunk of a K row supplies its fragment elements for
//    two k-steps (Q is loaded with the same permutation); V rows are paired
//    across keys with byte permutes, and the output dims come out in 16-byte
//    runs per head.  Each warp keeps the next block's K/V loads in flight
//    while it computes the current one (register double buffering).
//  * Online softmax in fp32, base 2: scores are scaled by scale*log2(e); the
//    running max is shared by the 8 lanes that hold a head (3 xor-shuffles
//    per block); the running sum stays per lane until the end.
//  * Keys past the row's length in its last block are masked by selection
//    (score -inf, V zeroed), so whatever the cache holds there (NaN
//    included) never reaches the output.
#include "common.cuh"
#include "kernels.h"

namespace pa {


template <int D>
struct KVFrag {
    uint4 k[2][D / 32];  // K rows g8 and g8+8, chunks 32i + 8*q4
    uint4 v[4][D / 64];  // V rows 2q4, 2q4+1, 2q4+8, 2q4+9, chunks 8*(g8 + 8j)
};

template <int D>
__device__ __forceinline__ void load_kv(KVFrag<D> &f, const __nv_bfloat16 *kb,
                                        const __nv_bfloat16 *vb, size_t row_stride, int g8,
                                        int q4) {
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
        f.k[0][i] = ld_stream16(kb + (size_t)g8 * row_stride + 32 * i + 8 * q4);
        f.k[1][i] = ld_stream16(kb + (size_t)(g8 + 8) * row_stride + 32 * i + 8 * q4);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int key = 2 * q4 + (e & 1) + 8 * (e >> 1);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
            f.v[e][j] = ld_stream16(vb + (size_t)key * row_stride + 8 * (g8 + 8 * j));
    }
}

__device__ __forceinline__ uint32_t word(const uint4 &x, int i) {
    return i == 0 ? x.x : i == 1 ? x.y : i == 2 ? x.z : x.w;
}

template <int D, int NT>
struct DecodeState {
    uint32_t qf[NT][D / 16][2];
    float o[D / 16][NT][4];
    float m[NT][2];
    float l[NT][2];
};

// One 16-key block: scores, online-softmax update, PV accumulation.
template <int D, int NT>
__device__ __forceinline__ void attend_block(DecodeState<D, NT> &st, KVFrag<D> &f, int valid,
                                             float scale_log2, int g8, int q4) {
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
            mma_16816(s[nt], f.k[0][i].x, f.k[1][i].x, f.k[0][i].y, f.k[1][i].y,
                      st.qf[nt][2 * i][0], st.qf[nt][2 * i][1]);
            mma_16816(s2, f.k[0][i].z, f.k[1][i].z, f.k[0][i].w, f.k[1][i].w,
                      st.qf[nt][2 * i + 1][0], st.qf[nt][2 * i + 1][1]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] += s2[e];
    }
    const bool partial = valid < 16;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = g8 + ((e & 2) ? 8 : 0);
            float x = s[nt][e] * scale_log2;
            if (partial && key >= valid) x = -INFINITY;
            s[nt][e] = x;
        }
    if (partial) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = 2 * q4 + (e & 1) + 8 * (e >> 1);
            if (key >= valid)
#pragma unroll
                for (int j = 0; j < D / 64; ++j) f.v[e][j] = make_uint4(0, 0, 0, 0);
        }
    }
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float mx = fmaxf(s[nt][e], s[nt][e + 2]);
            mx = warp_max_xor(mx, 4);
            mx = warp_max_xor(mx, 8);
            mx = warp_max_xor(mx, 16);
            const float mnew = fmaxf(st.m[nt][e], mx);
            const float alpha = exp2f(st.m[nt][e] - mnew);
            st.m[nt][e] = mnew;
            const float p0 = exp2f(s[nt][e] - mnew);
            const float p1 = exp2f(s[nt][e + 2] - mnew);
            st.l[nt][e] = st.l[nt][e] * alpha + p0 + p1;
            s[nt][e] = p0;
            s[nt][e + 2] = p1;
#pragma unroll
            for (int t = 0; t < D / 16; ++t) {
                st.o[t][nt][e] *= alpha;
                st.o[t][nt][e + 2] *= alpha;
            }
        }
        pb[nt][0] = movmatrix_trans(pack_bf16x2(s[nt][0], s[nt][1]));
        pb[nt][1] = movmatrix_trans(pack_bf16x2(s[nt][2], s[nt][3]));
    }
#pragma unroll
    for (int j = 0; j < D / 64; ++j)
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
            const uint32_t v0 = word(f.v[0][j], uu), v1 = word(f.v[1][j], uu);
            const uint32_t v2 = word(f.v[2][j], uu), v3 = word(f.v[3][j], uu);
            const uint32_t a0 = __byte_perm(v0, v1, 0x5410);
            const uint32_t a1 = __byte_perm(v0, v1, 0x7632);
            const uint32_t a2 = __byte_perm(v2, v3, 0x5410);
            const uint32_t a3 = __byte_perm(v2, v3, 0x7632);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mma_16816(st.o[4 * j + uu][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
        }
}

// Blocks [b, bend) of one row, by one warp.
template <int D, int NT, bool PIPE>
__device__ __forceinline__ void decode_piece(const DecodeParams &p, const DecodeRow row, int gkv,
                                             int b, int bend, int unit, int lane) {
    const int g8 = lane >> 2, q4 = lane & 3;
    const int G = p.group;
    const int h0 = gkv * G;
    DecodeState<D, NT> st;
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

    const int32_t *bt_row = p.block_tables + (size_t)row.seq * p.max_blocks_per_seq;
    const int nblk = (row.n_keys + 15) >> 4;
    const size_t row_stride = (size_t)p.num_kv_heads * D;  // elements between tokens of a block
    const __nv_bfloat16 *kbase = p.k_cache + (size_t)gkv * D;
    const __nv_bfloat16 *vbase = p.v_cache + (size_t)gkv * D;
    // Block ids are fetched 32 at a time, one per lane, and broadcast.
    int bt_base = -1, bt_val = 0;
    auto block_ptr_off = [&](int blk) -> size_t {
        if ((blk & ~31) != bt_base) {
            bt_base = blk & ~31;
            const int idx = bt_base + lane;
            bt_val = idx < nblk ? __ldg(bt_row + idx) : 0;
        }
        const int id = __shfl_sync(kFullMask, bt_val, blk & 31);
        return (size_t)id * 16 * row_stride;
    };

    if constexpr (PIPE) {
        KVFrag<D> fa, fb;
        size_t off = block_ptr_off(b);
        load_kv<D>(fa, kbase + off, vbase + off, row_stride, g8, q4);
        for (int blk = b; blk < bend; blk += 2) {
            if (blk + 1 < bend) {
                off = block_ptr_off(blk + 1);
                load_kv<D>(fb, kbase + off, vbase + off, row_stride, g8, q4);
            }
            attend_block<D, NT>(st, fa, row.n_keys - blk * 16, p.scale_log2, g8, q4);
            if (blk + 1 >= bend) break;
            if (blk + 2 < bend) {
                off = block_ptr_off(blk + 2);
                load_kv<D>(fa, kbase + off, vbase + off, row_stride, g8, q4);
            }
            attend_block<D, NT>(st, fb, row.n_keys - (blk + 1) * 16, p.scale_log2, g8, q4);
        }
    } else {
        for (int blk = b; blk < bend; ++blk) {
            KVFrag<D> fa;
            const size_t off = block_ptr_off(blk);
            load_kv<D>(fa, kbase + off, vbase + off, row_stride, g8, q4);
            attend_block<D, NT>(st, fa, row.n_keys - blk * 16, p.scale_log2, g8, q4);
        }
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
                for (int j = 0; j < D / 64; ++j) {
                    uint4 w;
                    w.x = pack_bf16x2(st.o[4 * j + 0][nt][e] * inv, st.o[4 * j + 0][nt][e + 2] * inv);
                    w.y = pack_bf16x2(st.o[4 * j + 1][nt][e] * inv, st.o[4 * j + 1][nt][e + 2] * inv);
                    w.z = pack_bf16x2(st.o[4 * j + 2][nt][e] * inv, st.o[4 * j + 2][nt][e + 2] * inv);
                    w.w = pack_bf16x2(st.o[4 * j + 3][nt][e] * inv, st.o[4 * j + 3][nt][e + 2] * inv);
                    st16(orow + 8 * (g8 + 8 * j), w);
                }
            }
    } else {
        const int slot = row.slot_base + unit;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int head = 8 * nt + 2 * q4 + e;
                if (head >= G) continue;
                float *po = p.partial_o + ((size_t)slot * G + head) * D;
#pragma unroll
                for (int j = 0; j < D / 64; ++j) {
                    float4 lo = make_float4(st.o[4 * j + 0][nt][e], st.o[4 * j + 0][nt][e + 2],
                                            st.o[4 * j + 1][nt][e], st.o[4 * j + 1][nt][e + 2]);
                    float4 hi = make_float4(st.o[4 * j + 2][nt][e], st.o[4 * j + 2][nt][e + 2],
                                            st.o[4 * j + 3][nt][e], st.o[4 * j + 3][nt][e + 2]);
                    float4 *dst = reinterpret_cast<float4 *>(po + 8 * (g8 + 8 * j));
                    dst[0] = lo;
                    dst[1] = hi;
                }
                if (g8 == 0) p.partial_ml[(size_t)slot * G + head] = make_float2(st.m[nt][e], st.l[nt][e]);
            }
    }
}

template <int D, int NT, int WARPS, int MIN_BLOCKS, bool PIPE>
__global__ void __launch_bounds__(WARPS * 32, MIN_BLOCKS) decode_kernel(const DecodeParams p) {
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x * WARPS + (threadIdx.x >> 5);
    if (unit >= p.num_units) return;
    const DecodeUnit start = p.units[unit];
    const DecodeUnit end = p.units[unit + 1];
    int r = start.row, b = start.block;
    while (r < end.row || (r == end.row && b < end.block)) {
        const DecodeRow row = p.rows[r];
        const int nblk = (row.n_keys + 15) >> 4;
        const int bend = (r == end.row) ? end.block : nblk;
        decode_piece<D, NT, PIPE>(p, row, r % p.num_kv_heads, b, bend, unit, lane);
        ++r;
        b = 0;
    }
}

// Merge the partials of rows cut across warps: O = sum_j 2^(m_j - M) O_j /
// sum_j 2^(m_j - M) l_j with M = max_j m_j.  One thread per (head, 8 dims).
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const CombineRow *__restrict__ combine,
                                                      const DecodeRow *__restrict__ rows,
                                                      const float *__restrict__ partial_o,
                                                      const float2 *__restrict__ partial_ml,
                                                      __nv_bfloat16 *__restrict__ out, int group,
                                                      int num_q_heads, int num_kv_heads) {
    const CombineRow c = combine[blockIdx.x];
    const int head = threadIdx.x / (D / 8);
    const int chunk = threadIdx.x % (D / 8);
    if (head >= group) return;
    const DecodeRow row = rows[c.row];
    const int gkv = c.row % num_kv_heads;
    float M = -INFINITY;
    for (int j = 0; j < c.piece_count; ++j)
        M = fmaxf(M, partial_ml[(size_t)(c.piece_base + j) * group + head].x);
    float den = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < c.piece_count; ++j) {
        const size_t slot = (size_t)(c.piece_base + j);
        const float2 ml = partial_ml[slot * group + head];
        const float w = exp2f(ml.x - M);
        den += w * ml.y;
        const float4 *po = reinterpret_cast<const float4 *>(partial_o + (slot * group + head) * D + 8 * chunk);
        const float4 lo = po[0], hi = po[1];
        acc[0] += w * lo.x; acc[1] += w * lo.y; acc[2] += w * lo.z; acc[3] += w * lo.w;
        acc[4] += w * hi.x; acc[5] += w * hi.y; acc[6] += w * hi.z; acc[7] += w * hi.w;
    }
    const float inv = 1.f / den;
    uint4 o;
    o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    st16(out + ((size_t)row.token * num_q_heads + gkv * group + head) * D + 8 * chunk, o);
}

constexpr int kDecodeWarps = 4;

template <int D, int NT>
static cudaError_t launch_decode_t(const DecodeParams &p, cudaStream_t stream) {
    const int grid = (p.num_units + kDecodeWarps - 1) / kDecodeWarps;
    if constexpr (D == 64 && NT == 1) {
        // 164 live registers; 4 CTAs of 4 warps per SM keep ~64 KB of KV in flight
        decode_kernel<D, NT, kDecodeWarps, 4, true><<<grid, kDecodeWarps * 32, 0, stream>>>(p);
    } else if constexpr (D == 64 || NT == 1) {
        decode_kernel<D, NT, kDecodeWarps, 2, true><<<grid, kDecodeWarps * 32, 0, stream>>>(p);
    } else {
        // two n-tiles at D = 128 leave no registers for a second block in flight
        decode_kernel<D, NT, kDecodeWarps, 2, false><<<grid, kDecodeWarps * 32, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams &p, int head_dim, cudaStream_t stream) {
    if (p.num_units == 0) return cudaSuccess;
    const int nt = p.group > 8 ? 2 : 1;
    if (head_dim == 64) return nt == 1 ? launch_decode_t<64, 1>(p, stream) : launch_decode_t<64, 2>(p, stream);
    return nt == 1 ? launch_decode_t<128, 1>(p, stream) : launch_decode_t<128, 2>(p, stream);
}

cudaError_t launch_combine(const CombineRow *combine, const DecodeRow *rows, const float *partial_o,
                           const float2 *partial_ml, __nv_bfloat16 *out, int num_combine,
                           int group, int num_q_heads, int num_kv_heads, int head_dim,
                           cudaStream_t stream) {
    if (num_combine == 0) return cudaSuccess;
    const int threads = ((group * (head_dim / 8) + 31) / 32) * 32;
    if (head_dim == 64)
        combine_kernel<64><<<num_combine, threads, 0, stream>>>(combine, rows, partial_o, partial_ml,
                                                                out, group, num_q_heads, num_kv_heads);
    else
        combine_kernel<128><<<num_combine, threads, 0, stream>>>(combine, rows, partial_o, partial_ml,
                                                                 out, group, num_q_heads, num_kv_heads);
    return cudaGetLastError();
}

}  // namespace pa
