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
// One CTA computes one tile: 128 consecutive queries of one segment for one
// query head (kv head g = h / G), looping over 128-key tiles of its causal
// range.  Warp roles (256 threads):
//   warp 0     allocates 512 TMEM columns and issues the MMAs (one thread):
//                S_j = Q K_j^T   (M 128 x N 128 x K D), into S buffer j % 2,
//                O  += P_j V_j   (M 128 x N D x K 128), into O,
//              S_{j+1} is issued before O += P_j V_j, so the tensor cores
//              work on the next scores while the softmax warps work on S_j.
//   warps 1-3  load Q once and K/V tiles (two stages) with 16-byte cp.async,
//              each 16-token block through the block table, into 128-byte-
//              swizzled tiles: rows of 64 dims x 2 bytes, chunk index XORed
//              by the row (the canonical SWIZZLE_128B layout the MMA
//              descriptors name).  Q and K are read K-major, V MN-major.  Rows
//              past the segment's length are written as zeros, so no NaN
//              ever meets the tensor cores.
//   warps 4-7  one query row per thread: tcgen05.ld the row of S_j, apply
//              the causal and length mask by selection, scale by
//              scale*log2(e), online softmax with exp2; the running max is
//              only moved (and O in TMEM rescaled) when it grows by more than
//              kRescaleThreshold.  P_j (bf16) goes to shared memory in the
//              same swizzled K-major layout as the A operand of O += P_j V_j.
//              At the end each thread reads its O row, divides by its sum and
//              writes bf16.
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
    static constexpr int kThreads = 256;
    static constexpr int kLoaders = 96;                  // warps 1-3
    static constexpr int kSoftWarp0 = 4;                 // warps 4-7
    static constexpr int kTileBytes = 128 * D * 2;       // a Q, K or V tile
    static constexpr int kPBytes = 128 * 128 * 2;        // P: 128 queries x 128 keys
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = kTileBytes;  // stage s: K at kKVOff + 2 s T, V at + T
    static constexpr int kPOff = kKVOff + 4 * kTileBytes;
    static constexpr int kBarOff = kPOff + kPBytes;
    static constexpr int kNumBars = 10;  // q_full, kv_full[2], kv_empty[2], s_full[2], s_free[2], p_full
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
    static constexpr int kUsed = kTmemSlotOff + 16;
    // At least 120 KiB, so that one CTA (holding 512 TMEM columns) fits per SM.
    static constexpr int kSmemBytes = kUsed + 1024 > 120 * 1024 ? kUsed + 1024 : 120 * 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kOCol = 256;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// Byte address of 16-byte chunk `chunk` (0 .. D/8-1) of row `row` in a
// 128-row tile stored as D/64 slabs of 128 rows x 128 bytes, 128-byte swizzle.
__device__ __forceinline__ uint32_t tile_addr(uint32_t tile, int row, int chunk) {
    return tile + (chunk >> 3) * 16384 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}

__device__ __forceinline__ void st_shared_zero16(uint32_t addr) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
}

__device__ __forceinline__ void st_shared16(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
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

template <int D>
__global__ void __launch_bounds__(256, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
    using C = PrefillCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(smem + C::kQOff);
    const uint32_t sKV = smem_u32(smem + C::kKVOff);
    const uint32_t sP = smem_u32(smem + C::kPOff);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *q_full = bars + 0;
    uint64_t *kv_full = bars + 1;   // [2]
    uint64_t *kv_empty = bars + 3;  // [2]: O += P V of the stage's tile is complete
    uint64_t *s_full = bars + 5;    // [2]
    uint64_t *s_free = bars + 7;    // [2]
    uint64_t *p_full = bars + 9;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kTmemSlotOff);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (blockIdx.x >= p.num_tiles) return;
    const PrefillTile tile = p.tiles[blockIdx.x];
    const int seq = tile.seq, q0 = tile.q_start, h = tile.head;
    const int tok0 = p.cu_seqlens_q[seq] + q0;
    const int L = p.cu_seqlens_q[seq + 1] - p.cu_seqlens_q[seq];
    const int n = p.seq_lens[seq];
    const int q_rows = min(128, L - q0);
    const int nkv = tile.n_kv_tiles;  // 128-key tiles covering keys 0 .. n - L + q0 + q_rows - 1
    const int g = h / p.group;

    if (tid == 0) {
        mbar_init(q_full, C::kLoaders);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&kv_full[s], C::kLoaders);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], 128);
        }
        mbar_init(p_full, 128);
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
            auto issue_pv = [&](int jj) {
                if (!err && !mbar_wait(p_full, jj & 1)) err = true;
                tc_fence_after();
                const uint32_t sV = sKV + (jj & 1) * 2 * C::kTileBytes + C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // 16 keys per MMA
                    const uint64_t a = umma_desc_sw128(sP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = umma_desc_sw128(sV + kk * 2048, 16384, 1024);
                    umma_bf16_ss(tmem + C::kOCol, a, b, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&kv_empty[jj & 1]);
            };
            if (!err && !mbar_wait(q_full, 0)) err = true;
            for (int j = 0; j < nkv; ++j) {
                const int s = j & 1;
                if (!err && !mbar_wait(&kv_full[s], (j >> 1) & 1)) err = true;
                if (j >= 2 && !err && !mbar_wait(&s_free[s], ((j - 2) >> 1) & 1)) err = true;
                tc_fence_after();
                const uint32_t sK = sKV + s * 2 * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {  // 16 dims per MMA
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint64_t a = umma_desc_sw128(sQ + off, 16, 1024);
                    const uint64_t b = umma_desc_sw128(sK + off, 16, 1024);
                    umma_bf16_ss(tmem + s * 128, a, b, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[s]);
                if (j >= 1) issue_pv(j - 1);
            }
            issue_pv(nkv - 1);
            // nothing of ours may be in flight when TMEM is released
            if (!err && !mbar_wait(&kv_empty[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1)) err = true;
        }
    } else if (warp < C::kSoftWarp0) {
        // ------------------------------------------------ loaders
        const int lt = tid - 32;
        const int32_t *bt_row = p.block_tables + (size_t)seq * p.max_blocks_per_seq;
        const size_t tok_stride = (size_t)p.num_kv_heads * D;  // elements between tokens of a block
        constexpr int kChunks = 128 * D / 8;
        // Q tile
        for (int c = lt; c < kChunks; c += C::kLoaders) {
            const int row = c / (D / 8), ch = c % (D / 8);
            const uint32_t dst = tile_addr(sQ, row, ch);
            if (row < q_rows)
                cp_async16(dst, p.q + ((size_t)(tok0 + row) * p.num_q_heads + h) * D + 8 * ch);
            else
                st_shared_zero16(dst);
        }
        cp_async_commit();
        // Tiles 0 and 1 go out at once; tile j >= 2 reuses the stage of tile
        // j - 2 once O += P V of that tile is complete.  A tile's arrival is
        // signalled before any wait on a stage, since the MMAs that free the
        // stage depend on it.
        auto issue_tile = [&](int j) {
            const uint32_t sK = sKV + (j & 1) * 2 * C::kTileBytes, sV = sK + C::kTileBytes;
            for (int c = lt; c < kChunks; c += C::kLoaders) {
                const int row = c / (D / 8), ch = c % (D / 8);
                const int key = 128 * j + row;
                const uint32_t dk = tile_addr(sK, row, ch), dv = tile_addr(sV, row, ch);
                if (key < n) {
                    const int blk = __ldg(bt_row + (key >> 4));
                    const size_t off = ((size_t)blk * 16 + (key & 15)) * tok_stride + (size_t)g * D + 8 * ch;
                    cp_async16(dk, p.k_cache + off);
                    cp_async16(dv, p.v_cache + off);
                } else {
                    st_shared_zero16(dk);
                    st_shared_zero16(dv);
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
        // ------------------------------------------------ softmax, one query row per thread
        const int sw = warp - C::kSoftWarp0;
        const int t = sw * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(sw * 32) << 16);
        // padding rows (past the segment's queries) see key 0 only
        const int pos = t < q_rows ? n - L + q0 + t : 0;
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < nkv; ++j) {
            const int s = j & 1;
            if (!err && !mbar_wait(&s_full[s], (j >> 1) & 1)) err = true;
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tmem_ld32(trow + s * 128 + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * i]));
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&s_free[s]);
            const int kbase = 128 * j;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                float x = __uint_as_float(sr[c]) * p.scale_log2;
                if (kbase + c > pos) x = -INFINITY;  // causal edge; pos < n covers the length
                sr[c] = __float_as_uint(x);
                mx = fmaxf(mx, x);
            }
            float alpha = 1.f;
            const bool rescale = mx > m + kPrefillRescaleThreshold;
            if (rescale) {
                alpha = fast_exp2(m - mx);
                m = mx;
            }
            uint32_t pk[64];
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float p0 = fast_exp2(__uint_as_float(sr[2 * c]) - m);
                const float p1 = fast_exp2(__uint_as_float(sr[2 * c + 1]) - m);
                pk[c] = pack_bf16x2(p0, p1);
                lsum += bf16x2_sum(pk[c]);
            }
            l = l * alpha + lsum;
            if (j >= 1) {
                // O += P_{j-1} V_{j-1} must be complete: it read the P buffer
                // and it wrote O, which may need rescaling now
                if (!err && !mbar_wait(&kv_empty[(j - 1) & 1], ((j - 1) >> 1) & 1)) err = true;
                tc_fence_after();
                // tcgen05.ld/st are warp-collective: rescale if any lane needs
                // it (alpha = 1 for the others)
                if (__any_sync(kFullMask, rescale)) {
#pragma unroll
                    for (int i = 0; i < D / 32; ++i) {
                        uint32_t o[32];
                        tmem_ld32(trow + C::kOCol + 32 * i, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        tmem_st32(trow + C::kOCol + 32 * i, o);
                    }
                    tmem_st_wait();
                }
            }
#pragma unroll
            for (int c = 0; c < 16; ++c)  // 8 keys per chunk
                st_shared16(tile_addr(sP, t, c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (!err && !mbar_wait(&kv_empty[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1)) err = true;
        tc_fence_after();
        const float inv = 1.f / l;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
            uint32_t o[32];
            tmem_ld32(trow + C::kOCol + 32 * i, o);
            tmem_ld_wait();
            if (t < q_rows) {
                __nv_bfloat16 *orow = p.out + ((size_t)(tok0 + t) * p.num_q_heads + h) * D + 32 * i;
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
