// Forward kernel: O = softmax(scale * Q K^T) V with causal / sliding-window
// masking, plus the natural-log row log-sum-exp.
//
// The tiling follows the FlashAttention idea the GPT-2 lecture describes in
// "Раздел 2" (never materialise the T x T matrix; softmax in pieces with a
// running max m and running sum l, rescaling the old sum by e^(m_old - m_new)
// when the max grows).  The mapping onto sm_100a is this file's own:
//
//   one CTA = one (batch*head, 128-query tile), 6 warps:
//     warp 0      TMA producer: Q once, then K_j / V_j through a 2-stage ring
//     warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//     warps 2..5  softmax warpgroup: thread r owns query row r of the tile
//   TMEM (256 columns): S = Q K_j^T fp32 in columns [0,128); P (bf16 pairs)
//   is written back over the first 64 of them and fed to the PV MMA straight
//   from TMEM; the O accumulator lives in columns [128, 128 + D).
//
// Tiles of keys entirely after the tile's last query, or entirely before the
// window of its first query, are never loaded; only the diagonal tile and the
// window-edge tiles evaluate the visibility predicate.
#pragma once

#include "sm100.cuh"

namespace gpt_attn {

constexpr int kTile = 128;           // rows per Q tile and per K/V tile
constexpr int kFwdStages = 2;        // K/V ring depth
constexpr int kFwdThreads = 192;

struct FwdParams {
    __nv_bfloat16* o;
    float* lse;
    int T;
    int BH;
    int n_tiles;          // ceil(T / 128)
    int window;           // <= 0: causal only
    float scale_log2;     // scale * log2(e)
    uint64_t timeout_ns;
};

template <int D>
struct FwdSmem {
    static constexpr int kTileBytes = kTile * D * 2;   // one bf16 [128, D] tile
    alignas(1024) uint8_t q[kTileBytes];
    alignas(1024) uint8_t k[kFwdStages][kTileBytes];
    alignas(1024) uint8_t v[kFwdStages][kTileBytes];
    uint64_t bar_q;
    uint64_t bar_k[kFwdStages];
    uint64_t bar_v[kFwdStages];
    uint64_t bar_kv_empty[kFwdStages];
    uint64_t bar_s_full;
    uint64_t bar_p_full;
    uint64_t bar_pv_done;
    uint64_t bar_drain;
    uint32_t tmem_base;
    int abort_flag;
};

// Key range of a query tile: tiles [j_lo, j_hi] hold every visible key.
__device__ __forceinline__ void fwd_key_range(int q_tile, int window, int& j_lo, int& j_hi) {
    const int q0 = q_tile * kTile;
    j_hi = q_tile;
    j_lo = 0;
    if (window > 0) {
        const int first = q0 - window + 1;
        j_lo = first > 0 ? first / kTile : 0;
    }
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    FwdSmem<D>& sm = *reinterpret_cast<FwdSmem<D>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    constexpr int kTileBytes = FwdSmem<D>::kTileBytes;
    constexpr int kBoxes = D / 64;                 // 64-column TMA boxes per tile
    constexpr uint32_t kColS = 0;                  // S / P columns
    constexpr uint32_t kColO = 128;                // O accumulator columns
    constexpr uint32_t kTmemCols = 256;
    constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bh = blockIdx.x % p.BH;
    const int q_tile = p.n_tiles - 1 - blockIdx.x / p.BH;   // longest tiles launch first
    const int q0 = q_tile * kTile;
    int j_lo, j_hi;
    fwd_key_range(q_tile, p.window, j_lo, j_hi);
    const int n_kv = j_hi - j_lo + 1;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < kFwdStages; ++s) {
            mbar_init(&sm.bar_k[s], 1);
            mbar_init(&sm.bar_v[s], 1);
            mbar_init(&sm.bar_kv_empty[s], 1);
        }
        mbar_init(&sm.bar_s_full, 1);
        mbar_init(&sm.bar_p_full, 128);
        mbar_init(&sm.bar_pv_done, 1);
        mbar_init(&sm.bar_drain, 1);
        sm.abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const AbortCtl ac{&sm.abort_flag, p.timeout_ns};

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(&sm.bar_q, kTileBytes);
            for (int b = 0; b < kBoxes; ++b) tma_load_3d(sm.q + b * 16384, &tm_q, &sm.bar_q, b * 64, q0, bh);
            int it = 0;
            for (; it < n_kv; ++it) {
                const int s = it % kFwdStages;
                const int n = it / kFwdStages;
                if (n > 0 && !mbar_wait(&sm.bar_kv_empty[s], (n - 1) & 1, ac)) break;
                const int k0 = (j_lo + it) * kTile;
                mbar_arrive_expect_tx(&sm.bar_k[s], kTileBytes);
                for (int b = 0; b < kBoxes; ++b)
                    tma_load_3d(sm.k[s] + b * 16384, &tm_k, &sm.bar_k[s], b * 64, k0, bh);
                mbar_arrive_expect_tx(&sm.bar_v[s], kTileBytes);
                for (int b = 0; b < kBoxes; ++b)
                    tma_load_3d(sm.v[s] + b * 16384, &tm_v, &sm.bar_v[s], b * 64, k0, bh);
            }
            if (sm.abort_flag) {
                // Let every load already issued land before the CTA exits.
                mbar_wait_drain(&sm.bar_q, 0, p.timeout_ns);
                for (int r = (it > kFwdStages ? it - kFwdStages : 0); r < it; ++r) {
                    const int s = r % kFwdStages, n = r / kFwdStages;
                    mbar_wait_drain(&sm.bar_k[s], n & 1, p.timeout_ns);
                    mbar_wait_drain(&sm.bar_v[s], n & 1, p.timeout_ns);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait(&sm.bar_q, 0, ac);
            const uint32_t q_addr = smem_u32(sm.q);
            for (int it = 0; ok && it < n_kv; ++it) {
                const int s = it % kFwdStages;
                const uint32_t ph = (it / kFwdStages) & 1;
                if (!mbar_wait(&sm.bar_k[s], ph, ac)) break;
                // S shares columns with the P the previous PV MMA reads: wait for it.
                if (it > 0 && !mbar_wait(&sm.bar_pv_done, (it - 1) & 1, ac)) break;
                tc_fence_after();
                const uint32_t k_addr = smem_u32(sm.k[s]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(tmem + kColS, sw128_desc(q_addr + off, 16, 1024), sw128_desc(k_addr + off, 16, 1024),
                           kIdescQK, kk > 0);
                }
                mma_commit(&sm.bar_s_full);
                if (!mbar_wait(&sm.bar_p_full, it & 1, ac)) break;
                if (!mbar_wait(&sm.bar_v[s], ph, ac)) break;
                tc_fence_after();
                const uint32_t v_addr = smem_u32(sm.v[s]);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    mma_ts(tmem + kColO, tmem + kColS + kk * 8, sw128_desc(v_addr + kk * 2048, 16384, 1024),
                           kIdescPV, (it > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&sm.bar_kv_empty[s]);
                mma_commit(&sm.bar_pv_done);
            }
            // Make sure no MMA is still running when TMEM is released.
            mma_commit(&sm.bar_drain);
            mbar_wait_drain(&sm.bar_drain, 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroup
        const int wq = warp & 3;                      // TMEM lane quarter this warp may access
        const int row = wq * 32 + lane;
        const int i_abs = q0 + row;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        const float sl2 = p.scale_log2;
        const int W = p.window;
        float m = -INFINITY;     // running max, log2 domain
        float l = 0.f;           // running sum of 2^(x - m)
        bool ok = true;
        for (int it = 0; it < n_kv; ++it) {
            const int k0 = (j_lo + it) * kTile;
            if (!warp_wait(&sm.bar_s_full, it & 1, ac)) { ok = false; break; }
            tc_fence_after();
            const bool need_mask = (j_lo + it == q_tile) || (W > 0 && k0 <= q0 + kTile - 1 - W);
            // pass 1: row max of the visible scores in this tile
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(t_lane + kColS + c * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float x = __uint_as_float(r[e]) * sl2;
                    if (need_mask) {
                        const int j = k0 + c * 32 + e;
                        if (j > i_abs || (W > 0 && j <= i_abs - W)) x = -INFINITY;
                    }
                    mx = fmaxf(mx, x);
                }
            }
            const float m_new = fmaxf(m, mx);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            // tcgen05.ld/st are warp-collective: rescale when any row of the warp needs it
            // (alpha = 1 for the others).
            if (it > 0 && __any_sync(0xffffffffu, m_new > m)) {
                // The previous PV MMA has completed (its commit preceded S's), so O may be rescaled in place.
                const float alpha = (m_new > m) ? ex2_approx(m - m_use) : 1.f;
                l *= alpha;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(t_lane + kColO + c * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                    tmem_st32(t_lane + kColO + c * 32, r);
                }
            }
            m = m_new;
            // pass 2: probabilities, row sum, bf16 P written over the consumed S columns
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(t_lane + kColS + c * 32, r);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float x0 = __uint_as_float(r[e]) * sl2;
                    float x1 = __uint_as_float(r[e + 1]) * sl2;
                    if (need_mask) {
                        const int j = k0 + c * 32 + e;
                        if (j > i_abs || (W > 0 && j <= i_abs - W)) x0 = -INFINITY;
                        if (j + 1 > i_abs || (W > 0 && j + 1 <= i_abs - W)) x1 = -INFINITY;
                    }
                    const float p0 = ex2_approx(x0 - m_use);
                    const float p1 = ex2_approx(x1 - m_use);
                    rs += p0 + p1;
                    pk[e >> 1] = pack_bf16x2(p0, p1);
                }
                tmem_st16(t_lane + kColS + c * 16, pk);
            }
            l += rs;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar_p_full);
        }
        // ---------------------------------------------------------- epilogue
        if (__all_sync(0xffffffffu, ok) && warp_wait(&sm.bar_pv_done, (n_kv - 1) & 1, ac)) {
            tc_fence_after();
            const float inv_l = 1.f / l;
            const bool store = i_abs < p.T;
            __nv_bfloat16* orow = p.o + ((size_t)bh * p.T + (store ? i_abs : 0)) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(t_lane + kColO + c * 32, r);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    pk[e >> 1] = pack_bf16x2(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
                if (store) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
                }
            }
            if (store) p.lse[(size_t)bh * p.T + i_abs] = (m + log2f(l)) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace gpt_attn
