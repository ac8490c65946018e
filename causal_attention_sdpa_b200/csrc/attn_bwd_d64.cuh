// Persistent pipelined backward kernel for head dimension 64 (the GPT-2 shapes).
//
// Same gradient and decomposition as attn_bwd.cuh (P, dV = P^T dO, dP, Delta,
// dS = P (dP - Delta), dK, dQ) and the same work unit: one (batch*head, 128-key
// tile), whose K and V stay in shared memory while the query tiles that see it
// stream past.  One CTA runs per SM and takes work units from a counter in the
// workspace, in the list order of schedule.h (head-major, so the units of a head
// run close together and its Q, dO and dQ rows are served from L2; a tail that
// ends with short units).  K/V are double-buffered across units,
// so the next unit's loads and first scores overlap the end of the current one.
//
//   16 warps:
//     warp 0        TMA producer: takes units, loads K/V and streams Q, dO, lse, Delta
//     warp 1        TMEM allocator; issues S^T = K Q^T and dP^T = V dO^T
//     warp 2        issues dV += P^T dO        warp 3   issues dK += dS^T Q and dQ = dS K
//     warps 4..7    P/dS warpgroup for query columns [0, 64) of each tile
//     warps 8..11   P/dS warpgroup for query columns [64, 128)
//     warps 12..15  dQ warpgroup: copies dQ(g) out of TMEM and adds it into the
//                   fp32 accumulator (staged in the dS buffer dQ(g) has just read,
//                   then TMA bulk reduce-add); writes each unit's dK (x scale) and dV,
//                   staged in the unit's own K and V buffers (no MMA reads them any
//                   more), with two TMA tile stores
//   The MMAs are spread over three issuing warps: one thread cannot issue
//   128-row MMAs of N <= 128 fast enough to keep the tensor pipe busy.
//   TMEM (512 columns): S^T [0,128)  dP^T [128,256)  P^T bf16 [256,320)
//                       dV [320,384)  dK [384,448)  dQ [448,512)
//   Shared memory: K, V x 2; 2 x (Q, dO, lse2, Delta); dS^T bf16 [key][query] x 2
//                  (each doubles as the fp32 staging of dQ for its reduction).
//
// Every per-tile barrier phase counts query tiles over all units the CTA has
// processed (g), so the pipeline runs on from one unit into the next.
// S(i+1) and dP(i+1) go in as soon as both P/dS warpgroups have copied S(i) and
// dP(i) into registers, so the tensor pipe computes the next scores while the
// exponentials of this tile run.
#pragma once

#include <climits>

#include "attn_bwd.cuh"

namespace gpt_attn {

constexpr int kBwd64Threads = 512;

struct Bwd64Cfg {
    static constexpr int D = 64;
    static constexpr int kStages = 2;                        // Q/dO ring depth
    static constexpr int kTileBytes = kTile * D * 2;         // 16 KB
    static constexpr uint32_t kColS = 0, kColDP = 128, kColP = 256, kColDV = 320, kColDK = 384, kColDQ = 448;
    // Threads that read each unit id: warps 1..3 (one lane each) + 256 P/dS + 128 dQ.
    static constexpr uint32_t kUnitReaders = 3 + 256 + 128;
};

struct Bwd64Smem {
    using C = Bwd64Cfg;
    alignas(1024) uint8_t k[2][C::kTileBytes];
    alignas(1024) uint8_t v[2][C::kTileBytes];
    alignas(1024) uint8_t q[C::kStages][C::kTileBytes];
    alignas(1024) uint8_t dout[C::kStages][C::kTileBytes];
    // dS^T bf16 [key][query] as two 64-query halves; once dK(g) and dQ(g) have read it, the same
    // 32 KB stages dQ(g) in fp32 as two [128 rows][32 cols] 128B-swizzled boxes for the reduce.
    alignas(1024) uint8_t ds[2][kTile * kTile * 2];
    alignas(16) float lse2[C::kStages][kTile];
    alignas(16) float delta[C::kStages][kTile];
    alignas(16) int lower[C::kStages][kTile];       // document masks only
    int unit[2];                  // work-unit ring: id, or -1 when there is no more work
    uint64_t bar_unit_full[2];
    uint64_t bar_unit_empty[2];
    uint64_t bar_kv_full[2];
    uint64_t bar_kv_empty[2];     // S/dP warp, dK/dQ warp and the dK/dV stores done with this K/V buffer
    uint64_t bar_qdo_full[C::kStages];
    uint64_t bar_qdo_empty[C::kStages];
    uint64_t bar_s_full;
    uint64_t bar_dp_full;
    uint64_t bar_sdp_free;        // both P/dS warpgroups have S(g), dP(g) in registers
    uint64_t bar_p_full;          // P^T(g) in TMEM
    uint64_t bar_dv_done;         // dV(g) MMA finished: P^T columns free
    uint64_t bar_ds_full[2];      // dS^T(g) in shared buffer g % 2
    uint64_t bar_ds_empty[2];     // buffer g % 2 free again: dK(g), dQ(g) read it, dQ(g) staged and reduced
    uint64_t bar_dq_full;
    uint64_t bar_dq_free;         // dQ(g) copied out of TMEM
    uint64_t bar_dkdv_full;       // last dV and dK of a unit finished
    uint64_t bar_dkdv_free;       // dK, dV of a unit copied out of TMEM
    uint64_t bar_stage_full;      // the dQ warpgroup has staged dQ(g)
    uint64_t bar_dkdv_staged;     // the dQ warpgroup has staged a unit's dK and dV
    uint64_t bar_drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct Bwd64Unit {
    int bh, kt, k0, qt_lo, n_q, W;
};

// Work unit u of the list (schedule.h): head bh, key tile kt, and the n_q query tiles
// [kt, kt + n_q) that see it.
template <typename Mask>
__device__ __forceinline__ Bwd64Unit bwd64_unit(int u, const BwdParams& p, const Mask& mask) {
    Bwd64Unit w;
    list_item(u, p.BH, p.n_tiles, p.tail, w.bh, w.kt);
    w.W = mask.head_window(w.bh);
    w.n_q = bwd_last_tile(p, w.bh, w.kt, w.W) - w.kt + 1;
    w.k0 = w.kt * kTile;
    w.qt_lo = w.kt;
    return w;
}

template <typename Mask>
__global__ void __launch_bounds__(kBwd64Threads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                const __grid_constant__ CUtensorMap tm_dv, const BwdParams p, const __grid_constant__ Mask mask) {
    using C = Bwd64Cfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    Bwd64Smem& sm = *reinterpret_cast<Bwd64Smem*>(smem_align1024(smem_raw));

    constexpr int kStages = C::kStages;
    constexpr int kTileBytes = C::kTileBytes;
    constexpr uint32_t kTmemCols = 512;
    constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);    // S^T = K Q^T, dP^T = V dO^T
    constexpr uint32_t kIdescKxMN = idesc_bf16_f32(128, D, 0, 1);    // dV (A = P^T in TMEM), dK
    constexpr uint32_t kIdescMNxMN = idesc_bf16_f32(128, D, 1, 1);   // dQ

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int total_units = p.BH * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.bar_unit_full[b], 1);
            mbar_init(&sm.bar_unit_empty[b], C::kUnitReaders);
            mbar_init(&sm.bar_kv_full[b], 1);
            mbar_init(&sm.bar_kv_empty[b], 3);
            mbar_init(&sm.bar_ds_full[b], 256);
            mbar_init(&sm.bar_ds_empty[b], 1);      // by the dQ reduce issuer
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.bar_qdo_full[s], 1);
            mbar_init(&sm.bar_qdo_empty[s], 2);     // dV warp + dK warp
        }
        mbar_init(&sm.bar_s_full, 1);
        mbar_init(&sm.bar_dp_full, 1);
        mbar_init(&sm.bar_sdp_free, 256);
        mbar_init(&sm.bar_p_full, 256);
        mbar_init(&sm.bar_dv_done, 1);
        mbar_init(&sm.bar_dq_full, 1);
        mbar_init(&sm.bar_dq_free, 128);
        mbar_init(&sm.bar_dkdv_full, 2);            // last dV + last dK of the unit
        mbar_init(&sm.bar_dkdv_free, 128);
        mbar_init(&sm.bar_stage_full, 128);
        mbar_init(&sm.bar_dkdv_staged, 128);
        mbar_init(&sm.bar_drain, 3);                // the three MMA-issuing threads
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

    // Next work unit for a consumer role: waits for ring slot n % 2, reads it, releases it.
    auto read_unit = [&](int n, int& u) -> bool {
        const int slot = n & 1;
        if (!mbar_wait(&sm.bar_unit_full[slot], (n >> 1) & 1, ac)) return false;
        u = *reinterpret_cast<volatile int*>(&sm.unit[slot]);
        mbar_arrive(&sm.bar_unit_empty[slot]);
        return true;
    };

    // Launched with 128 registers per thread (512 x 128 = 65536).  Warpgroup 0
    // (producer, MMA issuers) 48, the two P/dS warpgroups 184, the dQ
    // warpgroup 96: 128 x (48 + 184 + 184 + 96) = 65536.
    if (warp < 4) {
        regs_dec<48>();
        if (warp == 0 && lane == 0) {
            // -------------------------------------------------------- producer
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
            int g = 0;                         // query tiles loaded so far
            int n_kv = 0;                      // K/V buffers loaded so far
            bool ok = true;
            for (int n = 0; ok; ++n) {
                const int slot = n & 1;
                int u = atomicAdd(p.sched, 1);
                if (u >= total_units) u = -1;
                if (n >= 2 && !(ok = mbar_wait(&sm.bar_unit_empty[slot], ((n >> 1) - 1) & 1, ac))) break;
                *reinterpret_cast<volatile int*>(&sm.unit[slot]) = u;
                mbar_arrive(&sm.bar_unit_full[slot]);
                if (u < 0) break;
                const Bwd64Unit w = bwd64_unit(u, p, mask);
                const int kb = n & 1;
                if (n >= 2 && !(ok = mbar_wait(&sm.bar_kv_empty[kb], ((n >> 1) - 1) & 1, ac))) break;
                const int hh = w.bh % p.H, bb = w.bh / p.H;
                mbar_arrive_expect_tx(&sm.bar_kv_full[kb], 2 * kTileBytes);
                tma_load_4d(sm.k[kb], &tm_k, &sm.bar_kv_full[kb], 0, w.k0, hh, bb);
                tma_load_4d(sm.v[kb], &tm_v, &sm.bar_kv_full[kb], 0, w.k0, hh, bb);
                n_kv = n + 1;
                for (int i = 0; i < w.n_q; ++i, ++g) {
                    const int s = g % kStages;
                    const int m = g / kStages;
                    if (m > 0 && !(ok = mbar_wait(&sm.bar_qdo_empty[s], (m - 1) & 1, ac))) break;
                    if (debug_skip_load(2, g)) continue;           // debug builds: exercise the abort path
                    const int q0 = (w.qt_lo + i) * kTile;
                    mbar_arrive_expect_tx(&sm.bar_qdo_full[s], 2 * kTileBytes + (p.lower2 ? 3 : 2) * kTile * 4);
                    tma_load_4d(sm.q[s], &tm_q, &sm.bar_qdo_full[s], 0, q0, hh, bb);
                    tma_load_4d(sm.dout[s], &tm_do, &sm.bar_qdo_full[s], 0, q0, hh, bb);
                    const size_t roff = (size_t)w.bh * p.T_pad + q0;
                    bulk_load(sm.lse2[s], p.lse2 + roff, kTile * 4, &sm.bar_qdo_full[s]);
                    bulk_load(sm.delta[s], p.delta + roff, kTile * 4, &sm.bar_qdo_full[s]);
                    if (p.lower2) bulk_load(sm.lower[s], p.lower2 + roff, kTile * 4, &sm.bar_qdo_full[s]);
                }
            }
            if (sm.abort_flag) {
                // Let every load already issued land before the CTA exits.
                for (int r = (n_kv > 2 ? n_kv - 2 : 0); r < n_kv; ++r)
                    mbar_wait_drain(&sm.bar_kv_full[r & 1], (r >> 1) & 1, p.timeout_ns);
                for (int r = (g > kStages ? g - kStages : 0); r < g; ++r)
                    mbar_wait_drain(&sm.bar_qdo_full[r % kStages], (r / kStages) & 1, p.timeout_ns);
            }
        } else if (lane == 0 && warp >= 1) {
            // -------------------------------------------------------- MMA issuers
            bool ok = true;
            int g = 0;
            for (int n = 0; ok; ++n) {
                int u;
                if (!(ok = read_unit(n, u)) || u < 0) break;
                const Bwd64Unit w = bwd64_unit(u, p, mask);
                const int kb = n & 1;
                const uint32_t k_addr = smem_u32(sm.k[kb]);
                const uint32_t v_addr = smem_u32(sm.v[kb]);
                if (warp == 1) {
                    if (!(ok = mbar_wait(&sm.bar_kv_full[kb], (n >> 1) & 1, ac))) break;
                    for (int i = 0; i < w.n_q; ++i, ++g) {
                        const int s = g % kStages;
                        if (!(ok = mbar_wait(&sm.bar_qdo_full[s], (g / kStages) & 1, ac))) break;
                        if (g > 0 && !(ok = mbar_wait(&sm.bar_sdp_free, (g - 1) & 1, ac))) break;
                        tc_fence_after();
                        const uint32_t q_addr = smem_u32(sm.q[s]);
                        const uint32_t do_addr = smem_u32(sm.dout[s]);
#pragma unroll 1
                        for (int kk = 0; kk < D / 16; ++kk)
                            mma_ss(tmem + C::kColS, sw128_desc(k_addr + kk * 32, 16, 1024),
                                   sw128_desc(q_addr + kk * 32, 16, 1024), kIdescSS, kk > 0);
                        mma_commit(&sm.bar_s_full);
#pragma unroll 1
                        for (int kk = 0; kk < D / 16; ++kk)
                            mma_ss(tmem + C::kColDP, sw128_desc(v_addr + kk * 32, 16, 1024),
                                   sw128_desc(do_addr + kk * 32, 16, 1024), kIdescSS, kk > 0);
                        mma_commit(&sm.bar_dp_full);
                    }
                    if (ok) mma_commit(&sm.bar_kv_empty[kb]);
                } else if (warp == 2) {
                    // dV += P^T dO; the first one of a unit overwrites dV once the previous
                    // unit's dV has been copied out.
                    for (int i = 0; i < w.n_q; ++i, ++g) {
                        const int s = g % kStages;
                        if (!(ok = mbar_wait(&sm.bar_p_full, g & 1, ac))) break;
                        if (i == 0 && n > 0 && !(ok = mbar_wait(&sm.bar_dkdv_free, (n - 1) & 1, ac))) break;
                        tc_fence_after();
                        const uint32_t do_addr = smem_u32(sm.dout[s]);
#pragma unroll 1
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_ts(tmem + C::kColDV, tmem + C::kColP + kk * 8,
                                   sw128_desc(do_addr + kk * 2048, 16384, 1024), kIdescKxMN,
                                   (i > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&sm.bar_dv_done);
                        mma_commit(&sm.bar_qdo_empty[s]);
                    }
                    if (ok) mma_commit(&sm.bar_dkdv_full);
                } else if (warp == 3) {
                    // dK += dS^T Q, then dQ = dS K once the dQ warpgroup has copied out dQ(g-1)
                    for (int i = 0; i < w.n_q; ++i, ++g) {
                        const int s = g % kStages;
                        const int b = g & 1;
                        if (!(ok = mbar_wait(&sm.bar_ds_full[b], (g >> 1) & 1, ac))) break;
                        if (i == 0 && n > 0 && !(ok = mbar_wait(&sm.bar_dkdv_free, (n - 1) & 1, ac))) break;
                        tc_fence_after();
                        const uint32_t q_addr = smem_u32(sm.q[s]);
                        const uint32_t ds_addr = smem_u32(sm.ds[b]);
#pragma unroll 1
                        for (int kk = 0; kk < kTile / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            mma_ss(tmem + C::kColDK, sw128_desc(ds_addr + off, 16, 1024),
                                   sw128_desc(q_addr + kk * 2048, 16384, 1024), kIdescKxMN,
                                   (i > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(&sm.bar_qdo_empty[s]);
                        if (g > 0 && !(ok = mbar_wait(&sm.bar_dq_free, (g - 1) & 1, ac))) break;
                        tc_fence_after();
#pragma unroll 1
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_ss(tmem + C::kColDQ, sw128_desc(ds_addr + kk * 2048, 16384, 1024),
                                   sw128_desc(k_addr + kk * 2048, 16384, 1024), kIdescMNxMN, kk > 0);
                        mma_commit(&sm.bar_dq_full);      // dK(g) precedes dQ(g): both done when this fires
                    }
                    if (ok) {
                        mma_commit(&sm.bar_dkdv_full);
                        mma_commit(&sm.bar_kv_empty[kb]);
                    }
                }
            }
            // No MMA of this thread may still be running when TMEM is released.
            mma_commit(&sm.bar_drain);
            mbar_wait_drain(&sm.bar_drain, 0, p.timeout_ns);
        }
    } else if (warp < 12) {
        regs_inc<184>();
        // ------------------------------------------------------------ P / dS warpgroups (thread = key row)
        const int h = (warp - 4) >> 2;              // query-column half of this warpgroup
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        const float sl2 = p.scale_log2;
        const bool doc = p.lower2 != nullptr;
        bool ok = true;
        int g = 0;
        for (int n = 0; ok; ++n) {
            int u = -1;
            ok = __all_sync(0xffffffffu, read_unit(n, u));
            if (!ok || u < 0) break;
            const Bwd64Unit w = bwd64_unit(u, p, mask);
            const int W = w.W;
            const int key = w.k0 + r;
            for (int i = 0; i < w.n_q; ++i, ++g) {
                const int s = g % kStages;
                const int b = g & 1;
                const int qt = w.qt_lo + i;
                const int qc0 = qt * kTile + h * 64;       // first query column of this half
                if (!warp_wait(&sm.bar_qdo_full[s], (g / kStages) & 1, ac)) { ok = false; break; }
                if (!warp_wait(&sm.bar_s_full, g & 1, ac)) { ok = false; break; }
                if (!warp_wait(&sm.bar_dp_full, g & 1, ac)) { ok = false; break; }
                tc_fence_after();
                // The 64 query columns of this warpgroup are processed as two 32-column halves in a
                // loop that is not unrolled (half the code of an unrolled pass); the second half's
                // S^T and dP^T are read from TMEM while the first half is computed.
                // The diagonal tile, and tiles some of whose queries start seeing keys after this
                // key tile's first key (the tile's last row decides: lower bounds do not decrease).
                const bool need_mask = (qt == w.kt) || (doc ? sm.lower[s][kTile - 1] > w.k0
                                                            : (W > 0 && qt * kTile + kTile - 1 >= w.k0 + W));
                // Query columns that see this key form one range [c_lo, c_hi] (query >= key, and
                // query < key + W under a window): blocked pairs get score -inf, hence P = dS = 0.
                const int c_lo = key - qc0;
                const int c_hi = W > 0 ? key + W - 1 - qc0 : INT_MAX / 2;
                const uint32_t span = (uint32_t)(c_hi - c_lo);
                const uint32_t row_a = smem_u32(sm.ds[b]) + h * 16384 + r * 128;
                uint32_t xs[32], xd[32];
                tmem_ld32(t_lane + C::kColS + h * 64, xs);
                tmem_ld32(t_lane + C::kColDP + h * 64, xd);
                tmem_wait_ld_regs2(xs, xd);
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    if (need_mask) {
                        if (doc) {
                            // query column c sees this key iff c >= c_lo and lower(c) <= key
                            const int* lw = sm.lower[s] + h * 64 + hh * 32;
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                xs[e] = (hh * 32 + e >= c_lo && lw[e] <= key) ? xs[e] : 0xff800000u;
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                xs[e] = ((uint32_t)(hh * 32 + e - c_lo) <= span) ? xs[e] : 0xff800000u;   // -inf
                        }
                    }
                    const float4* lse4 = reinterpret_cast<const float4*>(sm.lse2[s] + h * 64 + hh * 32);
                    const float4* dl4 = reinterpret_cast<const float4*>(sm.delta[s] + h * 64 + hh * 32);
                    uint32_t pk[16], dk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float4 ls = lse4[e >> 2];
                        const float4 dl = dl4[e >> 2];
                        const float p0 = ex2_approx(fmaf(__uint_as_float(xs[e]), sl2, -ls.x));
                        const float p1 = ex2_approx(fmaf(__uint_as_float(xs[e + 1]), sl2, -ls.y));
                        const float p2 = ex2_approx(fmaf(__uint_as_float(xs[e + 2]), sl2, -ls.z));
                        const float p3 = ex2_approx(fmaf(__uint_as_float(xs[e + 3]), sl2, -ls.w));
                        const float d0 = p0 * (__uint_as_float(xd[e]) - dl.x);
                        const float d1 = p1 * (__uint_as_float(xd[e + 1]) - dl.y);
                        const float d2 = p2 * (__uint_as_float(xd[e + 2]) - dl.z);
                        const float d3 = p3 * (__uint_as_float(xd[e + 3]) - dl.w);
                        pk[e >> 1] = pack_bf16x2(p0, p1);
                        pk[(e >> 1) + 1] = pack_bf16x2(p2, p3);
                        dk[e >> 1] = pack_bf16x2(d0, d1);
                        dk[(e >> 1) + 1] = pack_bf16x2(d2, d3);
                    }
                    if (hh == 0) {
                        // second half in flight while the first half is stored
                        tmem_ld32(t_lane + C::kColS + h * 64 + 32, xs);
                        tmem_ld32(t_lane + C::kColDP + h * 64 + 32, xd);
                        // P^T(g) may go into TMEM once dV(g-1) has finished reading P^T(g-1); dS^T(g)
                        // into shared buffer b once dK(g-2), dQ(g-2) have finished with it.
                        if ((g > 0 && !warp_wait(&sm.bar_dv_done, (g - 1) & 1, ac)) ||
                            (g >= 2 && !warp_wait(&sm.bar_ds_empty[b], ((g >> 1) - 1) & 1, ac))) {
                            tmem_wait_ld();                // no load may be left in flight
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    tmem_st16(t_lane + C::kColP + h * 32 + hh * 16, pk);
                    // Row r of half h holds queries [64h, 64h + 64): 8 chunks of 16 bytes, swizzled by row.
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int ch = hh * 4 + c;
                        st_shared_v4(row_a + ((ch ^ (r & 7)) << 4), dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
                    }
                    if (hh == 0) {
                        tmem_wait_ld_regs2(xs, xd);
                        tc_fence_before();
                        mbar_arrive(&sm.bar_sdp_free);     // S^T, dP^T columns may be overwritten now
                    }
                }
                if (!ok) break;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.bar_p_full);
                fence_proxy_async_smem();
                mbar_arrive(&sm.bar_ds_full[b]);
            }
        }
    } else {
        regs_dec<96>();
        // ------------------------------------------------------------ dQ warpgroup (thread = query / key row)
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        bool ok = true;
        int g = 0;
        for (int n = 0; ok; ++n) {
            int u = -1;
            ok = __all_sync(0xffffffffu, read_unit(n, u));
            if (!ok || u < 0) break;
            const Bwd64Unit w = bwd64_unit(u, p, mask);
            const int kb = n & 1;
            // dK / dV of this unit (thread = key row): copied out of TMEM once the unit's last dQ
            // has been copied out and staged for its reduce-add.
            // They are staged as bf16 128B-swizzled tiles in this unit's V and K buffers, which no
            // MMA reads any more (the last dP and dQ of the unit completed before dkdv_full), and
            // written with TMA tile stores (rows past T are clipped), so every warp writes whole
            // lines.  The buffers go back to the producer once the stores have read them.
            auto write_dkdv = [&]() -> bool {
                if (!warp_wait(&sm.bar_dkdv_full, n & 1, ac)) return false;
                tc_fence_after();
#pragma unroll 1
                for (int which = 0; which < 2; ++which) {
                    const uint32_t col0 = which == 0 ? C::kColDV : C::kColDK;
                    const float mul = which == 0 ? 1.f : p.scale;     // dK = scale * dS^T Q
                    const uint32_t row_a = smem_u32(which == 0 ? sm.v[kb] : sm.k[kb]) + r * 128;
#pragma unroll 1
                    for (int c = 0; c < 2; ++c) {
                        uint32_t rr[32];
                        tmem_ld32(t_lane + col0 + c * 32, rr);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint32_t v4[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                v4[e] = pack_bf16x2(__uint_as_float(rr[8 * j + 2 * e]) * mul,
                                                    __uint_as_float(rr[8 * j + 2 * e + 1]) * mul);
                            const int chunk = c * 4 + j;             // 8 bf16 columns per 16-byte chunk
                            st_shared_v4(row_a + ((chunk ^ (r & 7)) << 4), v4[0], v4[1], v4[2], v4[3]);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&sm.bar_dkdv_free);
                fence_proxy_async_smem();
                mbar_arrive(&sm.bar_dkdv_staged);
                if (warp == 12 && lane == 0) {
                    if (!mbar_wait(&sm.bar_dkdv_staged, n & 1, ac)) return false;
                    tma_store_4d(&tm_dv, sm.v[kb], 0, w.k0, w.bh % p.H, w.bh / p.H);
                    tma_store_4d(&tm_dk, sm.k[kb], 0, w.k0, w.bh % p.H, w.bh / p.H);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                    mbar_arrive(&sm.bar_kv_empty[kb]);
                }
                return true;
            };
            for (int i = 0; i < w.n_q; ++i, ++g) {
                const int b = g & 1;
                if (!warp_wait(&sm.bar_dq_full, g & 1, ac)) { ok = false; break; }
                tc_fence_after();
                uint32_t rr[64];
                tmem_ld32(t_lane + C::kColDQ, *reinterpret_cast<uint32_t(*)[32]>(&rr[0]));
                tmem_ld32(t_lane + C::kColDQ + 32, *reinterpret_cast<uint32_t(*)[32]>(&rr[32]));
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&sm.bar_dq_free);
                // Add dQ(g) into the fp32 accumulator: stage it in dS buffer b (dK(g) and dQ(g), the
                // buffer's readers, completed before dq_full fired), two 32-column 128B-swizzled boxes,
                // then two TMA bulk reduce-adds of whole 128-byte rows (rows past T are skipped).
                const uint32_t stage = smem_u32(sm.ds[b]);
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                    const uint32_t row_a = stage + hq * 16384 + r * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        st_shared_v4(row_a + ((c ^ (r & 7)) << 4), rr[hq * 32 + 4 * c], rr[hq * 32 + 4 * c + 1],
                                     rr[hq * 32 + 4 * c + 2], rr[hq * 32 + 4 * c + 3]);
                }
                fence_proxy_async_smem();
                mbar_arrive(&sm.bar_stage_full);
                if (warp == 12 && lane == 0) {
                    if (!mbar_wait(&sm.bar_stage_full, g & 1, ac)) { ok = false; break; }
                    tma_reduce_add_3d(&tm_dq, sm.ds[b], 0, (w.qt_lo + i) * kTile, w.bh);
                    tma_reduce_add_3d(&tm_dq, sm.ds[b] + 16384, 32, (w.qt_lo + i) * kTile, w.bh);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                    mbar_arrive(&sm.bar_ds_empty[b]);        // dS(g + 2) may be written now
                }
                // The unit's dK and dV go out after its last dQ has been handed on, so the next
                // tile's dQ and dS buffer are not held up behind their copy and stores.
                if (i == w.n_q - 1 && !(ok = __all_sync(0xffffffffu, write_dkdv()))) break;
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
        }
        if (warp == 12 && lane == 0) bulk_wait_group0();   // every reduce and store has landed
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
