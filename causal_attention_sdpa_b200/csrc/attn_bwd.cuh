// Backward pass of L = sum(O * dO) for causal / sliding-window attention.
//
// The gradient is the exact one of the forward definition
// ("NanoGPT Speedrun baseline", section "El Mecanismo de Atencion"):
//   P = softmax(scale * Q K^T) (blocked keys 0), dV = P^T dO, dP = dO V^T,
//   Delta_i = dO_i . O_i, dS = P * (dP - Delta), dQ = scale dS K, dK = scale dS^T Q.
// The pages only call loss.backward(); the decomposition through Delta is an
// algebraic identity of this gradient, not a different result.
//
// Three stages run in order on the caller's stream:
//   attn_bwd_prep_kernel   Delta_i = dO_i . O_i and lse*log2(e) into padded
//                          per-head rows of the workspace; zeroes the fp32 dQ
//                          accumulator.  HBM-bound.
//   attn_bwd_kernel (D=64, attn_bwd_d64.cuh) / attn_bwd_serial_kernel (D=128,
//                          this file): per (batch*head, 128-key tile), K and V
//                          stay in shared memory while the query tiles that see
//                          them stream through a TMA ring (D=64: persistent CTAs
//                          taking these units from a counter; D=128: one CTA per
//                          unit), in the list order of schedule.h.  Per query tile, five tcgen05 MMAs:
//                            S^T  = K Q^T          (TMEM)
//                            dP^T = V dO^T         (TMEM)
//                            dV  += P^T dO         (P^T read from TMEM)
//                            dK  += dS^T Q         (dS^T from shared memory)
//                            dQ   = dS K           (same shared tile, MN-major)
//                          dQ is staged in shared memory and added into the
//                          fp32 accumulator by TMA bulk reduce-adds from a
//                          dedicated warpgroup.
//   attn_dq_convert_kernel dQ = bf16(scale * fp32 accumulator).
// dS is rounded to bf16 unscaled; the score scale is applied once per output
// element, in the dK epilogue and in the dQ conversion.
// The kernel below serves D = 128, whose accumulators fill all 512 TMEM columns
// (S^T, then P^T over it; dP^T, then dQ over it; dV; dK), so one query tile's
// P/dS pass runs at a time.  Its five 8-step MMA chains go out from three
// threads, each chain as soon as its operands and accumulator columns are free;
// Q has a two-stage ring and dO one buffer (dO's last reader, dV, comes first).
#pragma once

#include "attn_fwd.cuh"

namespace gpt_attn {

constexpr int kBwdThreads = 512;     // 16 warps

struct BwdParams {
    const float* lse2;      // [BH, T_pad]  lse * log2(e); +inf past T
    const float* delta;     // [BH, T_pad]  dO_i . O_i;    0 past T
    float* dq_acc;          // [BH, T, D]   fp32, zeroed by the prep kernel
    int* sched;             // work-unit counter of the persistent kernel, zeroed by the prep kernel
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    Strides dk_str, dv_str; // dK's and dV's layouts (the D = 128 kernel writes them with plain stores)
    int H;
    // Document masks only (else nullptr), written by the prep kernel into the workspace:
    const int* lower2;      // [BH, T_pad]   lower bound of each row's visible keys; INT_MAX past T
    const int* last_qt;     // [BH, n_tiles] last query tile that sees each key tile
    int T;
    int T_pad;
    int BH;
    int n_tiles;
    int tail;               // heads of the unit list's class-major tail (schedule.h)
    float scale_log2;       // scale * log2(e)
    float scale;
    uint64_t timeout_ns;
};

// Last query tile that sees key tile kt of head bh (window W).
__device__ __forceinline__ int bwd_last_tile(const BwdParams& p, int bh, int kt, int W) {
    return p.last_qt ? __ldg(p.last_qt + (size_t)bh * p.n_tiles + kt) : bwd_last_query_tile(kt, p.n_tiles, W);
}

template <int D>
struct BwdCfg {
    static constexpr int kStages = 2;                       // Q/dO ring depth
    static constexpr int kTileBytes = kTile * D * 2;
    static constexpr uint32_t kColS = 0;                    // S^T, then P^T (bf16) over its first 64 columns
    static constexpr uint32_t kColDP = 128;                 // dP^T, then dQ (D = 128)
    static constexpr uint32_t kColDV = 256;
    static constexpr uint32_t kColDK = 256 + D;
    static constexpr uint32_t kColDQ = (D == 64) ? 384 : kColDP;
};

// K and V of the unit, a two-stage ring of Q tiles (with their rows' lse, Delta and document
// bounds), one dO tile and the dS^T tile: 195 KB for D = 128.  Q's last reader (dK) comes at the
// end of a tile, dO's (dV) early, so Q gets the second stage.
template <int D>
struct BwdSmem {
    using C = BwdCfg<D>;
    alignas(1024) uint8_t k[C::kTileBytes];
    alignas(1024) uint8_t v[C::kTileBytes];
    alignas(1024) uint8_t q[C::kStages][C::kTileBytes];
    alignas(1024) uint8_t dout[C::kTileBytes];
    alignas(1024) uint8_t ds[kTile * kTile * 2];           // dS^T bf16 [key][query], two 64-query halves
    // 32 columns of dQ in fp32 for one bulk reduce-add into the accumulator, 128B-swizzled
    alignas(1024) uint8_t stage[kTile * 32 * 4];
    alignas(16) float lse2[C::kStages][kTile];
    alignas(16) float delta[C::kStages][kTile];
    alignas(16) int lower[C::kStages][kTile];               // document masks only
    uint64_t bar_kv;
    uint64_t bar_q_full[C::kStages];     // Q, lse, Delta (and bounds) of a query tile landed
    uint64_t bar_q_empty[C::kStages];    // dK done with the stage (S finished long before)
    uint64_t bar_do_full;
    uint64_t bar_do_empty;               // dV done with dO (dP finished long before)
    uint64_t bar_s_full;
    uint64_t bar_dp_full;
    uint64_t bar_p_full;
    uint64_t bar_ds_full;
    uint64_t bar_dv_done;         // dV(g) finished reading P^T(g) out of the S^T columns
    uint64_t bar_ds_empty;        // dK(g) and dQ(g) finished reading dS^T(g)
    uint64_t bar_dq_full;
    uint64_t bar_dq_empty;        // dQ(g) copied out of the dP^T columns
    uint64_t bar_stage_full;      // the dQ writer has staged a 32-column piece
    uint64_t bar_stage_free;      // the piece's reduce-add has read the staging buffer
    uint64_t bar_dkdv_full;
    uint64_t bar_drain;
    uint32_t tmem_base;
    int abort_flag;
};

// Delta_i = dO_i . O_i, lse2_i = lse_i * log2(e) for every padded row, and a
// zeroed fp32 dQ accumulator.  G = D / 8 threads per row, 16-byte accesses.
// No thread leaves before the group shuffle (every lane of the warp takes part).
// With document starts (lower2 != nullptr) it also writes each padded row's lower
// bound of visible keys (INT_MAX past T) and, from the first row of each key tile,
// the last query tile that sees the tile: the first rows' lower bounds do not
// decrease, so the query tiles that see a key tile are the ones up to the last
// whose first row's lower bound is at or before the tile's last key.
template <int D>
__global__ void __launch_bounds__(256)
attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                     const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ delta,
                     float* __restrict__ dq_acc, int* __restrict__ sched, int T, int T_pad,
                     long long total_rows_pad, const MaskParams mask, int* __restrict__ lower2,
                     int* __restrict__ last_qt, int n_tiles, const Strides o_str, const Strides do_str, int H) {
    constexpr int G = D / 8;
    if (blockIdx.x == 0 && threadIdx.x == 0) *sched = 0;
    const long long row = (long long)blockIdx.x * (256 / G) + threadIdx.x / G;
    const int g = threadIdx.x % G;
    const bool in_range = row < total_rows_pad;
    const long long bh = in_range ? row / T_pad : 0;
    const int t = in_range ? (int)(row - bh * T_pad) : 0;
    const bool valid = in_range && t < T;
    float acc = 0.f;
    long long src = 0;
    if (valid) {
        src = (bh * T + t) * (long long)D + g * 8;
        const uint4 a = *reinterpret_cast<const uint4*>(o + o_str.row((int)bh, H, t) + g * 8);
        const uint4 b = *reinterpret_cast<const uint4*>(dout + do_str.row((int)bh, H, t) + g * 8);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
            const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
            acc = fmaf(fa.x, fb.x, acc);
            acc = fmaf(fa.y, fb.y, acc);
        }
        float4* z = reinterpret_cast<float4*>(dq_acc + src);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (in_range && g == 0) {
        delta[row] = valid ? acc : 0.f;
        lse2[row] = valid ? lse[bh * T + t] * 1.4426950408889634f : INFINITY;
        if (lower2) {
            const int W = mask_window(mask, (int)bh);
            lower2[row] = valid ? mask_row_lower(mask, (int)bh, T, W, t) : INT_MAX;
            if ((t & (kTile - 1)) == 0) {
                const int b = (int)bh;
                last_qt[bh * n_tiles + t / kTile] = bwd_last_query_tile_lb(
                    t / kTile, n_tiles, [&](int qt) { return mask_row_lower(mask, b, T, W, qt * kTile); });
            }
        }
    }
}

// dQ = bf16(scale * acc): G = D / 8 threads per row of the accumulator [BH, T, D], 8 elements
// (two 16-byte loads, one 16-byte store) each, written to dQ's layout.  One division per thread
// finds the row's head.
template <int D>
__global__ void __launch_bounds__(256)
attn_dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, long long rows, float scale,
                       int T, int H, const Strides dq_str) {
    constexpr int G = D / 8;
    const long long row = (long long)blockIdx.x * (256 / G) + threadIdx.x / G;
    if (row >= rows) return;
    const int g = threadIdx.x % G;
    const float4 a = reinterpret_cast<const float4*>(acc + row * D)[2 * g];
    const float4 b = reinterpret_cast<const float4*>(acc + row * D)[2 * g + 1];
    uint4 r;
    r.x = pack_bf16x2(a.x * scale, a.y * scale);
    r.y = pack_bf16x2(a.z * scale, a.w * scale);
    r.z = pack_bf16x2(b.x * scale, b.y * scale);
    r.w = pack_bf16x2(b.z * scale, b.w * scale);
    const int bh = (int)(row / T);
    *reinterpret_cast<uint4*>(dq + dq_str.row(bh, H, row - (long long)bh * T) + g * 8) = r;
}

template <int D, typename Mask>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_serial_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_dq,
                const BwdParams p, const __grid_constant__ Mask mask) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(smem_align1024(smem_raw));

    constexpr int kStages = C::kStages;
    constexpr int kTileBytes = C::kTileBytes;
    constexpr int kBoxes = D / 64;
    constexpr uint32_t kTmemCols = 512;
    constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);    // S^T, dP^T
    constexpr uint32_t kIdescKxMN = idesc_bf16_f32(128, D, 0, 1);    // dV (A in TMEM), dK
    constexpr uint32_t kIdescMNxMN = idesc_bf16_f32(128, D, 1, 1);   // dQ

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Blocks of one head are adjacent in launch order (its Q, dO and dQ rows stay in
    // L2 across its key tiles); key tile 0 sees the most query tiles and launches first.
    int bh, kt;
    list_item(blockIdx.x, p.BH, p.n_tiles, p.tail, bh, kt);   // unit list order of schedule.h
    const int k0 = kt * kTile;
    const int qt_lo = kt;
    const int W = mask.head_window(bh);
    const int qt_hi = bwd_last_tile(p, bh, kt, W);
    const int n_q = qt_hi - qt_lo + 1;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_kv, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.bar_q_full[s], 1);
            mbar_init(&sm.bar_q_empty[s], 1);
        }
        mbar_init(&sm.bar_do_full, 1);
        mbar_init(&sm.bar_do_empty, 1);
        mbar_init(&sm.bar_s_full, 1);
        mbar_init(&sm.bar_dp_full, 1);
        mbar_init(&sm.bar_p_full, 256);             // both P/dS warpgroups
        mbar_init(&sm.bar_ds_full, 256);
        mbar_init(&sm.bar_dv_done, 1);
        mbar_init(&sm.bar_ds_empty, 2);             // dK issuer + dQ issuer
        mbar_init(&sm.bar_dq_full, 1);
        mbar_init(&sm.bar_dq_empty, 128);
        mbar_init(&sm.bar_stage_full, 128);
        mbar_init(&sm.bar_stage_free, 1);
        mbar_init(&sm.bar_dkdv_full, 1);
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

    // Launched with 128 registers per thread (512 x 128 = 65536): warpgroup 0 (producer and MMA
    // issuers) drops to 64, the P/dS warpgroups take 136, the dQ writer 176 to hold a whole row of
    // dQ: 128 x (64 + 136 + 136 + 176) = 65536.
    if (warp < 4) {
        regs_dec<64>();
        if (warp == 0) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_v);
                tma_prefetch_desc(&tm_do);
                const int hh = bh % p.H, bb = bh / p.H;
                mbar_arrive_expect_tx(&sm.bar_kv, 2 * kTileBytes);
                for (int b = 0; b < kBoxes; ++b) {
                    tma_load_4d(sm.k + b * 16384, &tm_k, &sm.bar_kv, b * 64, k0, hh, bb);
                    tma_load_4d(sm.v + b * 16384, &tm_v, &sm.bar_kv, b * 64, k0, hh, bb);
                }
                int nq = 0, ndo = 0;           // Q and dO tiles whose loads were issued
                for (int it = 0; it < n_q; ++it) {
                    const int s = it % kStages;
                    const int n = it / kStages;
                    if (n > 0 && !mbar_wait(&sm.bar_q_empty[s], (n - 1) & 1, ac)) break;
                    if (debug_skip_load(2, it)) continue;           // debug builds: exercise the abort path
                    const int q0 = (qt_lo + it) * kTile;
                    mbar_arrive_expect_tx(&sm.bar_q_full[s], kTileBytes + (p.lower2 ? 3 : 2) * kTile * 4);
                    for (int b = 0; b < kBoxes; ++b)
                        tma_load_4d(sm.q[s] + b * 16384, &tm_q, &sm.bar_q_full[s], b * 64, q0, hh, bb);
                    const size_t roff = (size_t)bh * p.T_pad + q0;
                    bulk_load(sm.lse2[s], p.lse2 + roff, kTile * 4, &sm.bar_q_full[s]);
                    bulk_load(sm.delta[s], p.delta + roff, kTile * 4, &sm.bar_q_full[s]);
                    if (p.lower2) bulk_load(sm.lower[s], p.lower2 + roff, kTile * 4, &sm.bar_q_full[s]);
                    nq = it + 1;
                    if (it > 0 && !mbar_wait(&sm.bar_do_empty, (it - 1) & 1, ac)) break;
                    mbar_arrive_expect_tx(&sm.bar_do_full, kTileBytes);
                    for (int b = 0; b < kBoxes; ++b)
                        tma_load_4d(sm.dout + b * 16384, &tm_do, &sm.bar_do_full, b * 64, q0, hh, bb);
                    ndo = it + 1;
                }
                if (sm.abort_flag) {
                    // Let every load already issued land before the CTA exits.
                    mbar_wait_drain(&sm.bar_kv, 0, p.timeout_ns);
                    for (int r = (nq > kStages ? nq - kStages : 0); r < nq; ++r)
                        mbar_wait_drain(&sm.bar_q_full[r % kStages], (r / kStages) & 1, p.timeout_ns);
                    if (ndo > 0) mbar_wait_drain(&sm.bar_do_full, (ndo - 1) & 1, p.timeout_ns);
                }
            }
        } else {
            // ------------------------------------------------------------ MMA issuers
            // One thread issues one tcgen05.mma per ~130 cycles, so the five 8-step chains of a tile
            // go out from three threads, each as soon as its operands and accumulator are free:
            //   warp 1: S^T(g) once dV(g-1) has read P^T(g-1) out of the S^T columns
            //   warp 2: dP^T(g) once dQ(g-1) has been copied out of the dP^T columns, then dQ(g) into
            //           those columns once the P/dS warpgroup has read dP^T(g) and written dS^T(g)
            //   warp 3: dV(g) once P^T(g) is in TMEM, then dK(g) once dS^T(g) is in shared memory
            if (lane == 0) {
                const uint32_t k_addr = smem_u32(sm.k);
                const uint32_t v_addr = smem_u32(sm.v);
                const uint32_t ds_addr = smem_u32(sm.ds);
                bool ok = mbar_wait(&sm.bar_kv, 0, ac);
                for (int it = 0; ok && it < n_q; ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    const uint32_t q_addr = smem_u32(sm.q[s]);
                    const uint32_t do_addr = smem_u32(sm.dout);
                    if (warp == 1) {
                        if (!(ok = mbar_wait(&sm.bar_q_full[s], ph, ac))) break;
                        if (it > 0 && !(ok = mbar_wait(&sm.bar_dv_done, (it - 1) & 1, ac))) break;
                        tc_fence_after();
    #pragma unroll 1
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            mma_ss(tmem + C::kColS, sw128_desc(k_addr + off, 16, 1024),
                                   sw128_desc(q_addr + off, 16, 1024), kIdescSS, kk > 0);
                        }
                        mma_commit(&sm.bar_s_full);
                    } else if (warp == 2) {
                        if (!(ok = mbar_wait(&sm.bar_do_full, it & 1, ac))) break;
                        if (it > 0 && !(ok = mbar_wait(&sm.bar_dq_empty, (it - 1) & 1, ac))) break;
                        tc_fence_after();
    #pragma unroll 1
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            mma_ss(tmem + C::kColDP, sw128_desc(v_addr + off, 16, 1024),
                                   sw128_desc(do_addr + off, 16, 1024), kIdescSS, kk > 0);
                        }
                        mma_commit(&sm.bar_dp_full);
                        // dQ = dS K
                        if (!(ok = mbar_wait(&sm.bar_ds_full, it & 1, ac))) break;
                        tc_fence_after();
    #pragma unroll 1
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_ss(tmem + C::kColDQ, sw128_desc(ds_addr + kk * 2048, 16384, 1024),
                                   sw128_desc(k_addr + kk * 2048, 16384, 1024), kIdescMNxMN, kk > 0);
                        mma_commit(&sm.bar_dq_full);
                        mma_commit(&sm.bar_ds_empty);
                    } else {
                        // dV += P^T dO
                        if (!(ok = mbar_wait(&sm.bar_p_full, it & 1, ac))) break;
                        tc_fence_after();
    #pragma unroll 1
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_ts(tmem + C::kColDV, tmem + C::kColS + (kk >> 2) * 64 + (kk & 3) * 8,
                                   sw128_desc(do_addr + kk * 2048, 16384, 1024), kIdescKxMN,
                                   (it > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&sm.bar_dv_done);
                        mma_commit(&sm.bar_do_empty);          // dV was dO's last reader
                        // dK += dS^T Q
                        if (!(ok = mbar_wait(&sm.bar_ds_full, it & 1, ac))) break;
                        tc_fence_after();
    #pragma unroll 1
                        for (int kk = 0; kk < kTile / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            mma_ss(tmem + C::kColDK, sw128_desc(ds_addr + off, 16, 1024),
                                   sw128_desc(q_addr + kk * 2048, 16384, 1024), kIdescKxMN,
                                   (it > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(&sm.bar_ds_empty);
                        mma_commit(&sm.bar_q_empty[s]);        // dK was Q's last reader
                    }
                }
                if (warp == 3 && ok) mma_commit(&sm.bar_dkdv_full);
                // No MMA of this thread may still be running when TMEM is released.
                mma_commit(&sm.bar_drain);
                mbar_wait_drain(&sm.bar_drain, 0, p.timeout_ns);
            }
    }
    } else if (warp < 12) {
        regs_inc<136>();
        // ------------------------------------------------------------ P / dS warpgroups (thread = key row)
        // Warpgroup h takes query columns [64h, 64h + 64) of each tile and writes their P^T over
        // S^T columns it has read itself: queries 64h + q go to bf16 column 64h + q/2 of the S^T
        // block, so neither warpgroup overwrites scores the other still has to read.
        const int h = (warp - 4) >> 2;
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const int key = k0 + r;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        const float sl2 = p.scale_log2;
        const bool doc = p.lower2 != nullptr;
        const uint32_t ds_row = smem_u32(sm.ds) + r * 128;
        bool ok = true;
        for (int it = 0; it < n_q; ++it) {
            const int s = it % kStages;
            const int qt = qt_lo + it;
            const int q0 = qt * kTile;
            if (!warp_wait(&sm.bar_q_full[s], (it / kStages) & 1, ac)) { ok = false; break; }
            if (!warp_wait(&sm.bar_s_full, it & 1, ac)) { ok = false; break; }
            if (!warp_wait(&sm.bar_dp_full, it & 1, ac)) { ok = false; break; }
            tc_fence_after();
            // The tile needs the per-element mask if it holds the diagonal or some query of it
            // starts seeing keys after this key tile's first key (lower bounds do not decrease
            // down a tile, so its last row decides).
            const bool need_mask =
                (qt == kt) || (doc ? sm.lower[s][kTile - 1] > k0 : (W > 0 && q0 + kTile - 1 >= k0 + W));
            const float2* lse2 = reinterpret_cast<const float2*>(sm.lse2[s]);
            const float2* dlt = reinterpret_cast<const float2*>(sm.delta[s]);
#pragma unroll 1
            for (int c = 2 * h; c < 2 * h + 2; ++c) {
                uint32_t rs[32], rd[32];
                tmem_ld32(t_lane + C::kColS + c * 32, rs);
                tmem_ld32(t_lane + C::kColDP + c * 32, rd);
                tmem_wait_ld();
                if (need_mask) {
                    const int c_lo = key - (q0 + c * 32);
                    if (doc) {
                        // query q sees this key iff q >= key and lower(q) <= key
                        const int* lw = sm.lower[s] + c * 32;
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            rs[e] = (e >= c_lo && lw[e] <= key) ? rs[e] : 0xff800000u;   // -inf: P = 0
                    } else {
                        // visible query columns of this key: one range, compare + select per element
                        const int c_hi = W > 0 ? key + W - 1 - (q0 + c * 32) : INT_MAX / 2;
                        const uint32_t span = (uint32_t)(c_hi - c_lo);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            rs[e] = ((uint32_t)(e - c_lo) <= span) ? rs[e] : 0xff800000u;   // -inf: P = 0
                    }
                }
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int col = c * 32 + e;
                    const float2 ls = lse2[col >> 1];
                    const float2 dl = dlt[col >> 1];
                    const float p0 = ex2_approx(__uint_as_float(rs[e]) * sl2 - ls.x);
                    const float p1 = ex2_approx(__uint_as_float(rs[e + 1]) * sl2 - ls.y);
                    const float d0 = p0 * (__uint_as_float(rd[e]) - dl.x);
                    const float d1 = p1 * (__uint_as_float(rd[e + 1]) - dl.y);
                    pk[e >> 1] = pack_bf16x2(p0, p1);
                    dk[e >> 1] = pack_bf16x2(d0, d1);
                }
                tmem_st16(t_lane + C::kColS + h * 64 + (c & 1) * 16, pk);
                // dS^T(it) may go into the shared buffer once dK(it-1) and dQ(it-1) have read it.
                if (c == 2 * h && it > 0 && !warp_wait(&sm.bar_ds_empty, (it - 1) & 1, ac)) {
                    tmem_wait_st();                    // no store may be left in flight
                    ok = false;
                    break;
                }
                // dS^T row r, queries [32c, 32c + 32): 4 chunks of 16 bytes in half c/2, swizzled by row.
                const uint32_t half = ds_row + (c >> 1) * 16384;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint32_t chunk = ((c & 1) * 4 + t) ^ (r & 7);
                    st_shared_v4(half + chunk * 16, dk[4 * t], dk[4 * t + 1], dk[4 * t + 2], dk[4 * t + 3]);
                }
            }
            if (!ok) break;
            tmem_wait_st();
            tc_fence_before();
            fence_proxy_async_smem();
            mbar_arrive(&sm.bar_p_full);
            mbar_arrive(&sm.bar_ds_full);
        }
        // ---------------------------------------------------------- dK / dV epilogue
        if (__all_sync(0xffffffffu, ok) && warp_wait(&sm.bar_dkdv_full, 0, ac)) {
            tc_fence_after();
            const bool store = key < p.T;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                __nv_bfloat16* dst_row = which == 0 ? p.dv + p.dv_str.row(bh, p.H, store ? key : 0)
                                                    : p.dk + p.dk_str.row(bh, p.H, store ? key : 0);
                const uint32_t col0 = which == 0 ? C::kColDV : C::kColDK;
                const float mul = which == 0 ? 1.f : p.scale;     // dK = scale * dS^T Q
#pragma unroll
                for (int c = h * D / 64; c < (h + 1) * D / 64; ++c) {     // this warpgroup's half of D
                    uint32_t rr[32];
                    tmem_ld32(t_lane + col0 + c * 32, rr);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        pk[e >> 1] = pack_bf16x2(__uint_as_float(rr[e]) * mul, __uint_as_float(rr[e + 1]) * mul);
                    if (store) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            d4[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
                    }
                }
            }
        }
    } else {
        regs_inc<176>();
        // ------------------------------------------------------------ dQ writer warpgroup (thread = query row)
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        for (int it = 0; it < n_q; ++it) {
            if (!warp_wait(&sm.bar_dq_full, it & 1, ac)) break;
            tc_fence_after();
            // The whole row comes out of TMEM first, so the next tile's dP^T may overwrite the
            // columns at once.  Then it is added into the fp32 accumulator in four 32-column
            // pieces, each staged in shared memory and sent by one TMA bulk reduce-add (rows past T
            // are skipped): the tensor cores' shared-memory reads slow down badly under as many
            // vector red.global.add from the LSU.
            static_assert(D == 128, "the dQ writer holds a row as four 32-column pieces");
            uint32_t r0[32], r1[32], r2[32], r3[32];
            tmem_ld32(t_lane + C::kColDQ, r0);
            tmem_ld32(t_lane + C::kColDQ + 32, r1);
            tmem_ld32(t_lane + C::kColDQ + 64, r2);
            tmem_ld32(t_lane + C::kColDQ + 96, r3);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_dq_empty);
            const uint32_t row_a = smem_u32(sm.stage) + r * 128;
            auto put = [&](int j, const uint32_t (&v)[32]) -> bool {
                const int n = it * 4 + j;                 // pieces staged so far
                if (n > 0 && !warp_wait(&sm.bar_stage_free, (n - 1) & 1, ac)) return false;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(row_a + ((c ^ (r & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                fence_proxy_async_smem();
                mbar_arrive(&sm.bar_stage_full);
                bool lok = true;
                if (warp == 12 && lane == 0) {
                    lok = mbar_wait(&sm.bar_stage_full, n & 1, ac);
                    if (lok) {
                        tma_reduce_add_3d(&tm_dq, sm.stage, j * 32, (qt_lo + it) * kTile, bh);
                        bulk_commit_group();
                        bulk_wait_group_read0();
                        mbar_arrive(&sm.bar_stage_free);
                    }
                }
                return __all_sync(0xffffffffu, lok);
            };
            if (!put(0, r0) || !put(1, r1) || !put(2, r2) || !put(3, r3)) break;
        }
        if (warp == 12 && lane == 0) bulk_wait_group0();   // every reduce-add has landed
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
