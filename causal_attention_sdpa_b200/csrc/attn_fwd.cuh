// Forward kernel: O = softmax(scale * Q K^T) V with causal / sliding-window
// masking, plus the natural-log row log-sum-exp.
//
// The tiling follows the FlashAttention idea the GPT-2 lecture describes in
// "Раздел 2" (never materialise the T x T matrix; softmax in pieces with a
// running max m and running sum l, rescaling the old sum by e^(m_old - m_new)
// when the max grows).  The mapping onto sm_100a is this file's own:
//
//   one work item = one (batch*head, 256-query block) = two 128-row Q tiles sharing
//   every K/V tile it loads.  Only one block fits on an SM, and a block that starts
//   does not stop after one item: the producer warp fetches item after item and passes
//   each to the other roles through a two-slot ring in shared memory, and every
//   barrier phase counts tiles over all the items a role has handled, so the next
//   item's Q load and first scores overlap the current item's last tiles and epilogue.
//   The items come in one of two orders (schedule.h):
//     - on demand: the grid has one block per item, in list order (head-major, so the
//       blocks of a head run at the same time and its K/V tiles come from HBM once and
//       from L2 to the others; a tail that ends with short items); each running block
//       takes the next item by cancelling, through cluster launch control, the launch
//       of the first block that has not started;
//     - static, for work of many full rounds: one block per SM, each running a fixed
//       sequence of items in waves of whole heads, its block class rotating from one
//       wave to the next.
//   12 warps:
//     warp 0       TMA producer and work-item fetcher: Q0, Q1 once, then K_j / V_j through a ring
//     warp 1       TMEM allocator; issues S0 = Q0 K_j^T and S1 = Q1 K_j^T
//     warps 2, 3   issue O0 += P0 V_j and O1 += P1 V_j (one MMA stream per warp)
//     warps 4..7   softmax warpgroup of Q tile 0 (thread r owns query row r)
//     warps 8..11  softmax warpgroup of Q tile 1
//   TMEM (512 columns):
//     D = 64 : S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384) O0 [384,448) O1 [448,512)
//     D = 128: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); P_t is written over S_t
//   With separate P columns (D = 64) a softmax warpgroup hands its S columns back as
//   soon as it has read them into registers, so the MMA warp computes S(j+1) while the
//   exponentials of S(j) are still running.  With P written over S (D = 128)
//   each S waits for the PV that read its columns.
//
// The running max is rescaled lazily: O and l are rescaled only when a row's max
// grows by more than 8 (log2 units) over the max the exponentials use.  Every
// probability then stays <= 2^8, and since the final O / l and lse use the same
// reference max the result is unchanged.
//
// Key tiles entirely after a Q tile's last query, or entirely before the window
// of its first query, are never loaded for it; only the diagonal tile and the
// window-edge tiles evaluate the visibility predicate.
#pragma once

#include <climits>

#include "schedule.h"
#include "sm100.cuh"

namespace gpt_attn {

constexpr int kFwdThreads = 384;
constexpr float kLazyRescale = 8.0f; // log2 units

// Which keys each query sees, shared by the forward and backward kernels.  The kernels are
// instantiated for two mask types with the same interface: WindowMask (causal, or one window for
// every head: the common case, with nothing but one integer in the kernel parameters) and
// MaskParams (a window per head position h = bh % H, and optional document starts [B, T] in
// device memory, row b = bh / H).
struct WindowMask {
    int window;                // <= 0: causal only
    __device__ __forceinline__ int head_window(int) const { return window; }
    // Lower bound of the keys query i sees (schedule.h row_lower).
    __device__ __forceinline__ int row_lower_of(int, int, int W, int i) const { return row_lower(i, W, 0); }
    static constexpr bool kDoc = false;
};

constexpr int kMaxHeadWindows = 64;   // per-head windows travel in the kernel parameters

struct MaskParams {
    const int* doc_start;      // nullptr: each row is one document
    int H;
    int window;                // used when head_windows == 0; <= 0: causal only
    int head_windows;          // 1: win[bh % H]
    int win[kMaxHeadWindows];
    __device__ __forceinline__ int head_window(int bh) const { return head_windows ? win[bh % H] : window; }
    // Rows past T use the document of the last token.
    __device__ __forceinline__ int row_lower_of(int bh, int T, int W, int i) const {
        int d = 0;
        if (doc_start) d = __ldg(doc_start + (size_t)(bh / H) * T + (i < T ? i : T - 1));
        return row_lower(i, W, d);
    }
    static constexpr bool kDoc = true;
};

__device__ __forceinline__ int mask_window(const MaskParams& m, int bh) { return m.head_window(bh); }
__device__ __forceinline__ int mask_row_lower(const MaskParams& m, int bh, int T, int W, int i) {
    return m.row_lower_of(bh, T, W, i);
}

// Element strides of a bf16 tensor indexed [b, h, t, d] (d contiguous).
struct Strides {
    long long b, h, t;
    __host__ __device__ __forceinline__ long long row(int bh, int H, long long t_) const {
        return (long long)(bh / H) * b + (long long)(bh % H) * h + t_ * t;
    }
};

struct FwdParams {
    __nv_bfloat16* o;
    float* lse;
    Strides o_str;        // O's layout (the D = 128 epilogue writes O with plain stores)
    int H;
    int T;
    int BH;
    int n_tiles;          // ceil(T / 128)
    int n_blocks;         // ceil(n_tiles / 2): 256-query blocks per head
    int tail;             // heads of the item list's class-major tail (schedule.h)
    int static_hpw;       // static order (schedule.h): heads per wave, and
    int static_waves;     // waves (0: items taken from the list through cluster launch control)
    float scale_log2;     // scale * log2(e)
    uint64_t timeout_ns;
};

// Item i of the list: head bh and 256-query block qb.
__device__ __forceinline__ void fwd_list_item(const FwdParams& p, int i, int& bh, int& qb) {
    fwd_item(i, p.BH, p.n_blocks, p.tail, bh, qb);
}

// This block's static item after wave *k (advancing *k past it); bh = -1 when there is none.
__device__ __forceinline__ void fwd_next_static_item(const FwdParams& p, int& k, int& bh, int& qb) {
    bh = -1;
    for (; k < p.static_waves; ++k) {
        fwd_static_item(p.static_hpw, p.n_blocks, p.BH, blockIdx.x, k, bh, qb);
        if (bh >= 0) {
            ++k;
            return;
        }
    }
}

// Roles that read each work item from the ring: the S warp, the two PV warps (one lane each) and
// the eight softmax warps (one arrival per warp).
constexpr int kFwdItemReaders = 3 + 8;

// Key tiles [lo, hi] of query tile qt of head bh with window W.
template <typename Mask>
__device__ __forceinline__ void fwd_tile_range(const FwdParams& p, const Mask& m, int bh, int W, int qt, int& lo,
                                               int& hi) {
    fwd_key_range_lb(qt, m.row_lower_of(bh, p.T, W, qt * kTile), lo, hi);
}

template <int D>
struct FwdCfg {
    static constexpr int kStages = (D == 64) ? 3 : 2;
    static constexpr int kQBufs = (D == 64) ? 2 : 1;   // items whose Q tiles can be resident at once
    static constexpr int kTileBytes = kTile * D * 2;
    static constexpr bool kSeparateP = (D == 64);
    static constexpr bool kOStage = (D == 64);          // O tiles staged in shared memory for TMA stores
    static constexpr uint32_t kColS0 = 0, kColS1 = 128;
    static constexpr uint32_t kColP0 = kSeparateP ? 256u : 0u, kColP1 = kSeparateP ? 320u : 128u;
    static constexpr uint32_t kColO0 = kSeparateP ? 384u : 256u, kColO1 = kSeparateP ? 448u : 384u;
};

template <int D>
struct FwdSmem {
    using C = FwdCfg<D>;
    alignas(1024) uint8_t q[C::kQBufs][2][C::kTileBytes];
    alignas(1024) uint8_t k[C::kStages][C::kTileBytes];
    alignas(1024) uint8_t v[C::kStages][C::kTileBytes];
    alignas(1024) uint8_t ostage[C::kOStage ? 2 : 1][C::kOStage ? C::kTileBytes : 16];
    uint64_t bar_q[C::kQBufs];
    uint64_t bar_q_empty[C::kQBufs];  // every S MMA of the item using this Q buffer finished
    uint64_t bar_k[C::kStages];
    uint64_t bar_v[C::kStages];
    uint64_t bar_kv_empty[C::kStages];
    uint64_t bar_s_full[2];
    uint64_t bar_s_free[2];
    uint64_t bar_p_full[2];
    uint64_t bar_o_done[2];
    uint64_t bar_o_free[2];       // softmax warpgroup t has read its item's O out of TMEM
    uint64_t bar_ostage_free[2];  // warpgroup t's previous O tile store has read its staging buffer
    uint64_t bar_ostage_full[2];  // warpgroup t has staged its O tile
    uint64_t bar_drain;
    uint64_t bar_item_full[2];    // work-item ring: slot written by the producer
    uint64_t bar_item_empty[2];   // slot read by every role
    uint64_t bar_clc;             // cluster launch control response landed
    alignas(16) uint32_t clc_resp[4];
    int item_bh[2];               // work item: head, or -1 when there is none left,
    int item_qb[2];               // and 256-query block
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int D, typename Mask>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const FwdParams p, const __grid_constant__ Mask mask) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    FwdSmem<D>& sm = *reinterpret_cast<FwdSmem<D>*>(smem_align1024(smem_raw));

    constexpr int kStages = C::kStages;
    constexpr int kQBufs = C::kQBufs;
    constexpr int kTileBytes = C::kTileBytes;
    constexpr int kBoxes = D / 64;                 // 64-column TMA boxes per tile
    constexpr uint32_t kTmemCols = 512;
    constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < kQBufs; ++b) {
            mbar_init(&sm.bar_q[b], 1);
            mbar_init(&sm.bar_q_empty[b], 1);         // S warp
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.bar_k[s], 1);
            mbar_init(&sm.bar_v[s], 1);
            mbar_init(&sm.bar_kv_empty[s], 3);        // S warp + two PV warps
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&sm.bar_s_full[t], 1);
            mbar_init(&sm.bar_s_free[t], 128);
            mbar_init(&sm.bar_p_full[t], 128);
            mbar_init(&sm.bar_o_done[t], 1);
            mbar_init(&sm.bar_o_free[t], 128);
            mbar_init(&sm.bar_ostage_free[t], 1);
            mbar_init(&sm.bar_ostage_full[t], 128);
        }
        mbar_init(&sm.bar_drain, 3);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.bar_item_full[b], 1);
            mbar_init(&sm.bar_item_empty[b], kFwdItemReaders);
        }
        mbar_init(&sm.bar_clc, 1);
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
    // Work item n of this block for a single-lane role: waits for ring slot n % 2, reads it,
    // releases it.
    auto read_item = [&](int n, int& bh, int& qb) -> bool {
        const int slot = n & 1;
        if (!mbar_wait(&sm.bar_item_full[slot], (n >> 1) & 1, ac)) return false;
        bh = *reinterpret_cast<volatile int*>(&sm.item_bh[slot]);
        qb = *reinterpret_cast<volatile int*>(&sm.item_qb[slot]);
        mbar_arrive(&sm.bar_item_empty[slot]);
        return true;
    };
    // Launched with 168 registers per thread (384 x 168 = 64512): warpgroup 0
    // (producer, MMA) drops to 56, the softmax warpgroups take 224:
    // 128 x 56 + 256 x 224 = 64512.  The softmax pass runs faster with 224 than with
    // 216 (more exponentials in flight); 232 gains nothing more.
    // Each role's code sits under its own setmaxnreg so the compiler allocates it
    // with that role's budget.
    if (warp < 4) {
        regs_dec<56>();
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int it = 0;              // K/V tiles loaded, over all items
            int n_item = 0;          // items whose Q was loaded
            int n_clc = 0;           // launch-control responses received
            bool clc_pending = false;
            bool ok = true;
            const bool dynamic = p.static_waves == 0;
            int k_static = 0;        // static order: next wave
            // This block's own item first.
            int bh, qb;
            if (dynamic)
                fwd_list_item(p, blockIdx.x, bh, qb);
            else
                fwd_next_static_item(p, k_static, bh, qb);
            for (int n = 0; ok; ++n) {
                const int slot = n & 1;
                if (n >= 2 && !(ok = mbar_wait(&sm.bar_item_empty[slot], ((n >> 1) - 1) & 1, ac))) break;
                *reinterpret_cast<volatile int*>(&sm.item_bh[slot]) = bh;
                *reinterpret_cast<volatile int*>(&sm.item_qb[slot]) = qb;
                mbar_arrive(&sm.bar_item_full[slot]);
                if (bh < 0) break;
                if (dynamic) {
                    // Ask now for the item after this one (the item of the first block that has not
                    // started); the answer is read once this item's loads are out.
                    mbar_arrive_expect_tx(&sm.bar_clc, 16);
                    clc_try_cancel(sm.clc_resp, &sm.bar_clc);
                    clc_pending = true;
                }
                const int W = mask.head_window(bh);
                int lo0, hi0, lo1, hi1;
                fwd_tile_range(p, mask, bh, W, 2 * qb, lo0, hi0);
                fwd_tile_range(p, mask, bh, W, 2 * qb + 1, lo1, hi1);
                const int qbuf = n_item % kQBufs;
                if (n_item >= kQBufs &&
                    !(ok = mbar_wait(&sm.bar_q_empty[qbuf], ((n_item / kQBufs) - 1) & 1, ac)))
                    break;
                const int hh = bh % p.H, bb = bh / p.H;
                mbar_arrive_expect_tx(&sm.bar_q[qbuf], 2 * kTileBytes);
                for (int t = 0; t < 2; ++t)
                    for (int b = 0; b < kBoxes; ++b)
                        tma_load_4d(sm.q[qbuf][t] + b * 16384, &tm_q, &sm.bar_q[qbuf], b * 64, (2 * qb + t) * kTile,
                                    hh, bb);
                ++n_item;
                for (int j = lo0; j <= hi1; ++j, ++it) {
                    const int s = it % kStages;
                    const int n = it / kStages;
                    if (n > 0 && !(ok = mbar_wait(&sm.bar_kv_empty[s], (n - 1) & 1, ac))) break;
                    if (debug_skip_load(1, it)) continue;         // debug builds: exercise the abort path
                    mbar_arrive_expect_tx(&sm.bar_k[s], kTileBytes);
                    for (int b = 0; b < kBoxes; ++b)
                        tma_load_4d(sm.k[s] + b * 16384, &tm_k, &sm.bar_k[s], b * 64, j * kTile, hh, bb);
                    mbar_arrive_expect_tx(&sm.bar_v[s], kTileBytes);
                    for (int b = 0; b < kBoxes; ++b)
                        tma_load_4d(sm.v[s] + b * 16384, &tm_v, &sm.bar_v[s], b * 64, j * kTile, hh, bb);
                }
                if (!ok) break;
                if (!dynamic) {
                    fwd_next_static_item(p, k_static, bh, qb);
                    continue;
                }
                if (!(ok = mbar_wait(&sm.bar_clc, n_clc & 1, ac))) break;
                clc_pending = false;
                ++n_clc;
                const int b = clc_cancelled_block(sm.clc_resp);
                if (b < 0)
                    bh = -1;
                else
                    fwd_list_item(p, b, bh, qb);
            }
            // A request still out when the block gave up must land before the block exits.
            if (clc_pending) mbar_wait_drain(&sm.bar_clc, n_clc & 1, p.timeout_ns);
            if (sm.abort_flag) {
                // Let every load already issued land before the CTA exits.
                for (int r = (n_item > kQBufs ? n_item - kQBufs : 0); r < n_item; ++r)
                    mbar_wait_drain(&sm.bar_q[r % kQBufs], (r / kQBufs) & 1, p.timeout_ns);
                for (int r = (it > kStages ? it - kStages : 0); r < it; ++r) {
                    mbar_wait_drain(&sm.bar_k[r % kStages], (r / kStages) & 1, p.timeout_ns);
                    mbar_wait_drain(&sm.bar_v[r % kStages], (r / kStages) & 1, p.timeout_ns);
                }
            }
        }
    } else if (lane == 0) {
        // ------------------------------------------------------------ MMA issuers
        // One tcgen05.mma stream per warp: a single issuing thread cannot keep the
        // tensor pipe busy with 128-row MMAs of N <= 128, several streams can.
        //   warp 1: S0 = Q0 K_j^T and S1 = Q1 K_j^T
        //   warp 2: O0 += P0 V_j        warp 3: O1 += P1 V_j
        // Each of the three warps releases a K/V stage once its own MMAs on it are done (the S
        // warp also on behalf of a PV warp with no work on the tile).
        bool ok = true;
        int it = 0;                  // K/V tiles consumed, over all items
        int n_item = 0;
        if (warp == 1) {
            int ct[2] = {0, 0};      // S tiles issued per warpgroup, over all items
            for (int n = 0; ok; ++n) {
                int bh, qb;
                if (!(ok = read_item(n, bh, qb)) || bh < 0) break;
                const int W = mask.head_window(bh);
                int lo[2], hi[2];
                fwd_tile_range(p, mask, bh, W, 2 * qb, lo[0], hi[0]);
                fwd_tile_range(p, mask, bh, W, 2 * qb + 1, lo[1], hi[1]);
                const int qbuf = n_item % kQBufs;
                if (!(ok = mbar_wait(&sm.bar_q[qbuf], (n_item / kQBufs) & 1, ac))) break;
                const uint32_t q_addr0 = smem_u32(sm.q[qbuf][0]), q_addr1 = smem_u32(sm.q[qbuf][1]);
                for (int j = lo[0]; ok && j <= hi[1]; ++j, ++it) {
                    const int s = it % kStages;
                    if (!(ok = mbar_wait(&sm.bar_k[s], (it / kStages) & 1, ac))) break;
                    const uint32_t k_addr = smem_u32(sm.k[s]);
                    for (int t = 0; ok && t < 2; ++t) {
                        if (j < lo[t] || j > hi[t]) continue;
                        if (ct[t] > 0) {
                            // S_t shares TMEM with what the previous tile still needs: the softmax
                            // copy of S (separate P) or, when P is written over S, the PV MMA that reads it.
                            uint64_t* freed = C::kSeparateP ? &sm.bar_s_free[t] : &sm.bar_o_done[t];
                            if (!(ok = mbar_wait(freed, (ct[t] - 1) & 1, ac))) break;
                        }
                        tc_fence_after();
                        const uint32_t q_addr = t ? q_addr1 : q_addr0;
                        const uint32_t col = t ? C::kColS1 : C::kColS0;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            mma_ss(tmem + col, sw128_desc(q_addr + off, 16, 1024), sw128_desc(k_addr + off, 16, 1024),
                                   kIdescQK, kk > 0);
                        }
                        mma_commit(&sm.bar_s_full[t]);
                        ++ct[t];
                    }
                    if (ok) {
                        mma_commit(&sm.bar_kv_empty[s]);
                        // A PV warp with nothing to do on this tile leaves its release of stage s
                        // to this warp: made here, after the stage's load was waited for, it can
                        // only count towards this tile's phase.
                        for (int t = 0; t < 2; ++t)
                            if (j < lo[t] || j > hi[t]) mma_commit(&sm.bar_kv_empty[s]);
                    }
                }
                if (ok) mma_commit(&sm.bar_q_empty[qbuf]);    // the item's Q buffer may be reloaded
                ++n_item;
            }
        } else if (warp == 2 || warp == 3) {
            const int t = warp - 2;
            const uint32_t col_o = t ? C::kColO1 : C::kColO0;
            const uint32_t col_p = t ? C::kColP1 : C::kColP0;
            int ct = 0;              // PV tiles issued, over all items
            for (int n = 0; ok; ++n) {
                int bh, qb;
                if (!(ok = read_item(n, bh, qb)) || bh < 0) break;
                const int W = mask.head_window(bh);
                int lo0, hi0, lo1, hi1;
                fwd_tile_range(p, mask, bh, W, 2 * qb, lo0, hi0);
                fwd_tile_range(p, mask, bh, W, 2 * qb + 1, lo1, hi1);
                const int lo = t ? lo1 : lo0, hi = t ? hi1 : hi0;
                for (int j = lo0; ok && j <= hi1; ++j, ++it) {
                    const int s = it % kStages;
                    if (j < lo || j > hi) continue;      // the S warp releases stage s for this warp
                    const int i = j - lo;
                    if (!(ok = mbar_wait(&sm.bar_v[s], (it / kStages) & 1, ac))) break;
                    if (!(ok = mbar_wait(&sm.bar_p_full[t], ct & 1, ac))) break;
                    // The item's first PV overwrites O: the previous item's epilogue must have read it.
                    if (i == 0 && n_item > 0 && !(ok = mbar_wait(&sm.bar_o_free[t], (n_item - 1) & 1, ac))) break;
                    tc_fence_after();
                    const uint32_t v_addr = smem_u32(sm.v[s]);
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        mma_ts(tmem + col_o, tmem + col_p + kk * 8, sw128_desc(v_addr + kk * 2048, 16384, 1024),
                               kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&sm.bar_o_done[t]);
                    mma_commit(&sm.bar_kv_empty[s]);
                    ++ct;
                }
                ++n_item;
            }
        }
        if (warp <= 3) {
            // No MMA of this warp may still be running when TMEM is released.
            mma_commit(&sm.bar_drain);
            mbar_wait_drain(&sm.bar_drain, 0, p.timeout_ns);
        }
    }
    } else {
        regs_inc<224>();
        // ------------------------------------------------------------ softmax warpgroups
        const int t = (warp - 4) >> 2;               // Q tile of this warpgroup
        const int wq = warp & 3;                     // TMEM lane quarter this warp may access
        const int row = wq * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t col_s = t ? C::kColS1 : C::kColS0;
        const uint32_t col_p = t ? C::kColP1 : C::kColP0;
        const uint32_t col_o = t ? C::kColO1 : C::kColO0;
        const float sl2 = p.scale_log2;
        bool ok = true;
        int ct = 0;                  // tiles of this warpgroup, over all items
        int n_items = 0;
        const bool o_issuer = wq == 0 && lane == 0;   // issues this warpgroup's O tile stores
        for (int n = 0; ok; ++n) {
            const int slot = n & 1;
            if (!warp_wait(&sm.bar_item_full[slot], (n >> 1) & 1, ac)) { ok = false; break; }
            const int bh = *reinterpret_cast<volatile int*>(&sm.item_bh[slot]);
            const int qb = *reinterpret_cast<volatile int*>(&sm.item_qb[slot]);
            __syncwarp();                                // every lane has read the slot
            if (lane == 0) mbar_arrive(&sm.bar_item_empty[slot]);
            if (bh < 0) break;
            const int qt = 2 * qb + t;
            const int i_abs = qt * kTile + row;
            const int W = mask.head_window(bh);
            int lo, hi;
            fwd_tile_range(p, mask, bh, W, qt, lo, hi);
            // Visible keys of this row: [row_lo, i_abs].  A key tile needs the per-element mask if
            // it holds the diagonal or starts before the lower bound of the tile's last row (lower
            // bounds do not decrease down the tile).
            const int row_lo = mask.row_lower_of(bh, p.T, W, i_abs);
            const int last_lo = mask.row_lower_of(bh, p.T, W, qt * kTile + kTile - 1);
            float m_used = -INFINITY;    // reference max of the exponentials (log2 units)
            float l = 0.f;               // running sum of 2^(x - m_used)
            const int n_t = hi - lo + 1;
            for (int i = 0; i < n_t; ++i) {
                const int c = ct + i;    // phase index of this tile
                const int j = lo + i;
                const int k0 = j * kTile;
                if (!warp_wait(&sm.bar_s_full[t], c & 1, ac)) { ok = false; break; }
                tc_fence_after();
                float s[128];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(t_lane + col_s + cc * 32, r);
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[cc * 32 + e] = __uint_as_float(r[e]);
                }
                tmem_wait_ld();
                if (C::kSeparateP) {
                    tc_fence_before();
                    mbar_arrive(&sm.bar_s_free[t]);        // S columns may be overwritten now
                }
                const bool need_mask = (j == qt) || (k0 < last_lo);
                if (need_mask) {
                    // Visible columns of this row form one range [c_lo, c_hi]; one unsigned compare
                    // and a select per element, no per-element branch.
                    const int c_hi = i_abs - k0;
                    const int c_lo = row_lo - k0;
                    const uint32_t span = (uint32_t)(c_hi - c_lo);
#pragma unroll
                    for (int e = 0; e < 128; ++e)
                        s[e] = ((uint32_t)(e - c_lo) <= span) ? s[e] : -INFINITY;
                }
                // Exponentials.  After the first tile of a row the reference max m_used is finite and
                // the exponentials start at once with it, the tile's own max being computed in the
                // same pass.  Only if some row's max now exceeds m_used by more than the lazy-rescale
                // margin (rare) is the tile redone below with the new max; nothing has been stored or
                // accumulated at that point.
                uint32_t pk[64];
                float rs = 0.f;
                float mx;
                if (i == 0) {
                    // First tile of this item: its max becomes the reference (O is still empty).
                    float m0 = fmax3(s[0], s[1], s[2]), m1 = fmax3(s[3], s[4], s[5]);
                    float m2 = fmax3(s[6], s[7], s[8]), m3 = fmax3(s[9], s[10], s[11]);
#pragma unroll
                    for (int e = 12; e < 120; e += 8) {
                        m0 = fmax3(m0, s[e], s[e + 1]);
                        m1 = fmax3(m1, s[e + 2], s[e + 3]);
                        m2 = fmax3(m2, s[e + 4], s[e + 5]);
                        m3 = fmax3(m3, s[e + 6], s[e + 7]);
                    }
                    m0 = fmax3(m0, s[124], s[125]);
                    m1 = fmax3(m1, s[126], s[127]);
                    m2 = fmax3(m2, s[120], s[121]);
                    m3 = fmax3(m3, s[122], s[123]);
                    m_used = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * sl2;
                }
                {
                    const float m_spec = (m_used == -INFINITY) ? 0.f : m_used;
                    float m0 = -INFINITY, m1 = -INFINITY;
                    float r0 = 0.f, r1 = 0.f;
#pragma unroll
                    for (int e = 0; e < 128; e += 4) {
                        m0 = fmax3(m0, s[e], s[e + 1]);
                        m1 = fmax3(m1, s[e + 2], s[e + 3]);
                        const float a = ex2_approx(fmaf(s[e], sl2, -m_spec));
                        const float b = ex2_approx(fmaf(s[e + 1], sl2, -m_spec));
                        const float cx = ex2_approx(fmaf(s[e + 2], sl2, -m_spec));
                        const float d = ex2_approx(fmaf(s[e + 3], sl2, -m_spec));
                        r0 += a + b;
                        r1 += cx + d;
                        pk[e >> 1] = pack_bf16x2(a, b);
                        pk[(e >> 1) + 1] = pack_bf16x2(cx, d);
                    }
                    mx = fmaxf(m0, m1);
                    rs = r0 + r1;
                }
                const float m_new = mx * sl2;               // -inf stays -inf (sl2 > 0)
                const bool need = m_new > m_used + kLazyRescale;
                if (__any_sync(0xffffffffu, need)) {
                    const float alpha = need ? ex2_approx(m_used - m_new) : 1.f;
                    if (need) m_used = m_new;
                    l *= alpha;
                    if (i > 0) {
                        // O holds PV up to the previous tile: wait for it, then rescale in place.
                        if (!warp_wait(&sm.bar_o_done[t], (c - 1) & 1, ac)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int cc = 0; cc < D / 32; ++cc) {
                            uint32_t r[32];
                            tmem_ld32(t_lane + col_o + cc * 32, r);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                            tmem_st32(t_lane + col_o + cc * 32, r);
                        }
                    }
                    // Redo this tile's exponentials against the new reference (rows that kept their
                    // reference recompute the same values).
                    const float m_use = (m_used == -INFINITY) ? 0.f : m_used;
                    float r0 = 0.f, r1 = 0.f;
#pragma unroll
                    for (int e = 0; e < 128; e += 2) {
                        const float a = ex2_approx(fmaf(s[e], sl2, -m_use));
                        const float b = ex2_approx(fmaf(s[e + 1], sl2, -m_use));
                        r0 += a;
                        r1 += b;
                        pk[e >> 1] = pack_bf16x2(a, b);
                    }
                    rs = r0 + r1;
                }
                l += rs;
                // Separate P columns: the previous PV (possibly the previous item's last) must have
                // finished reading them.
                if (C::kSeparateP && c > 0) {
                    if (!warp_wait(&sm.bar_o_done[t], (c - 1) & 1, ac)) { ok = false; break; }
                    tc_fence_after();
                }
                tmem_st32(t_lane + col_p, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
                tmem_st32(t_lane + col_p + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.bar_p_full[t]);
            }
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ct += n_t;
            // ------------------------------------------------------ epilogue of this item
            if (!warp_wait(&sm.bar_o_done[t], (ct - 1) & 1, ac)) { ok = false; break; }
            tc_fence_after();
            const float inv_l = 1.f / l;
            const bool store = i_abs < p.T;
            if constexpr (C::kOStage) {
                // O is staged as a bf16 128B-swizzled tile and written with one TMA tile store (rows
                // past T are clipped), so every warp writes whole lines; the staging buffer is
                // reused once the previous item's store has read it.
                if (o_issuer) {
                    bulk_wait_group_read0();
                    mbar_arrive(&sm.bar_ostage_free[t]);
                }
                if (!warp_wait(&sm.bar_ostage_free[t], n_items & 1, ac)) { ok = false; break; }
                const uint32_t row_a = smem_u32(sm.ostage[t]) + row * 128;
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(t_lane + col_o + cc * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j4 = 0; j4 < 4; ++j4) {
                        uint32_t v4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            v4[e] = pack_bf16x2(__uint_as_float(r[8 * j4 + 2 * e]) * inv_l,
                                                __uint_as_float(r[8 * j4 + 2 * e + 1]) * inv_l);
                        const int chunk = cc * 4 + j4;           // 16-byte chunk of the 128-byte row
                        st_shared_v4(row_a + ((chunk ^ (row & 7)) << 4), v4[0], v4[1], v4[2], v4[3]);
                    }
                }
                tc_fence_before();
                mbar_arrive(&sm.bar_o_free[t]);           // O columns may be overwritten now
                fence_proxy_async_smem();
                mbar_arrive(&sm.bar_ostage_full[t]);
                if (o_issuer) {
                    if (!mbar_wait(&sm.bar_ostage_full[t], n_items & 1, ac)) {
                        ok = false;
                    } else if (qt * kTile < p.T) {               // a tile wholly past T stores nothing
                        tma_store_4d(&tm_o, sm.ostage[t], 0, qt * kTile, bh % p.H, bh / p.H);
                        bulk_commit_group();
                    }
                }
            } else {
                __nv_bfloat16* orow = p.o + p.o_str.row(bh, p.H, store ? i_abs : 0);
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(t_lane + col_o + cc * 32, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        pk[e >> 1] = pack_bf16x2(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
                    if (store) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
                    }
                }
                tc_fence_before();
                mbar_arrive(&sm.bar_o_free[t]);           // O columns may be overwritten now
            }
            ++n_items;
            if (store) p.lse[(size_t)bh * p.T + i_abs] = (m_used + log2f(l)) * 0.69314718055994531f;
        }
        if (C::kOStage && o_issuer) bulk_wait_group0();   // the last O store has landed
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
