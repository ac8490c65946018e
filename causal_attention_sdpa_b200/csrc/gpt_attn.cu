// C ABI of the attention library: argument checks, TMA descriptor encoding
// and kernel launches on the caller's stream.  No allocation, no host sync
// (except in gpt_attn_check, which exists to sync).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "attn_bwd.cuh"
#include "attn_bwd_d64.cuh"
#include "attn_decode.cuh"
#include "attn_fwd.cuh"
#include "gpt_attn.h"
#include "qk_prologue.cuh"
#include "tmap_cache.h"

extern "C" size_t gpt_attn_bwd_workspace_bytes(int B, int H, int T, int D);

namespace gpt_attn {
namespace {

constexpr uint64_t kDefaultTimeoutNs = 1000ull * 1000ull * 1000ull;   // 1 s per wait

uint64_t wait_timeout_ns() {
    static uint64_t v = []() -> uint64_t {
        const char* s = getenv("GPT_ATTN_WAIT_TIMEOUT_MS");
        if (s && *s) {
            const long long ms = atoll(s);
            if (ms > 0) return (uint64_t)ms * 1000000ull;
        }
        return kDefaultTimeoutNs;
    }();
    return v;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Encodes the tensor map of `key` (see TmapKind): 128-row boxes whose width is 128 bytes of
// elements (64 bf16 or 32 fp32 columns), 128-byte swizzle (the UMMA canonical 128B-swizzled
// layout), zero fill outside the tensor so ragged tails read as zeros.  bf16 maps are 4-D
// (D, T, H, B) with the tensor's own token, head and batch strides, so any [b, h, t, d] view with
// contiguous d (e.g. the q, k, v columns of a fused [B, T, 3, H, D] projection) is read and
// written in place; the fp32 accumulator map is 3-D (D, T, B*H), contiguous.
bool encode_tmap(const TmapKey& key, CUtensorMap* m) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const bool f32 = key.kind == (int)TmapKind::kF32Box32x128;
    const cuuint64_t esz = f32 ? 4 : 2;
    const cuuint32_t rank = f32 ? 3 : 4;
    cuuint64_t dims[4] = {(cuuint64_t)key.d0, (cuuint64_t)key.d1, (cuuint64_t)key.d2, (cuuint64_t)key.d3};
    cuuint64_t strides[3] = {(cuuint64_t)key.s1 * esz, (cuuint64_t)key.s2 * esz, (cuuint64_t)key.s3 * esz};
    cuuint32_t box[4] = {f32 ? 32u : 64u, 128, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                    reinterpret_cast<void*>(key.base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

TmapCache<CUtensorMap>& tmap_cache() {
    static TmapCache<CUtensorMap> c;
    return c;
}

bool cached_tmap(CUtensorMap* m, const TmapKey& key) {
    return tmap_cache().get(key, m, [](const TmapKey& k, CUtensorMap* v) { return encode_tmap(k, v); });
}

// bf16 tensor indexed [b, h, t, d] with strides `st`; 64-column x 128-row boxes.
bool make_tmap_bf16(CUtensorMap* m, const void* base, int B, int H, int T, int D, const Strides& st) {
    const TmapKey key{reinterpret_cast<uintptr_t>(base), (int)TmapKind::kBf16Box64x128, D, T, H, B, st.t, st.h, st.b};
    return cached_tmap(m, key);
}

// fp32 dQ accumulator [BH, T, D]; 32-column x 128-row boxes for the bulk reduce-add.
bool make_tmap_f32_acc(CUtensorMap* m, const void* base, int BH, int T, int D) {
    const TmapKey key{reinterpret_cast<uintptr_t>(base), (int)TmapKind::kF32Box32x128, D, T, BH, 1,
                      (long long)D, (long long)T * D, (long long)BH * T * D};
    return cached_tmap(m, key);
}

// Strides of every tensor of one call.
struct Layout {
    Strides q, k, v, o, dO, dq, dk, dv;
};

Strides contiguous(int H, int T, int D) { return Strides{(long long)H * T * D, (long long)T * D, (long long)D}; }

Layout contiguous_layout(int H, int T, int D) {
    const Strides c = contiguous(H, T, D);
    return Layout{c, c, c, c, c, c, c, c};
}

// From the C ABI's description (nullptr: contiguous [B, H, T, D]).  TMA needs every stride to be
// a multiple of 16 bytes (8 elements).
int make_layout(Layout* L, const gpt_attn_layout* a, int H, int T, int D) {
    *L = contiguous_layout(H, T, D);
    if (!a) return GPT_ATTN_OK;
    const gpt_attn_strides* in[8] = {&a->q, &a->k, &a->v, &a->o, &a->dO, &a->dq, &a->dk, &a->dv};
    Strides* out[8] = {&L->q, &L->k, &L->v, &L->o, &L->dO, &L->dq, &L->dk, &L->dv};
    for (int i = 0; i < 8; ++i) {
        const gpt_attn_strides& x = *in[i];
        if (x.batch < 0 || x.head < 0 || x.token < 0) return GPT_ATTN_ERR_SHAPE;
        if ((x.batch | x.head | x.token) & 7) return GPT_ATTN_ERR_ALIGN;
        *out[i] = Strides{x.batch, x.head, x.token};
    }
    return GPT_ATTN_OK;
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

int check_shape(int B, int H, int T, int D) {
    if (B < 1 || H < 1 || T < 1) return GPT_ATTN_ERR_SHAPE;
    if (D != 64 && D != 128) return GPT_ATTN_ERR_UNSUPPORTED_D;
    // Every element index must fit in int64, and the TMA coordinates (T, B*H) in int32.
    const long long bh = (long long)B * H;
    if (bh > 0x7fffffffLL) return GPT_ATTN_ERR_SHAPE;
    const long long tp = ((long long)T + 127) / 128 * 128;
    if (tp > (0x7fffffffffffffffLL / D) / bh) return GPT_ATTN_ERR_SHAPE;
    if ((tp / 128) * bh > 0x7fffffffLL) return GPT_ATTN_ERR_SHAPE;   // grid size
    return GPT_ATTN_OK;
}

template <typename Kern>
bool set_smem(Kern k, size_t bytes) {
    // The attribute is a per-function setting: raise it once per kernel and device (and again only
    // for a larger size) instead of paying a driver call on every launch.
    struct Entry { const void* fn; int dev; size_t bytes; };
    static std::mutex mu;
    static std::vector<Entry> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const void* fn = reinterpret_cast<const void*>(k);
    std::lock_guard<std::mutex> g(mu);
    for (auto& e : done)
        if (e.fn == fn && e.dev == dev) {
            if (e.bytes >= bytes) return true;
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
                return false;
            e.bytes = bytes;
            return true;
        }
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) return false;
    done.push_back({fn, dev, bytes});
    return true;
}

int sm_count();

// Kernel-side mask parameters from the C ABI's description (nullptr: plain causal).  Per-head
// windows are copied out of the caller's host array into the kernel parameters.
int make_mask(MaskParams* m, const gpt_attn_mask* a, int H) {
    memset(m, 0, sizeof(*m));
    m->H = H;
    if (!a) return GPT_ATTN_OK;
    m->window = a->window > 0 ? a->window : 0;
    m->doc_start = a->doc_start;
    if (a->doc_start && (reinterpret_cast<uintptr_t>(a->doc_start) & 3u)) return GPT_ATTN_ERR_ALIGN;
    if (a->head_windows) {
        if (H > kMaxHeadWindows) return GPT_ATTN_ERR_SHAPE;
        m->head_windows = 1;
        for (int h = 0; h < H; ++h) m->win[h] = a->head_windows[h] > 0 ? a->head_windows[h] : 0;
    }
    return GPT_ATTN_OK;
}

// True when every head shares one window and there are no document starts.
bool plain_window(const MaskParams& m) { return !m.head_windows && !m.doc_start; }

MaskParams window_mask(int window, int H) {
    gpt_attn_mask a{window, nullptr, nullptr};
    MaskParams m;
    make_mask(&m, &a, H);
    return m;
}

template <int D>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int T, float scale,
               const MaskParams& mask, const Layout& L, cudaStream_t st) {
    const int BH = B * H;
    CUtensorMap mq, mk, mv, mo;
    if (!make_tmap_bf16(&mq, q, B, H, T, D, L.q) || !make_tmap_bf16(&mk, k, B, H, T, D, L.k) ||
        !make_tmap_bf16(&mv, v, B, H, T, D, L.v) || !make_tmap_bf16(&mo, o, B, H, T, D, L.o))
        return GPT_ATTN_ERR_CUDA;
    FwdParams p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.o_str = L.o;
    p.H = H;
    p.T = T;
    p.BH = BH;
    p.n_tiles = (T + kTile - 1) / kTile;
    p.n_blocks = (p.n_tiles + 1) / 2;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = wait_timeout_ns();
    // Work order (schedule.h): static waves with one block per SM when they make enough full
    // rotations (D = 64), else one block per item, the blocks that start taking the items of
    // those that have not through cluster launch control.
    const int sms = sm_count();
    p.tail = tail_heads(BH, p.n_blocks, sms);
    p.static_hpw = 0;
    p.static_waves = 0;
    int hpw, waves;
    const bool stat = D == 64 && fwd_static_grid(sms, p.n_blocks, BH, hpw, waves);
    if (stat) {
        p.static_hpw = hpw;
        p.static_waves = waves;
    }
    const size_t smem = sizeof(FwdSmem<D>) + 1024;
    const unsigned grid = stat ? (unsigned)(hpw * p.n_blocks) : (unsigned)((long long)BH * p.n_blocks);
    if (plain_window(mask)) {
        // Causal or one window for every head: the instantiation without per-head or document data.
        if (!set_smem(attn_fwd_kernel<D, WindowMask>, smem)) return GPT_ATTN_ERR_CUDA;
        attn_fwd_kernel<D, WindowMask><<<grid, kFwdThreads, smem, st>>>(mq, mk, mv, mo, p, WindowMask{mask.window});
    } else {
        if (!set_smem(attn_fwd_kernel<D, MaskParams>, smem)) return GPT_ATTN_ERR_CUDA;
        attn_fwd_kernel<D, MaskParams><<<grid, kFwdThreads, smem, st>>>(mq, mk, mv, mo, p, mask);
    }
    return cudaGetLastError() == cudaSuccess ? GPT_ATTN_OK : GPT_ATTN_ERR_CUDA;
}

struct WsLayout {
    float* dq_acc;
    float* lse2;
    float* delta;
    int* lower2;
    int* last_qt;
    int* sched;
    int n_tiles;
    int T_pad;
};

// Workspace: fp32 dQ accumulator [BH, T, D] | lse*log2(e) [BH, T_pad] | Delta [BH, T_pad] |
// row lower bounds [BH, T_pad] and last query tile per key tile [BH, n_tiles] (both used
// with document masks only) | the persistent kernel's work-unit counter.
WsLayout ws_layout(void* ws, int BH, int T, int D) {
    WsLayout w;
    w.n_tiles = (T + kTile - 1) / kTile;
    w.T_pad = w.n_tiles * kTile;
    w.dq_acc = static_cast<float*>(ws);
    w.lse2 = w.dq_acc + (size_t)BH * T * D;
    w.delta = w.lse2 + (size_t)BH * w.T_pad;
    w.lower2 = reinterpret_cast<int*>(w.delta + (size_t)BH * w.T_pad);
    w.last_qt = w.lower2 + (size_t)BH * w.T_pad;
    w.sched = w.last_qt + (size_t)BH * w.n_tiles;
    return w;
}

// SM count of the current device, cached per device.  Host threads may call the library at the
// same time: the cache entries are atomics (every thread would store the same value).
int sm_count() {
    static std::atomic<int> counts[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = counts[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

int launch_bwd_delta(const void* o, const float* lse, const void* dout, int B, int H, int T, int D, void* ws,
                     const MaskParams& mask, const Layout& L, cudaStream_t st) {
    const int BH = B * H;
    const WsLayout w = ws_layout(ws, BH, T, D);
    const long long rows = (long long)BH * w.T_pad;
    const int rows_per_block = 256 / (D / 8);
    const unsigned grid = (unsigned)((rows + rows_per_block - 1) / rows_per_block);
    const auto* o16 = static_cast<const __nv_bfloat16*>(o);
    const auto* do16 = static_cast<const __nv_bfloat16*>(dout);
    const bool doc = mask.doc_start != nullptr;
    if (D == 64)
        attn_bwd_prep_kernel<64><<<grid, 256, 0, st>>>(o16, do16, lse, w.lse2, w.delta, w.dq_acc, w.sched, T,
                                                        w.T_pad, rows, mask, doc ? w.lower2 : nullptr,
                                                        w.last_qt, w.n_tiles, L.o, L.dO, H);
    else
        attn_bwd_prep_kernel<128><<<grid, 256, 0, st>>>(o16, do16, lse, w.lse2, w.delta, w.dq_acc, w.sched, T,
                                                         w.T_pad, rows, mask, doc ? w.lower2 : nullptr,
                                                         w.last_qt, w.n_tiles, L.o, L.dO, H);
    return cudaGetLastError() == cudaSuccess ? GPT_ATTN_OK : GPT_ATTN_ERR_CUDA;
}

template <int D>
int launch_bwd_grads(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B,
                     int H, int T, float scale, const MaskParams& mask, const Layout& L, void* ws, cudaStream_t st) {
    const int BH = B * H;
    const WsLayout w = ws_layout(ws, BH, T, D);
    CUtensorMap mq, mk, mv, mdo;
    if (!make_tmap_bf16(&mq, q, B, H, T, D, L.q) || !make_tmap_bf16(&mk, k, B, H, T, D, L.k) ||
        !make_tmap_bf16(&mv, v, B, H, T, D, L.v) || !make_tmap_bf16(&mdo, dout, B, H, T, D, L.dO))
        return GPT_ATTN_ERR_CUDA;
    BwdParams p;
    p.lse2 = w.lse2;
    p.delta = w.delta;
    p.dq_acc = w.dq_acc;
    p.sched = w.sched;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.dk_str = L.dk;
    p.dv_str = L.dv;
    p.H = H;
    p.T = T;
    p.T_pad = w.T_pad;
    p.BH = BH;
    p.n_tiles = w.n_tiles;
    p.tail = tail_heads(BH, p.n_tiles, sm_count());
    p.lower2 = mask.doc_start ? w.lower2 : nullptr;
    p.last_qt = mask.doc_start ? w.last_qt : nullptr;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.scale = scale;
    p.timeout_ns = wait_timeout_ns();
    const long long units = (long long)w.n_tiles * BH;
    const unsigned grid = (unsigned)units;
    if constexpr (D == 64) {
        CUtensorMap mdq, mdk, mdv;
        if (!make_tmap_f32_acc(&mdq, w.dq_acc, BH, T, D) || !make_tmap_bf16(&mdk, dk, B, H, T, D, L.dk) ||
            !make_tmap_bf16(&mdv, dv, B, H, T, D, L.dv))
            return GPT_ATTN_ERR_CUDA;
        const size_t smem = sizeof(Bwd64Smem) + 1024;
        // persistent: one CTA per SM, work units taken from the counter in the workspace
        const unsigned pgrid = (unsigned)(units < sm_count() ? units : sm_count());
        if (plain_window(mask)) {
            if (!set_smem(attn_bwd_kernel<WindowMask>, smem)) return GPT_ATTN_ERR_CUDA;
            attn_bwd_kernel<WindowMask><<<pgrid, kBwd64Threads, smem, st>>>(mq, mk, mv, mdo, mdq, mdk, mdv, p,
                                                                          WindowMask{mask.window});
        } else {
            if (!set_smem(attn_bwd_kernel<MaskParams>, smem)) return GPT_ATTN_ERR_CUDA;
            attn_bwd_kernel<MaskParams><<<pgrid, kBwd64Threads, smem, st>>>(mq, mk, mv, mdo, mdq, mdk, mdv, p, mask);
        }
    } else {
        CUtensorMap mdq;
        if (!make_tmap_f32_acc(&mdq, w.dq_acc, BH, T, D)) return GPT_ATTN_ERR_CUDA;
        const size_t smem = sizeof(BwdSmem<D>) + 1024;
        if (plain_window(mask)) {
            if (!set_smem(attn_bwd_serial_kernel<D, WindowMask>, smem)) return GPT_ATTN_ERR_CUDA;
            attn_bwd_serial_kernel<D, WindowMask><<<grid, kBwdThreads, smem, st>>>(mq, mk, mv, mdo, mdq, p,
                                                                                 WindowMask{mask.window});
        } else {
            if (!set_smem(attn_bwd_serial_kernel<D, MaskParams>, smem)) return GPT_ATTN_ERR_CUDA;
            attn_bwd_serial_kernel<D, MaskParams><<<grid, kBwdThreads, smem, st>>>(mq, mk, mv, mdo, mdq, p, mask);
        }
    }
    return cudaGetLastError() == cudaSuccess ? GPT_ATTN_OK : GPT_ATTN_ERR_CUDA;
}

int launch_dq_convert(void* dq, int B, int H, int T, int D, float scale, void* ws, const Layout& L, cudaStream_t st) {
    const int BH = B * H;
    const WsLayout w = ws_layout(ws, BH, T, D);
    const long long rows = (long long)BH * T;
    const int rows_per_block = 256 / (D / 8);
    const unsigned grid = (unsigned)((rows + rows_per_block - 1) / rows_per_block);
    auto* dq16 = static_cast<__nv_bfloat16*>(dq);
    if (D == 64)
        attn_dq_convert_kernel<64><<<grid, 256, 0, st>>>(w.dq_acc, dq16, rows, scale, T, H, L.dq);
    else
        attn_dq_convert_kernel<128><<<grid, 256, 0, st>>>(w.dq_acc, dq16, rows, scale, T, H, L.dq);
    return cudaGetLastError() == cudaSuccess ? GPT_ATTN_OK : GPT_ATTN_ERR_CUDA;
}

int check_ws(int B, int H, int T, int D, const void* ws, size_t ws_bytes) {
    if (!ws || ws_bytes < gpt_attn_bwd_workspace_bytes(B, H, T, D)) return GPT_ATTN_ERR_WORKSPACE;
    return misaligned(ws) ? GPT_ATTN_ERR_ALIGN : GPT_ATTN_OK;
}

// Decode split: as many splits per head as fit all CTAs on a B200 (148 SMs, kDecodeBlocksPerSm
// resident each) in one wave, at least one, at least 64 keys per split, at most kDecodeMaxChunk.
// A CTA's passes over its keys and values are chains of dependent load rounds, so shorter chunks
// over more CTAs keep more of HBM busy, and a second wave would add a whole chain.  The same
// function sizes the workspace and the launch.
int decode_splits(int BH, int T_max, int window, int* chunk) {
    const int span = (window > 0 && window < T_max) ? window : T_max;   // keys one query can see
    int n = kDecodeBlocksPerSm * 148 / BH;
    const int by_len = (span + 63) / 64;
    if (n > by_len) n = by_len;
    if (n < 1) n = 1;
    if ((span + n - 1) / n > kDecodeMaxChunk) n = (span + kDecodeMaxChunk - 1) / kDecodeMaxChunk;
    *chunk = (span + n - 1) / n;
    return n;
}

int check_decode_shape(int B, int H, int T_max, int D) {
    if (B < 1 || H < 1 || T_max < 1) return GPT_ATTN_ERR_SHAPE;
    if (D != 64 && D != 128) return GPT_ATTN_ERR_UNSUPPORTED_D;
    const long long bh = (long long)B * H;
    if (bh > 0x7fffffffLL) return GPT_ATTN_ERR_SHAPE;                    // grid x
    if ((long long)T_max / 64 + 1 > 65535) return GPT_ATTN_ERR_SHAPE;     // splits on grid y
    if ((long long)T_max > (0x7fffffffffffffffLL / D) / bh) return GPT_ATTN_ERR_SHAPE;
    return GPT_ATTN_OK;
}

template <int D>
int launch_decode(const void* q, const void* k, const void* v, const int* lens, void* o, float* lse, int B, int H,
                  int T_max, float scale, int window, void* ws, cudaStream_t st) {
    DecodeParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.lens = lens;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.H = H;
    p.T_max = T_max;
    p.window = window > 0 ? window : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    const int BH = B * H;
    p.n_split = decode_splits(BH, T_max, p.window, &p.chunk);
    p.part_o = static_cast<float*>(ws);
    p.part_ml = p.part_o + (size_t)BH * p.n_split * D;
    constexpr int R = kDecodeThreads / (D / 8);
    const size_t smem = (size_t)(p.chunk > R * D ? p.chunk : R * D) * sizeof(float);
    if (!set_smem(attn_decode_split_kernel<D>, smem)) return GPT_ATTN_ERR_CUDA;
    const dim3 grid(BH, p.n_split);
    attn_decode_split_kernel<D><<<grid, kDecodeThreads, smem, st>>>(p);
    if (p.n_split > 1) attn_decode_combine_kernel<D><<<BH, D, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? GPT_ATTN_OK : GPT_ATTN_ERR_CUDA;
}

// Strides of n tensors from the C ABI (nullptr: contiguous [B, H, T, D]); same rules as layouts.
int prologue_strides(Strides* out, const gpt_attn_strides* in, int n, int H, int T, int D) {
    for (int i = 0; i < n; ++i) {
        out[i] = contiguous(H, T, D);
        if (!in) continue;
        const gpt_attn_strides& x = in[i];
        if (x.batch < 0 || x.head < 0 || x.token < 0) return GPT_ATTN_ERR_SHAPE;
        if ((x.batch | x.head | x.token) & 7) return GPT_ATTN_ERR_ALIGN;
        out[i] = Strides{x.batch, x.head, x.token};
    }
    return GPT_ATTN_OK;
}

int launch_prologue(bool backward, const PrologueParams& p, int D, cudaStream_t st) {
    // persistent: 2 blocks per SM for each of q and k, all resident at once (4 x 256 threads of
    // at most 64 registers); a lane group takes a row, or a whole token for token-major inputs
    const long long per_block = kPrologueThreads / (D / 16);
    const long long units = p.token_major ? p.rows / p.H : p.rows;
    const long long need = (units + per_block - 1) / per_block;
    const dim3 grid((unsigned)std::min<long long>(need, 2LL * sm_count()), 2);
    if (p.token_major) {
        if (backward) {
            if (D == 64) qk_prologue_bwd_tok_kernel<64><<<grid, 256, 0, st>>>(p);
            else qk_prologue_bwd_tok_kernel<128><<<grid, 256, 0, st>>>(p);
        } else {
            if (D == 64) qk_prologue_fwd_tok_kernel<64><<<grid, 256, 0, st>>>(p);
            else qk_prologue_fwd_tok_kernel<128><<<grid, 256, 0, st>>>(p);
        }
        return cudaGetLastError() == cudaSuccess ? GPT_ATTN_OK : GPT_ATTN_ERR_CUDA;
    }
    if (backward) {
        if (D == 64) qk_prologue_bwd_kernel<64><<<grid, 256, 0, st>>>(p);
        else qk_prologue_bwd_kernel<128><<<grid, 256, 0, st>>>(p);
    } else {
        if (D == 64) qk_prologue_fwd_kernel<64><<<grid, 256, 0, st>>>(p);
        else qk_prologue_fwd_kernel<128><<<grid, 256, 0, st>>>(p);
    }
    return cudaGetLastError() == cudaSuccess ? GPT_ATTN_OK : GPT_ATTN_ERR_CUDA;
}

__global__ void debug_wait_kernel(uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);   // nothing ever arrives
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const AbortCtl ac{&abort_flag, timeout_ns};
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, ac);
    __syncthreads();
}

}  // namespace

// ---------------------------------------------------------------------------
// Built-in scratch for gpt_attn_bwd_noalloc.  A file-scope device array is
// created when the library's module is loaded on a device and lives until the
// process exits, so the entry point below never allocates.  In host code the
// name g_noalloc_scratch is only a host-side shadow symbol, not a device
// address: the device address is looked up with cudaGetSymbolAddress with the
// caller's device current.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of the scratch array on the current device, or nullptr on a
// CUDA error.  Looked up on every call (a table lookup once the module is
// loaded) rather than cached: after a cudaDeviceReset the module is loaded
// again and the array may live at a different address.
void* noalloc_scratch_current_device() {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    return ptr;
}
}  // namespace
}  // namespace gpt_attn

using namespace gpt_attn;

extern "C" {

int gpt_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int T, int D,
                    float scale, const gpt_attn_mask* mask, const gpt_attn_layout* layout, void* stream) {
    if (!q || !k || !v || !o || !lse) return GPT_ATTN_ERR_NULL;
    int sc = check_shape(B, H, T, D);
    if (sc != GPT_ATTN_OK) return sc;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(o) || misaligned(lse)) return GPT_ATTN_ERR_ALIGN;
    MaskParams m;
    if ((sc = make_mask(&m, mask, H)) != GPT_ATTN_OK) return sc;
    Layout L;
    if ((sc = make_layout(&L, layout, H, T, D)) != GPT_ATTN_OK) return sc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return D == 64 ? launch_fwd<64>(q, k, v, o, lse, B, H, T, scale, m, L, st)
                   : launch_fwd<128>(q, k, v, o, lse, B, H, T, scale, m, L, st);
}

int gpt_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int T, int D,
                 float scale, int window, void* stream) {
    const gpt_attn_mask m{window, nullptr, nullptr};
    return gpt_attn_fwd_ex(q, k, v, o, lse, B, H, T, D, scale, &m, nullptr, stream);
}

size_t gpt_attn_bwd_workspace_bytes(int B, int H, int T, int D) {
    if (check_shape(B, H, T, D) != GPT_ATTN_OK) return 0;
    const size_t bh = (size_t)B * H;
    const size_t t_pad = ((size_t)T + 127) / 128 * 128;
    return 4 * (bh * T * D + 3 * bh * t_pad + bh * (t_pad / 128)) + 16;
}

int gpt_attn_bwd_delta(const void* o, const float* lse, const void* dO, int B, int H, int T, int D,
                       void* workspace, size_t workspace_bytes, void* stream) {
    if (!o || !lse || !dO) return GPT_ATTN_ERR_NULL;
    int sc = check_shape(B, H, T, D);
    if (sc != GPT_ATTN_OK) return sc;
    if ((sc = check_ws(B, H, T, D, workspace, workspace_bytes)) != GPT_ATTN_OK) return sc;
    if (misaligned(o) || misaligned(lse) || misaligned(dO)) return GPT_ATTN_ERR_ALIGN;
    return launch_bwd_delta(o, lse, dO, B, H, T, D, workspace, window_mask(0, H), contiguous_layout(H, T, D),
                            static_cast<cudaStream_t>(stream));
}

int gpt_attn_bwd_grads(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, int B,
                       int H, int T, int D, float scale, int window, void* workspace, size_t workspace_bytes,
                       void* stream) {
    if (!q || !k || !v || !dO || !dk || !dv) return GPT_ATTN_ERR_NULL;
    int sc = check_shape(B, H, T, D);
    if (sc != GPT_ATTN_OK) return sc;
    if ((sc = check_ws(B, H, T, D, workspace, workspace_bytes)) != GPT_ATTN_OK) return sc;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(dO) || misaligned(dk) || misaligned(dv))
        return GPT_ATTN_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const MaskParams m = window_mask(window, H);
    const Layout L = contiguous_layout(H, T, D);
    return D == 64 ? launch_bwd_grads<64>(q, k, v, dO, dk, dv, B, H, T, scale, m, L, workspace, st)
                   : launch_bwd_grads<128>(q, k, v, dO, dk, dv, B, H, T, scale, m, L, workspace, st);
}

int gpt_attn_bwd_dq_convert(void* dq, int B, int H, int T, int D, float scale, void* workspace,
                            size_t workspace_bytes, void* stream) {
    if (!dq) return GPT_ATTN_ERR_NULL;
    int sc = check_shape(B, H, T, D);
    if (sc != GPT_ATTN_OK) return sc;
    if ((sc = check_ws(B, H, T, D, workspace, workspace_bytes)) != GPT_ATTN_OK) return sc;
    if (misaligned(dq)) return GPT_ATTN_ERR_ALIGN;
    return launch_dq_convert(dq, B, H, T, D, scale, workspace, contiguous_layout(H, T, D),
                             static_cast<cudaStream_t>(stream));
}

int gpt_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                    void* dq, void* dk, void* dv, int B, int H, int T, int D, float scale, const gpt_attn_mask* mask,
                    const gpt_attn_layout* layout, void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return GPT_ATTN_ERR_NULL;
    int sc = check_shape(B, H, T, D);
    if (sc != GPT_ATTN_OK) return sc;
    if ((sc = check_ws(B, H, T, D, workspace, workspace_bytes)) != GPT_ATTN_OK) return sc;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(o) || misaligned(lse) || misaligned(dO) ||
        misaligned(dq) || misaligned(dk) || misaligned(dv))
        return GPT_ATTN_ERR_ALIGN;
    MaskParams m;
    if ((sc = make_mask(&m, mask, H)) != GPT_ATTN_OK) return sc;
    Layout L;
    if ((sc = make_layout(&L, layout, H, T, D)) != GPT_ATTN_OK) return sc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((sc = launch_bwd_delta(o, lse, dO, B, H, T, D, workspace, m, L, st)) != GPT_ATTN_OK) return sc;
    sc = D == 64 ? launch_bwd_grads<64>(q, k, v, dO, dk, dv, B, H, T, scale, m, L, workspace, st)
                 : launch_bwd_grads<128>(q, k, v, dO, dk, dv, B, H, T, scale, m, L, workspace, st);
    if (sc != GPT_ATTN_OK) return sc;
    return launch_dq_convert(dq, B, H, T, D, scale, workspace, L, st);
}

int gpt_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                 void* dq, void* dk, void* dv, int B, int H, int T, int D, float scale, int window, void* workspace,
                 size_t workspace_bytes, void* stream) {
    const gpt_attn_mask m{window, nullptr, nullptr};
    return gpt_attn_bwd_ex(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale, &m, nullptr, workspace,
                           workspace_bytes, stream);
}

size_t gpt_attn_decode_workspace_bytes(int B, int H, int T_max, int D, int window) {
    if (check_decode_shape(B, H, T_max, D) != GPT_ATTN_OK) return 0;
    int chunk = 0;
    const int n = decode_splits(B * H, T_max, window > 0 ? window : 0, &chunk);
    return n > 1 ? (size_t)B * H * n * (D + 2) * sizeof(float) : 16;
}

int gpt_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int* seq_lens, void* o,
                    float* lse, int B, int H, int T_max, int D, float scale, int window, void* workspace,
                    size_t workspace_bytes, void* stream) {
    if (!q || !k_cache || !v_cache || !seq_lens || !o || !lse) return GPT_ATTN_ERR_NULL;
    const int sc = check_decode_shape(B, H, T_max, D);
    if (sc != GPT_ATTN_OK) return sc;
    const size_t need = gpt_attn_decode_workspace_bytes(B, H, T_max, D, window);
    if (!workspace || workspace_bytes < need) return GPT_ATTN_ERR_WORKSPACE;
    if (misaligned(q) || misaligned(k_cache) || misaligned(v_cache) || misaligned(o) || misaligned(workspace) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return GPT_ATTN_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return D == 64 ? launch_decode<64>(q, k_cache, v_cache, seq_lens, o, lse, B, H, T_max, scale, window, workspace, st)
                   : launch_decode<128>(q, k_cache, v_cache, seq_lens, o, lse, B, H, T_max, scale, window, workspace,
                                        st);
}

int gpt_attn_qk_prologue_fwd(const void* q_raw, const void* k_raw, void* q_out, void* k_out, int B, int H, int T,
                             int D, int qk_norm, float rope_base, const gpt_attn_strides* strides, void* stream) {
    if (!q_raw || !k_raw || !q_out || !k_out) return GPT_ATTN_ERR_NULL;
    int sc = check_shape(B, H, T, D);
    if (sc != GPT_ATTN_OK) return sc;
    if (misaligned(q_raw) || misaligned(k_raw) || misaligned(q_out) || misaligned(k_out)) return GPT_ATTN_ERR_ALIGN;
    Strides st[4];
    if ((sc = prologue_strides(st, strides, 4, H, T, D)) != GPT_ATTN_OK) return sc;
    PrologueParams p{};
    p.x[0] = static_cast<const __nv_bfloat16*>(q_raw);
    p.x[1] = static_cast<const __nv_bfloat16*>(k_raw);
    p.out[0] = static_cast<__nv_bfloat16*>(q_out);
    p.out[1] = static_cast<__nv_bfloat16*>(k_out);
    p.xs[0] = st[0], p.xs[1] = st[1], p.outs[0] = st[2], p.outs[1] = st[3];
    p.H = H;
    p.T = T;
    p.rows = (long long)B * H * T;
    p.token_major = st[0].h < st[0].t ? 1 : 0;    // heads of a token adjacent: walk rows token by token
    p.norm = qk_norm ? 1 : 0;
    p.base = rope_base;
    return launch_prologue(false, p, D, static_cast<cudaStream_t>(stream));
}

int gpt_attn_qk_prologue_bwd(const void* q_raw, const void* k_raw, const void* dq_out, const void* dk_out,
                             void* dq_raw, void* dk_raw, int B, int H, int T, int D, int qk_norm, float rope_base,
                             const gpt_attn_strides* strides, void* stream) {
    if (!q_raw || !k_raw || !dq_out || !dk_out || !dq_raw || !dk_raw) return GPT_ATTN_ERR_NULL;
    int sc = check_shape(B, H, T, D);
    if (sc != GPT_ATTN_OK) return sc;
    if (misaligned(q_raw) || misaligned(k_raw) || misaligned(dq_out) || misaligned(dk_out) || misaligned(dq_raw) ||
        misaligned(dk_raw))
        return GPT_ATTN_ERR_ALIGN;
    Strides st[6];
    if ((sc = prologue_strides(st, strides, 6, H, T, D)) != GPT_ATTN_OK) return sc;
    PrologueParams p{};
    p.x[0] = static_cast<const __nv_bfloat16*>(q_raw);
    p.x[1] = static_cast<const __nv_bfloat16*>(k_raw);
    p.dy[0] = static_cast<const __nv_bfloat16*>(dq_out);
    p.dy[1] = static_cast<const __nv_bfloat16*>(dk_out);
    p.out[0] = static_cast<__nv_bfloat16*>(dq_raw);
    p.out[1] = static_cast<__nv_bfloat16*>(dk_raw);
    p.xs[0] = st[0], p.xs[1] = st[1], p.dys[0] = st[2], p.dys[1] = st[3], p.outs[0] = st[4], p.outs[1] = st[5];
    p.H = H;
    p.T = T;
    p.rows = (long long)B * H * T;
    p.token_major = st[0].h < st[0].t ? 1 : 0;    // heads of a token adjacent: walk rows token by token
    p.norm = qk_norm ? 1 : 0;
    p.base = rope_base;
    return launch_prologue(true, p, D, static_cast<cudaStream_t>(stream));
}

int gpt_attn_check(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GPT_ATTN_ERR_CUDA;
    int st = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&st, gpt_attn::g_status, sizeof(int)) != cudaSuccess) return GPT_ATTN_ERR_CUDA;
    if (cudaMemcpyToSymbol(gpt_attn::g_status, &zero, sizeof(int)) != cudaSuccess) return GPT_ATTN_ERR_CUDA;
    if (cudaPeekAtLastError() != cudaSuccess) return GPT_ATTN_ERR_CUDA;
    return st;
}

const char* gpt_attn_status_string(int status) {
    switch (status) {
        case GPT_ATTN_OK: return "ok";
        case GPT_ATTN_ERR_NULL: return "null pointer argument";
        case GPT_ATTN_ERR_SHAPE: return "invalid shape (B, H, T must be >= 1; sizes must fit int64)";
        case GPT_ATTN_ERR_UNSUPPORTED_D: return "unsupported head dimension (D must be 64 or 128)";
        case GPT_ATTN_ERR_ALIGN: return "pointer not 16-byte aligned";
        case GPT_ATTN_ERR_CUDA: return "CUDA error";
        case GPT_ATTN_ERR_TIMEOUT: return "device-side wait timed out";
        case GPT_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case GPT_ATTN_ERR_UNAVAILABLE: return "not available in this build";
        case GPT_ATTN_ERR_BOUNDS: return "debug build: a kernel bounds check failed";
        default: return "unknown status";
    }
}

int gpt_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, int B, int H, int T, int D, float scale,
                         int window, void* stream) {
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return GPT_ATTN_ERR_NULL;
    const int sc = check_shape(B, H, T, D);
    if (sc != GPT_ATTN_OK) return sc;
    const size_t need = gpt_attn_bwd_workspace_bytes(B, H, T, D);
    if (need > kNoAllocScratchBytes) return GPT_ATTN_ERR_WORKSPACE;
    void* ws = noalloc_scratch_current_device();
    if (!ws) return GPT_ATTN_ERR_CUDA;
    // The scratch keeps whatever the previous call left; the gpt_attn_bwd stages
    // rewrite every byte they read (dQ accumulator zeroed, row vectors written
    // including padding), so nothing else needs clearing here.
    return gpt_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, D, scale, window, ws, need, stream);
}

void gpt_attn_tmap_cache_stats(long long* hits, long long* misses, int* entries) {
    long long h = 0, m = 0;
    int u = 0;
    gpt_attn::tmap_cache().stats(&h, &m, &u);
    if (hits) *hits = h;
    if (misses) *misses = m;
    if (entries) *entries = u;
}

int gpt_attn_debug_skip_load(int which) {
#ifdef GPT_ATTN_DEBUG
    if (which < 0 || which > 2) return GPT_ATTN_ERR_SHAPE;
    return cudaMemcpyToSymbol(gpt_attn::g_debug_skip, &which, sizeof(int)) == cudaSuccess ? GPT_ATTN_OK
                                                                                         : GPT_ATTN_ERR_CUDA;
#else
    (void)which;
    return GPT_ATTN_ERR_UNAVAILABLE;
#endif
}

int gpt_attn_debug_wait_timeout(int timeout_us, void* stream) {
    if (timeout_us < 1 || timeout_us > 10 * 1000 * 1000) return GPT_ATTN_ERR_SHAPE;
    gpt_attn::debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)timeout_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? GPT_ATTN_OK : GPT_ATTN_ERR_CUDA;
}

}  // extern "C"
