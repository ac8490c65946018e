// Work decomposition of the attention kernels, as plain integer code: which key tiles a query
// tile sees, which query tiles a key tile reaches, the forward kernel's persistent item order and
// the backward kernel's work units.  nvcc compiles it into the kernels and the host launcher; the
// CPU tests compile the same header with a host compiler and check it against brute force.
//
// Visibility follows the masked softmax of the causal attention definition: query i sees key j
// when j <= i and, with a sliding window W > 0, j > i - W.
#pragma once

#if defined(__CUDACC__)
#define GPT_ATTN_HD __host__ __device__ __forceinline__
#else
#define GPT_ATTN_HD inline
#endif

namespace gpt_attn {

constexpr int kTile = 128;           // rows per Q tile and per K/V tile

// Lower bound of the keys query i may see: key j is visible iff row_lower(i, ...) <= j <= i.
// window > 0 keeps the last `window` keys (diagonal included); doc_start_i is the first position
// of the document holding token i (0 when the row is one document).  Document starts are clamped
// to [0, i], so every query sees at least itself whatever the input holds.
GPT_ATTN_HD int row_lower(int i, int window, int doc_start_i) {
    int lo = window > 0 ? i - window + 1 : 0;
    int d = doc_start_i < 0 ? 0 : (doc_start_i > i ? i : doc_start_i);
    if (lo < d) lo = d;
    return lo < 0 ? 0 : lo;
}

// Key tiles [lo, hi] hold every key visible to some query of query tile qt, given the lower
// bound of the tile's first row (lower bounds do not decrease along a row of documents).
GPT_ATTN_HD void fwd_key_range_lb(int qt, int first_row_lower, int& lo, int& hi) {
    hi = qt;
    lo = first_row_lower / kTile;
    if (lo > hi) lo = hi;
}

// Key tiles [lo, hi] hold every key visible to some query of query tile qt.
GPT_ATTN_HD void fwd_key_range(int qt, int window, int& lo, int& hi) {
    hi = qt;
    lo = 0;
    if (window > 0) {
        const int first = qt * kTile - window + 1;
        lo = first > 0 ? first / kTile : 0;
    }
}

// Query tiles that see at least one key of key tile kt: [kt, bwd_last_query_tile(...)].
GPT_ATTN_HD int bwd_last_query_tile(int kt, int n_tiles, int window) {
    if (window <= 0) return n_tiles - 1;
    const long long last = (long long)kt * kTile + kTile - 1 + window - 1;   // last query seeing the tile
    const long long t = last / kTile;
    return t < n_tiles - 1 ? (int)t : n_tiles - 1;
}

// Last query tile that sees key tile kt when rows carry lower bounds (document masks):
// lower_of_tile(qt) is the lower bound of query tile qt's first row.  Lower bounds do not
// decrease along a row, so tile qt > kt sees the key tile iff its first row's bound is at or
// before the tile's last key, and those tiles form a prefix [kt, last].
template <typename LowerOfTile>
GPT_ATTN_HD int bwd_last_query_tile_lb(int kt, int n_tiles, LowerOfTile lower_of_tile) {
    const int kend = kt * kTile + kTile - 1;
    int qt = kt;
    while (qt + 1 < n_tiles && lower_of_tile(qt + 1) <= kend) ++qt;
    return qt;
}

// Forward grid.  A work item is one (head, 256-query block); n_blocks = ceil(n_tiles / 2) per
// head.  Persistent (D = 64): waves of whole heads, heads_per_wave * n_blocks CTAs, at most one
// per SM unless a single head has more blocks than the GPU has SMs.  D = 128: one item per CTA
// (a single wave of all heads).
GPT_ATTN_HD void fwd_grid(int sms, int n_blocks, int BH, bool persistent, int& heads_per_wave, int& n_waves) {
    int hpw = persistent ? sms / n_blocks : BH;
    if (hpw < 1) hpw = 1;
    if (hpw > BH) hpw = BH;
    heads_per_wave = hpw;
    n_waves = (BH + hpw - 1) / hpw;
}

// Work item of CTA `cta` in wave `k`: head bh (or -1 when the wave has no item for it) and
// 256-query block qb.  Slot s of a wave holds block class s / heads_per_wave (longest first)
// of head s % heads_per_wave; a CTA's slot moves on by heads_per_wave each wave, so each CTA
// gets an even mix of long and short blocks while the blocks of a head run at the same time.
GPT_ATTN_HD void fwd_item(int heads_per_wave, int n_blocks, int BH, int cta, int k, int& bh, int& qb) {
    const int G = heads_per_wave * n_blocks;
    const int slot = (int)(((long long)cta + (long long)heads_per_wave * k) % G);
    bh = heads_per_wave * k + slot % heads_per_wave;
    qb = n_blocks - 1 - slot / heads_per_wave;
    if (bh >= BH) bh = -1;
}

// Backward work unit u of the persistent kernel: head bh, key tile kt, and the n_q query tiles
// [kt, kt + n_q) that see it.  Units are numbered head-major.
GPT_ATTN_HD void bwd_unit(int u, int n_tiles, int window, int& bh, int& kt, int& n_q) {
    bh = u / n_tiles;
    kt = u % n_tiles;
    n_q = bwd_last_query_tile(kt, n_tiles, window) - kt + 1;
}

}  // namespace gpt_attn
