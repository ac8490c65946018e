// Work decomposition of the attention kernels, as plain integer code: which key tiles a query
// tile sees, which query tiles a key tile reaches, and the order in which the work items of both
// passes go to the SMs.  nvcc compiles it into the kernels and the host launcher; the
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

// Work order of both passes.  Every pass splits into work items of one head each, n_cls of
// them per head (the forward: 256-query blocks; the backward: 128-key tiles), and the items go
// to the SMs in a fixed list order, each SM taking the next item when it is ready for one (the
// forward kernel through cluster launch control, the backward kernel from a counter; the
// forward kernel also has a static order, below).  The
// items of one head should run at the same time, so that what they share (K/V in the forward;
// Q, dO and the dQ accumulator in the backward) is read from HBM once and from L2 by the
// others while it is still there: the list is head-major, each head's items longest first
// (class 0: the last query block in the forward, the first key tile in the backward).  Taken
// that way, though, the list would end with the long items of the last heads while the other
// SMs run dry; so the last `tail` heads go class-major instead (all their class-0 items, then
// all their class-1 items, ...), and the list ends with short items.

// Heads of the class-major tail: enough for the tail to hold two items per SM.
GPT_ATTN_HD int tail_heads(int BH, int n_cls, int sms) {
    const int t = (2 * sms + n_cls - 1) / n_cls;
    return t < BH ? t : BH;
}

// Item i of the list (0 <= i < BH * n_cls) whose last `tail` heads go class-major.  Returns
// head and class.
GPT_ATTN_HD void list_item(int i, int BH, int n_cls, int tail, int& bh, int& cls) {
    const int head_major = (BH - tail) * n_cls;     // items before the tail
    if (i < head_major) {
        bh = i / n_cls;
        cls = i % n_cls;
    } else {
        const int l = i - head_major;
        cls = l / tail;
        bh = BH - tail + l % tail;
    }
}

// The forward kernel has a second, static order for work that comes in many full rounds: items
// go out in waves of whole heads, heads_per_wave * n_blocks blocks, one per SM, and from one wave
// to the next the block class each block gets rotates, so that over n_blocks waves every block
// runs every class once.  Measured on the GPT-2 shapes this beats taking items on demand when
// the waves make at least kStaticCycles full rotations; with fewer, the partial rotation leaves
// some SMs with much more work than others, and the list above is used instead.
constexpr int kStaticCycles = 4;

// Static forward grid for n_blocks blocks per head: heads_per_wave and n_waves, and whether the
// static order applies at all.
GPT_ATTN_HD bool fwd_static_grid(int sms, int n_blocks, int BH, int& heads_per_wave, int& n_waves) {
    int hpw = sms / n_blocks;
    if (hpw < 1) hpw = 1;
    if (hpw > BH) hpw = BH;
    heads_per_wave = hpw;
    n_waves = (BH + hpw - 1) / hpw;
    return hpw * n_blocks <= sms && n_waves >= kStaticCycles * n_blocks;
}

// Static item of block `cta` in wave k: head bh (or -1 when the wave has none for it) and block
// qb.  Slot s of a wave holds block class s / heads_per_wave (longest first) of head
// s % heads_per_wave; a block's slot moves on by heads_per_wave each wave, so each block keeps
// to the same head position and cycles through the classes, while the blocks of a head run at
// the same time.
GPT_ATTN_HD void fwd_static_item(int heads_per_wave, int n_blocks, int BH, int cta, int k, int& bh, int& qb) {
    const int G = heads_per_wave * n_blocks;
    const int slot = (cta + heads_per_wave * (k % n_blocks)) % G;   // hpw * k mod G cycles with k mod n_blocks
    bh = heads_per_wave * k + slot % heads_per_wave;
    qb = n_blocks - 1 - slot / heads_per_wave;
    if (bh >= BH) bh = -1;
}

// Forward item i: head bh and 256-query block qb (class 0 = the last block, the longest under
// a causal mask).
GPT_ATTN_HD void fwd_item(int i, int BH, int n_blocks, int tail, int& bh, int& qb) {
    int cls;
    list_item(i, BH, n_blocks, tail, bh, cls);
    qb = n_blocks - 1 - cls;
}

// Backward work unit u: head bh, key tile kt (class 0 = key tile 0, seen by the most query
// tiles), and the n_q query tiles [kt, kt + n_q) that see it under a window (no document mask).
GPT_ATTN_HD void bwd_unit(int u, int BH, int n_tiles, int tail, int window, int& bh, int& kt, int& n_q) {
    list_item(u, BH, n_tiles, tail, bh, kt);
    n_q = bwd_last_query_tile(kt, n_tiles, window) - kt + 1;
}

}  // namespace gpt_attn
