// Host build of the kernels' work decomposition (causal_attention_sdpa_b200/csrc/schedule.h) for
// the CPU tests: C entry points over the same inline functions the kernels and launcher use.
#include "schedule.h"

extern "C" {
void sch_fwd_key_range(int qt, int window, int* lo, int* hi) { gpt_attn::fwd_key_range(qt, window, *lo, *hi); }
int sch_bwd_last_query_tile(int kt, int n_tiles, int window) {
    return gpt_attn::bwd_last_query_tile(kt, n_tiles, window);
}
void sch_fwd_grid(int sms, int n_blocks, int BH, int persistent, int* hpw, int* n_waves) {
    gpt_attn::fwd_grid(sms, n_blocks, BH, persistent != 0, *hpw, *n_waves);
}
void sch_fwd_item(int hpw, int n_blocks, int BH, int cta, int k, int* bh, int* qb) {
    gpt_attn::fwd_item(hpw, n_blocks, BH, cta, k, *bh, *qb);
}
void sch_bwd_unit(int u, int n_tiles, int window, int* bh, int* kt, int* n_q) {
    gpt_attn::bwd_unit(u, n_tiles, window, *bh, *kt, *n_q);
}
int sch_tile() { return gpt_attn::kTile; }
int sch_row_lower(int i, int window, int doc_start_i) { return gpt_attn::row_lower(i, window, doc_start_i); }
void sch_fwd_key_range_lb(int qt, int first_row_lower, int* lo, int* hi) {
    gpt_attn::fwd_key_range_lb(qt, first_row_lower, *lo, *hi);
}
// The prep kernel's table entry for key tile kt: rows' lower bounds from `ds` (T entries) and window.
int sch_bwd_last_query_tile_lb(int kt, int n_tiles, int T, int window, const int* ds) {
    return gpt_attn::bwd_last_query_tile_lb(kt, n_tiles, [&](int qt) {
        const int i = qt * gpt_attn::kTile;
        return gpt_attn::row_lower(i, window, ds[i < T ? i : T - 1]);
    });
}
}
