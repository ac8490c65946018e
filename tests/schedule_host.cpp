// Host build of the kernels' work decomposition (causal_attention_sdpa_b200/csrc/schedule.h) for
// the CPU tests: C entry points over the same inline functions the kernels and launcher use.
#include "schedule.h"

extern "C" {
void sch_fwd_key_range(int qt, int window, int* lo, int* hi) { gpt_attn::fwd_key_range(qt, window, *lo, *hi); }
int sch_bwd_last_query_tile(int kt, int n_tiles, int window) {
    return gpt_attn::bwd_last_query_tile(kt, n_tiles, window);
}
int sch_tail_heads(int BH, int n_cls, int sms) { return gpt_attn::tail_heads(BH, n_cls, sms); }
void sch_list_item(int i, int BH, int n_cls, int tail, int* bh, int* cls) {
    gpt_attn::list_item(i, BH, n_cls, tail, *bh, *cls);
}
int sch_fwd_static_grid(int sms, int n_blocks, int BH, int* hpw, int* n_waves) {
    return gpt_attn::fwd_static_grid(sms, n_blocks, BH, *hpw, *n_waves) ? 1 : 0;
}
void sch_fwd_static_item(int hpw, int n_blocks, int BH, int cta, int k, int* bh, int* qb) {
    gpt_attn::fwd_static_item(hpw, n_blocks, BH, cta, k, *bh, *qb);
}
void sch_fwd_item(int i, int BH, int n_blocks, int tail, int* bh, int* qb) {
    gpt_attn::fwd_item(i, BH, n_blocks, tail, *bh, *qb);
}
void sch_bwd_unit(int u, int BH, int n_tiles, int tail, int window, int* bh, int* kt, int* n_q) {
    gpt_attn::bwd_unit(u, BH, n_tiles, tail, window, *bh, *kt, *n_q);
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
